"""Deterministic top-k MoE routing over trajectory positions (oracle side): the expanded computation
that the compact routing with occurrence counts must reproduce.

HARTS pages: the abstract says that, for deterministic top-k routing without token dropping,
occurrence counts restore MoE objective weights and expert-load statistics; Figure 1: the
occurrence count q_B = 2 restores them without repeating routing or expert computation; Figure
C.1(d): compact routing uses multiplicity-weighted router losses and expert-load counts.  The pages
give no router or loss formulas; the plainest ones (Switch-style balance loss plus router z-loss):

  per position j with hidden row h_j:  z_j = W_r h_j (E logits),  p_j = softmax(z_j),
  lse_j = log sum exp z_j,  top-k experts of z_j (ties: lower expert index), gates = p_j on the top-k
  renormalised to sum 1;
  load_e  = number of positions routed to e (no dropping);   P_e = sum_j p_je;
  L_aux   = E / (k N^2) sum_e load_e P_e,   L_z = (1/N) sum_j lse_j^2,   L = a L_aux + b L_z
  (N = number of positions).  dL/dz_j = a E/(k N^2) p_j * (load - <load, p_j>) + b (2 lse_j / N) p_j,
  the top-k choice (and so load) being piecewise constant.

The top-k decision is taken in the kernel's precision: z_j in fp32 as a fixed-order sum over the
hidden dimension of separately rounded products (c = 0, 1, ..., D - 1), reproduced here exactly with
numpy float32; everything else is fp64.  Positions are processed one by one in the expanded layout
(trajectory by trajectory); nothing is shared between positions.

This module is test infrastructure: only tests and the benchmark's CPU baseline use it.
"""
from __future__ import annotations

import numpy as np


def router_logits_fp32(h, w):
    """z [n, E] in fp32: acc = fl(acc + fl(h_c w_c)) for c = 0 .. D-1 (h [n, D], w [E, D] exact in fp32)."""
    h = np.asarray(h, np.float32)
    w = np.asarray(w, np.float32)
    acc = np.zeros((h.shape[0], w.shape[0]), np.float32)
    for c in range(h.shape[1]):
        acc = (acc + (h[:, c:c + 1] * w[None, :, c]).astype(np.float32)).astype(np.float32)
    return acc


def topk_sorted(z, k):
    """Indices of the k largest entries of each row, larger first, ties to the lower index."""
    order = np.lexsort((np.broadcast_to(np.arange(z.shape[1]), z.shape), -z.astype(np.float64)), axis=1)
    return order[:, :k]


def route_expanded(h_pos, w, k):
    """Per position: logits (fp32), probabilities and lse (fp64), top-k experts and gates."""
    z = router_logits_fp32(h_pos, w)
    z64 = z.astype(np.float64)
    m = z64.max(axis=1, keepdims=True)
    e = np.exp(z64 - m)
    s = e.sum(axis=1, keepdims=True)
    p = e / s
    lse = (m + np.log(s))[:, 0]
    idx = topk_sorted(z, k)
    g = np.take_along_axis(p, idx, axis=1)
    g = g / g.sum(axis=1, keepdims=True)
    return z, p, lse, idx, g


def losses_expanded(p, lse, idx, E, k, a=1.0, b=1.0):
    """(load [E] int, P [E], L_aux, L_z, dz [n, E]) over the positions, the definitions above."""
    n = p.shape[0]
    load = np.zeros(E, np.int64)
    for j in range(n):
        for e in idx[j]:
            load[e] += 1
    P = p.sum(axis=0)
    alpha = E / (k * float(n) ** 2)
    l_aux = alpha * float(np.dot(load, P))
    l_z = float(np.mean(lse ** 2))
    dz = a * alpha * p * (load[None, :] - (p @ load)[:, None]) + b * (2.0 * lse / n)[:, None] * p
    return load, P, l_aux, l_z, dz


def expanded_then_unique(dz_pos, rows, n_unique):
    """Sum of the per-position gradients over the occurrences of each compact row."""
    out = np.zeros((n_unique, dz_pos.shape[1]))
    np.add.at(out, rows, dz_pos)
    return out
