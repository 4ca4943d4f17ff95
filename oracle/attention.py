"""Tree-masked softmax attention in fp64 (oracle side).

HARTS Figure 1(b): full attention reads ancestor keys and values;
Figure C.1(c): a query in segment B reads the rows of B's ancestors and,
within B, only earlier rows (causal diagonal blocks).  Along any
trajectory this is exactly causal softmax attention over that
trajectory's prefix, so the oracle runs textbook causal attention per
trajectory and checks that rows shared by several trajectories agree.

Backward (textbook): P = softmax(scale Q K^T) (causal), dV = P^T dO,
dP = dO V^T, dS = P * (dP - rowsum(dO * O)), dQ = scale dS K,
dK = scale dS^T Q.
"""
from __future__ import annotations

import numpy as np


def causal_forward(q, k, v, scale):
    """q,k [T,H,d], v [T,H,dv] -> o [T,H,dv], lse [T,H]."""
    T, H, _ = q.shape
    o = np.zeros((T, H, v.shape[2]))
    lse = np.zeros((T, H))
    mask = np.tril(np.ones((T, T), bool))
    for h in range(H):
        s = scale * (q[:, h] @ k[:, h].T)
        s = np.where(mask, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        o[:, h] = (p / l) @ v[:, h]
        lse[:, h] = (m + np.log(l))[:, 0]
    return o, lse


def causal_backward(q, k, v, scale, dO):
    T, H, _ = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    mask = np.tril(np.ones((T, T), bool))
    for h in range(H):
        s = np.where(mask, scale * (q[:, h] @ k[:, h].T), -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o = p @ v[:, h]
        dv[:, h] = p.T @ dO[:, h]
        dp = dO[:, h] @ v[:, h].T
        ds = p * (dp - np.sum(dO[:, h] * o, axis=1, keepdims=True))
        dq[:, h] = scale * ds @ k[:, h]
        dk[:, h] = scale * ds.T @ q[:, h]
    return dq, dk, dv


def tree_forward(tree, q, k, v, scale):
    """Node-order rows -> o [N,H,dv], lse [N,H]; every occurrence of a row must agree."""
    N, H, _ = q.shape
    o_u = np.full((N, H, v.shape[2]), np.nan)
    lse_u = np.full((N, H), np.nan)
    for leaf in tree.leaves():
        rows = tree.trajectory_rows(leaf)
        o, lse = causal_forward(q[rows], k[rows], v[rows], scale)
        seen = ~np.isnan(lse_u[rows, 0])
        if seen.any():
            assert np.allclose(o_u[rows[seen]], o[seen], rtol=1e-9, atol=1e-9)
        o_u[rows] = o
        lse_u[rows] = lse
    return o_u, lse_u


def tree_backward(tree, q, k, v, scale, d_o_unique):
    """Gradients of sum_u <d_o[u], o_u> w.r.t. node-order q, k, v (first-occurrence convention)."""
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    taken = np.zeros(q.shape[0], bool)
    for leaf in tree.leaves():
        rows = tree.trajectory_rows(leaf)
        dO = np.where(taken[rows][:, None, None], 0.0, d_o_unique[rows])
        taken[rows] = True
        a, b, c = causal_backward(q[rows], k[rows], v[rows], scale, dO)
        np.add.at(dq, rows, a)
        np.add.at(dk, rows, b)
        np.add.at(dv, rows, c)
    return dq, dk, dv
