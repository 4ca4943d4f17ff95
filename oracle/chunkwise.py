"""Chunkwise KDA form and the fp64 tree executor (oracle side).

Chunkwise form (derived from the recurrence in ``oracle.kda``): with the
chunk-local inclusive cumulative gate G_r = sum_{i<=r} g_i and the chunk's
last row G_C,
    Kbar = k*exp(G), Kbrv = k*exp(-G), Qbar = q*exp(G), Khat = k*exp(G_C - G)
    A = strict_lower(diag(beta) Kbar Kbrv^T),   T = (I + A)^{-1}
    W = T diag(beta) Kbar,   U' = T diag(beta) V,   U = U' - W S0
    O = Qbar S0 + lower_incl(Qbar Kbrv^T) U
    S_C = Diag(exp(G_C)) S0 + Khat^T U
Chunks are aligned to absolute trajectory positions (multiples of C).

Tree executor (HARTS Figure 2(c) and Figure C.1(b)): rounds run in order;
each round runs its sequences (continuation chains from the planner),
each starting from the initial state or from a boundary state exported by
an earlier round, replaying the tokens between the aligned boundary and its
own first token without writing outputs.
"""
from __future__ import annotations

import numpy as np

from . import planner as _planner


def chunk_step(S0, q, k, v, g, beta):
    """One chunk (rows = positions of the chunk), all heads. Returns (O, S_C)."""
    G = np.cumsum(g, axis=0)                     # [n,H,dk]
    GC = G[-1]                                   # [H,dk]
    Kbar = k * np.exp(G)
    Kbrv = k * np.exp(-G)
    Qbar = q * np.exp(G)
    Khat = k * np.exp(GC[None] - G)
    n = k.shape[0]
    low = np.tril(np.ones((n, n)), -1)
    lowi = np.tril(np.ones((n, n)), 0)
    A = np.einsum("rh,rhc,ihc->hri", beta, Kbar, Kbrv) * low[None]
    T = np.linalg.inv(np.eye(n)[None] + A)      # [H,n,n]
    W = np.einsum("hri,ih,ihc->hrc", T, beta, Kbar)
    Up = np.einsum("hri,ih,ihc->hrc", T, beta, v)
    U = Up - np.einsum("hrc,hcv->hrv", W, S0)
    P = np.einsum("rhc,ihc->hri", Qbar, Kbrv) * lowi[None]
    O = np.einsum("rhc,hcv->rhv", Qbar, S0) + np.einsum("hri,hiv->rhv", P, U)
    S = np.exp(GC)[:, :, None] * S0 + np.einsum("rhc,hrv->hcv", Khat, U)
    return O, S


def sequence_forward(S0, q, k, v, g, beta, start, C):
    """Chunkwise over positions start .. start+T-1 (start a multiple of C)."""
    T = k.shape[0]
    O = np.zeros((T,) + v.shape[1:])
    S = S0
    p = start
    states = {}
    while p < start + T:
        e = min((p // C + 1) * C, start + T)
        sl = slice(p - start, e - start)
        O[sl], S = chunk_step(S, q[sl], k[sl], v[sl], g[sl], beta[sl])
        states[e] = S
        p = e
    return O, S, states


def chunked_forward(q, k, v, g, beta, C, S0=None):
    H, dk = k.shape[1], k.shape[2]
    S0 = np.zeros((H, dk, v.shape[2])) if S0 is None else S0
    O, S, _ = sequence_forward(S0, q, k, v, g, beta, 0, C)
    return O, S


def tree_execute(tree, inputs, C, init=None):
    """Round-by-round tree execution in fp64.

    Returns o_unique (node order), final states per leaf (leaf order) and the plan.
    """
    q, k, v, g, beta = inputs
    N, H, dk = k.shape
    dv = v.shape[2]
    pl = _planner.plan(tree.parent, tree.length, C)
    assert pl.round.min() >= 1
    leaves = list(pl.leaves)
    o_u = np.full((N, H, dv), np.nan)
    finals = np.zeros((len(leaves), H, dk, dv))
    slot_state = {}
    exports = {}
    for sid, sl in enumerate(pl.slots):
        exports.setdefault(sl["producer_seq"], {})[sl["b"]] = sid
    for r in range(1, pl.n_rounds + 1):
        for si, sq in enumerate(pl.seqs):
            if sq["round"] != r:
                continue
            if sq["import_kind"] == "slot":
                S0 = slot_state[sq["import_id"]]
            else:
                S0 = np.zeros((H, dk, dv)) if init is None else init[sq["import_id"]]
            rows = tree.trajectory_rows(sq["leaf"])[sq["start"]:sq["end"]]
            O, S, states = sequence_forward(S0, q[rows], k[rows], v[rows], g[rows], beta[rows], sq["start"], C)
            own = sq["replay"]
            o_u[rows[own:]] = O[own:]
            for bpos, sid in exports.get(si, {}).items():
                slot_state[sid] = states[bpos]
            finals[leaves.index(sq["leaf"])] = S
    return o_u, finals, pl
