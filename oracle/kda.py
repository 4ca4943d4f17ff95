"""Token-by-token gated delta-rule (KDA) recurrence in fp64 -- the definition.

The HARTS pages name KDA as the linear-attention layer of their hybrid
models (Table 1, "KDA:MLA per group") without its formula; the recurrence
used here is the one the workload fixes:

    S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
    o_t = S_t^T q_t

with g_t = log(alpha_t) per key channel, beta_t a scalar per (token, head),
S in R^{d_k x d_v}, independently per head.  Run trajectory by trajectory
(a root-to-leaf path of the rollout tree, HARTS Figure 1(a)).

Backward: the hand adjoint of one step, with M = Diag(exp(g_t)) S_{t-1}:
    dS_t += q_t dO_t^T;      dq_t = S_t dO_t
    dM   = dS_t - beta k (k^T dS_t)          dS_{t-1} = Diag(exp(g)) dM
    dg   = exp(g) * rowsum(dM * S_{t-1})
    dbeta = k^T dS_t (v - M^T k)
    dk   = beta (dS_t v - dS_t M^T k - M dS_t^T k)
    dv   = beta dS_t^T k
States are checkpointed every ``ckpt`` tokens and recomputed.
Arrays carry a leading head axis: q,k,g [T,H,dk], v [T,H,dv], beta [T,H].
"""
from __future__ import annotations

import numpy as np


def step(S, q, k, v, g, beta):
    """One token for all heads: returns (S_t, o_t, M)."""
    M = np.exp(g)[:, :, None] * S
    kM = np.einsum("hk,hkv->hv", k, M)
    S_new = M - beta[:, None, None] * k[:, :, None] * kM[:, None, :] + beta[:, None, None] * k[:, :, None] * v[:, None, :]
    o = np.einsum("hkv,hk->hv", S_new, q)
    return S_new, o, M


def forward(q, k, v, g, beta, S0=None):
    """o [T,H,dv] and the final state [H,dk,dv] of one trajectory."""
    T, H, dk = k.shape
    dv = v.shape[2]
    S = np.zeros((H, dk, dv)) if S0 is None else np.array(S0, np.float64)
    o = np.zeros((T, H, dv))
    for t in range(T):
        S, o[t], _ = step(S, q[t], k[t], v[t], g[t], beta[t])
    return o, S


def backward(q, k, v, g, beta, dO, dS_final=None, S0=None, ckpt=256):
    """Gradients of <dO, o> + <dS_final, S_T> for one trajectory.

    Returns dq, dk, dv, dg, dbeta (same shapes as the inputs) and dS0.
    """
    T, H, dk = k.shape
    dv_ = v.shape[2]
    S = np.zeros((H, dk, dv_)) if S0 is None else np.array(S0, np.float64)
    cps = {}
    for t in range(T):
        if t % ckpt == 0:
            cps[t] = S.copy()
        S, _, _ = step(S, q[t], k[t], v[t], g[t], beta[t])
    dS = np.zeros((H, dk, dv_)) if dS_final is None else np.array(dS_final, np.float64)
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dg = np.zeros_like(g)
    db = np.zeros_like(beta)
    starts = sorted(cps)
    for t0 in reversed(starts):
        t1 = min(T, t0 + ckpt)
        prev = [cps[t0]]  # prev[i] = S_{t0+i-1}
        for t in range(t0, t1):
            Sn, _, _ = step(prev[-1], q[t], k[t], v[t], g[t], beta[t])
            prev.append(Sn)
        for t in range(t1 - 1, t0 - 1, -1):
            Sp = prev[t - t0]
            St = prev[t - t0 + 1]
            e = np.exp(g[t])
            M = e[:, :, None] * Sp
            dS = dS + q[t][:, :, None] * dO[t][:, None, :]
            dq[t] = np.einsum("hkv,hv->hk", St, dO[t])
            kdS = np.einsum("hk,hkv->hv", k[t], dS)            # k^T dS      [H,dv]
            dM = dS - beta[t][:, None, None] * k[t][:, :, None] * kdS[:, None, :]
            Mk = np.einsum("hkv,hk->hv", M, k[t])              # M^T k       [H,dv]
            db[t] = np.einsum("hv,hv->h", kdS, v[t] - Mk)
            dS_v = np.einsum("hkv,hv->hk", dS, v[t])
            dS_Mk = np.einsum("hkv,hv->hk", dS, Mk)
            M_kdS = np.einsum("hkv,hv->hk", M, kdS)
            dkk[t] = beta[t][:, None] * (dS_v - dS_Mk - M_kdS)
            dvv[t] = beta[t][:, None] * kdS
            dg[t] = e * np.einsum("hkv,hkv->hk", dM, Sp)
            dS = e[:, :, None] * dM
    return dq, dkk, dvv, dg, db, dS


# --------------------------------------------------------------- whole tree, expanded
def tree_forward(tree, inputs, init=None):
    """Forward over every trajectory of ``tree`` (synth.Tree) with node-order ``inputs``.

    Returns o_unique [N,H,dv] (node order; checks that every occurrence of a
    row produced the same value) and final states [n_leaves,H,dk,dv].
    """
    q, k, v, g, beta = inputs
    N, H, _ = q.shape
    o_u = np.full((N, H, v.shape[2]), np.nan)
    finals = []
    for li, leaf in enumerate(tree.leaves()):
        rows = tree.trajectory_rows(leaf)
        root = tree.path(leaf)[0]
        S0 = None if init is None else init[root]
        o, S = forward(q[rows], k[rows], v[rows], g[rows], beta[rows], S0)
        seen = ~np.isnan(o_u[rows, 0, 0])
        if seen.any():
            assert np.allclose(o_u[rows[seen]], o[seen], rtol=1e-9, atol=1e-9)
        o_u[rows] = o
        finals.append(S)
    return o_u, np.stack(finals)


def tree_backward(tree, inputs, d_o_unique, d_final=None, init=None, ckpt=256):
    """Gradients w.r.t. the unique (node-order) inputs: the sum over all occurrences.

    The upstream output gradient is given per unique row and attached to the
    first trajectory (lowest leaf index) through that row; the loss is
    sum_u <d_o[u], o_u> + sum_leaves <d_final, S_final>.
    """
    q, k, v, g, beta = inputs
    grads = [np.zeros_like(x) for x in (q, k, v, g, beta)]
    n_roots = int(np.sum(tree.parent < 0))
    d_init = None
    taken = np.zeros(q.shape[0], bool)
    for li, leaf in enumerate(tree.leaves()):
        rows = tree.trajectory_rows(leaf)
        dO = np.where(taken[rows][:, None, None], 0.0, d_o_unique[rows])
        taken[rows] = True
        root = tree.path(leaf)[0]
        S0 = None if init is None else init[root]
        dF = None if d_final is None else d_final[li]
        res = backward(q[rows], k[rows], v[rows], g[rows], beta[rows], dO, dF, S0, ckpt)
        for G, r in zip(grads, res[:5]):
            np.add.at(G, rows, r)
        if d_init is None:
            d_init = np.zeros((tree.n,) + res[5].shape)
        d_init[root] += res[5]
    return grads + [d_init]


def expanded_forward(tree, inputs, init=None):
    """Per-trajectory outputs, concatenated in leaf order ([N_exp,H,dv])."""
    q, k, v, g, beta = inputs
    outs = []
    for leaf in tree.leaves():
        rows = tree.trajectory_rows(leaf)
        root = tree.path(leaf)[0]
        o, _ = forward(q[rows], k[rows], v[rows], g[rows], beta[rows], None if init is None else init[root])
        outs.append(o)
    return np.concatenate(outs)
