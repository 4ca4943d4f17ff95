"""Per-position log-probability recovery in fp64 (oracle side).

HARTS abstract: log-probabilities are recovered for each original
trajectory position; Figure 1 caption: one logit row z_B supplies the
distinct target log-probabilities of every trajectory through B;
Figure C.1(d): mapped log-probabilities restore the original token order
without expanded vocabulary-sized logits.

Definition: for unique row u with hidden state h_u and output matrix W
[V, D]: z_u = W h_u, lse_u = log sum_j exp(z_u[j]); for every occurrence
(trajectory t, position j) of row u with target y:  logp = z_u[y] - lse_u.
Backward of L = sum_occ w_occ logp_occ:
  dz_u = sum_occ w_occ (onehot(y_occ) - softmax(z_u)),  dh_u = W^T dz_u,
  dW = sum_u dz_u h_u^T.
Occurrence count q_u = number of occurrences of row u.
"""
from __future__ import annotations

import numpy as np


def forward(h, W, occ_row, occ_target):
    """h [N,D], W [V,D], occ_row/occ_target [M] -> logp [M], lse [N]."""
    z = h @ W.T
    m = z.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0]
    logp = z[occ_row, occ_target] - lse[occ_row]
    return logp, lse


def backward(h, W, occ_row, occ_target, d_logp):
    z = h @ W.T
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    N = h.shape[0]
    wsum = np.zeros(N)
    np.add.at(wsum, occ_row, d_logp)
    dz = -wsum[:, None] * p
    np.add.at(dz, (occ_row, occ_target), d_logp)
    return dz @ W, dz.T @ h


def occurrence_counts(occ_row, n_rows):
    q = np.zeros(n_rows, np.int64)
    np.add.at(q, occ_row, 1)
    return q
