"""Pins of the MoE routing oracle (oracle/moe.py) against closed forms, the fp32 error bound and
finite differences.  CPU only."""
import numpy as np

from oracle import moe


def test_router_logits_within_fp32_bound():
    rng = np.random.default_rng(0)
    h = rng.standard_normal((20, 300)).astype(np.float32)
    w = (0.05 * rng.standard_normal((16, 300))).astype(np.float32)
    z = moe.router_logits_fp32(h, w)
    exact = h.astype(np.float64) @ w.astype(np.float64).T
    bound = 300 * 2.0 ** -23 * (np.abs(h).astype(np.float64) @ np.abs(w).astype(np.float64).T)
    assert np.all(np.abs(z - exact) <= bound)
    assert z.dtype == np.float32


def test_uniform_router_closed_form():
    """Zero router weights: every position sees p = 1/E, the top-k are experts 0 .. k-1 (ties to
    the lower index), all n positions load them, L_aux = E/(k n^2) * (k n) * (n/E) = 1 and
    L_z = (log E)^2."""
    E, k, n = 8, 2, 13
    h = np.ones((n, 5), np.float32)
    w = np.zeros((E, 5), np.float32)
    z, p, lse, idx, g = moe.route_expanded(h, w, k)
    assert np.array_equal(idx, np.tile([0, 1], (n, 1)))
    assert np.allclose(g, 0.5) and np.allclose(p, 1.0 / E)
    load, P, l_aux, l_z, dz = moe.losses_expanded(p, lse, idx, E, k)
    assert list(load) == [n, n] + [0] * (E - 2)
    assert abs(l_aux - 1.0) < 1e-12 and abs(l_z - np.log(E) ** 2) < 1e-12


def test_topk_order_and_ties():
    z = np.array([[1.0, 3.0, 3.0, 2.0, 3.0]], np.float32)
    assert list(moe.topk_sorted(z, 3)[0]) == [1, 2, 4]
    assert list(moe.topk_sorted(z, 4)[0]) == [1, 2, 4, 3]


def test_loss_gradient_finite_differences():
    """dL/dz of a L_aux + b L_z with the routing held fixed (top-k is piecewise constant)."""
    rng = np.random.default_rng(1)
    n, E, k, a, b = 9, 6, 2, 0.7, 0.3
    z = rng.standard_normal((n, E))
    idx = moe.topk_sorted(z.astype(np.float32), k)

    def loss(zz):
        m = zz.max(axis=1, keepdims=True)
        e = np.exp(zz - m)
        p = e / e.sum(axis=1, keepdims=True)
        lse = (m + np.log(e.sum(axis=1, keepdims=True)))[:, 0]
        _, _, la, lz, _ = moe.losses_expanded(p, lse, idx, E, k, a, b)
        return a * la + b * lz

    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    p = e / e.sum(axis=1, keepdims=True)
    lse = (m + np.log(e.sum(axis=1, keepdims=True)))[:, 0]
    dz = moe.losses_expanded(p, lse, idx, E, k, a, b)[4]
    fd = np.zeros_like(z)
    eps = 1e-6
    for i in range(n):
        for j in range(E):
            zp, zm = z.copy(), z.copy()
            zp[i, j] += eps
            zm[i, j] -= eps
            fd[i, j] = (loss(zp) - loss(zm)) / (2 * eps)
    assert np.max(np.abs(fd - dz)) <= 1e-7 * max(1.0, np.max(np.abs(dz)))


def test_unique_sum_equals_expanded_sum():
    dz = np.arange(12.0).reshape(6, 2)
    rows = np.array([0, 2, 0, 1, 2, 2])
    out = moe.expanded_then_unique(dz, rows, 3)
    assert np.array_equal(out, [[0 + 4, 1 + 5], [6, 7], [2 + 8 + 10, 3 + 9 + 11]])
