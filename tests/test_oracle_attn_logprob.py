"""Pins for the attention and log-probability oracles."""
import numpy as np
import pytest

import synth
from oracle import attention, logprob


def test_single_token_attention_returns_value():
    rng = np.random.default_rng(0)
    q, k, v = rng.standard_normal((1, 3, 8)), rng.standard_normal((1, 3, 8)), rng.standard_normal((1, 3, 5))
    o, lse = attention.causal_forward(q, k, v, 0.3)
    assert np.allclose(o, v) and np.allclose(lse, 0.3 * np.sum(q * k, -1))


def test_attention_matches_library_sdpa():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    T, H, d, dv = 19, 3, 8, 6
    q, k, v = rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d)), rng.standard_normal((T, H, dv))
    o, _ = attention.causal_forward(q, k, v, 0.25)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.tensor(x).permute(1, 0, 2) for x in (q, k, v)), is_causal=True, scale=0.25).permute(1, 0, 2)
    assert np.allclose(o, ref.numpy(), atol=1e-13)


def test_attention_backward_finite_differences():
    rng = np.random.default_rng(2)
    T, H, d, dv = 5, 2, 3, 2
    q, k, v = rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d)), rng.standard_normal((T, H, dv))
    dO = rng.standard_normal((T, H, dv))
    grads = attention.causal_backward(q, k, v, 0.7, dO)
    h = 1e-6
    for which, base in enumerate((q, k, v)):
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            a = [x.copy() for x in (q, k, v)]
            b = [x.copy() for x in (q, k, v)]
            a[which][idx] += h
            b[which][idx] -= h
            num[idx] = (np.sum(attention.causal_forward(*a, 0.7)[0] * dO) -
                        np.sum(attention.causal_forward(*b, 0.7)[0] * dO)) / (2 * h)
        assert np.abs(num - grads[which]).max() < 1e-8 * max(1.0, np.abs(num).max())


def test_tree_attention_rows_consistent_and_grad():
    t = synth.Tree(np.array([-1, 0, 0, 1, 1], np.int32), np.array([3, 2, 2, 1, 2], np.int32))
    rng = np.random.default_rng(3)
    N, H, d = t.n_rows, 2, 4
    q, k, v = rng.standard_normal((N, H, d)), rng.standard_normal((N, H, d)), rng.standard_normal((N, H, d))
    o, _ = attention.tree_forward(t, q, k, v, 0.5)
    assert not np.isnan(o).any()
    d_o = rng.standard_normal((N, H, d))
    grads = attention.tree_backward(t, q, k, v, 0.5, d_o)
    h = 1e-6
    for which in range(3):
        base = (q, k, v)[which]
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            a = [x.copy() for x in (q, k, v)]
            b = [x.copy() for x in (q, k, v)]
            a[which][idx] += h
            b[which][idx] -= h
            num[idx] = (np.sum(attention.tree_forward(t, *a, 0.5)[0] * d_o) -
                        np.sum(attention.tree_forward(t, *b, 0.5)[0] * d_o)) / (2 * h)
        assert np.abs(num - grads[which]).max() < 1e-8 * max(1.0, np.abs(num).max())


def test_logprob_matches_library_log_softmax_and_normalises():
    from scipy.special import log_softmax
    rng = np.random.default_rng(4)
    N, D, V = 6, 5, 11
    h, W = rng.standard_normal((N, D)), rng.standard_normal((V, D))
    rows = np.array([0, 0, 1, 3, 3, 3, 5])
    tg = np.array([1, 4, 10, 0, 0, 7, 2])
    logp, lse = logprob.forward(h, W, rows, tg)
    ref = log_softmax(h @ W.T, axis=1)
    assert np.allclose(logp, ref[rows, tg], atol=1e-13)
    full, _ = logprob.forward(h, W, np.repeat(np.arange(N), V), np.tile(np.arange(V), N))
    assert np.allclose(np.exp(full).reshape(N, V).sum(1), 1.0)
    assert logp[3] == logp[4]  # same row, same target -> same value
    assert np.array_equal(logprob.occurrence_counts(rows, N), [2, 1, 0, 3, 0, 1])


def test_logprob_backward_finite_differences():
    rng = np.random.default_rng(5)
    N, D, V = 4, 3, 7
    h, W = rng.standard_normal((N, D)), rng.standard_normal((V, D))
    rows = np.array([0, 1, 1, 3, 2, 0])
    tg = np.array([6, 0, 3, 3, 5, 6])
    w = rng.standard_normal(rows.shape[0])
    dh, dW = logprob.backward(h, W, rows, tg, w)
    e = 1e-6
    for base, g in ((h, dh), (W, dW)):
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            base[idx] += e
            a = np.sum(logprob.forward(h, W, rows, tg)[0] * w)
            base[idx] -= 2 * e
            b = np.sum(logprob.forward(h, W, rows, tg)[0] * w)
            base[idx] += e
            num[idx] = (a - b) / (2 * e)
        assert np.abs(num - g).max() < 1e-8
