"""Pins for the fp64 KDA oracle: closed forms, special cases that reduce to
textbook routines, finite differences, an independent autograd derivative,
and the chunkwise / tree invariants."""
import numpy as np
import pytest

import synth
from oracle import kda, chunkwise

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def rand_inputs(rng, T, H, dk, dv, normalize=True, gscale=0.3):
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if normalize:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    g = -gscale * np.log1p(np.exp(rng.standard_normal((T, H, dk))))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    return q, k, v, g, beta


def test_single_token_closed_form():
    rng = np.random.default_rng(1)
    q, k, v, g, beta = rand_inputs(rng, 1, 2, 4, 3)
    o, S = kda.forward(q, k, v, g, beta)
    # from the zero state one token writes beta k v^T and reads it with q
    for h in range(2):
        assert np.allclose(o[0, h], beta[0, h] * np.dot(q[0, h], k[0, h]) * v[0, h], atol=1e-14)
        assert np.allclose(S[h], beta[0, h] * np.outer(k[0, h], v[0, h]), atol=1e-14)


def test_pure_decay():
    rng = np.random.default_rng(2)
    T, H, dk, dv = 7, 2, 4, 3
    q, k, v, g, _ = rand_inputs(rng, T, H, dk, dv)
    beta = np.zeros((T, H))
    S0 = rng.standard_normal((H, dk, dv))
    o, S = kda.forward(q, k, v, g, beta, S0)
    G = np.cumsum(g, axis=0)
    assert np.allclose(S, np.exp(G[-1])[:, :, None] * S0, atol=1e-13)
    for t in range(T):
        St = np.exp(G[t])[:, :, None] * S0
        assert np.allclose(o[t], np.einsum("hkv,hk->hv", St, q[t]), atol=1e-13)


def test_reduces_to_causal_linear_attention():
    # g = 0, beta = 1 and orthonormal keys: (I - k k^T) S = S, so o_t = sum_{i<=t} (q_t . k_i) v_i
    rng = np.random.default_rng(3)
    T, dk, dv = 6, 8, 5
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:T][:, None, :]
    q = rng.standard_normal((T, 1, dk))
    v = rng.standard_normal((T, 1, dv))
    o, _ = kda.forward(q, k, v, np.zeros((T, 1, dk)), np.ones((T, 1)))
    scores = np.tril(q[:, 0] @ k[:, 0].T)
    assert np.allclose(o[:, 0], scores @ v[:, 0], atol=1e-13)


def test_overwrite_with_repeated_unit_key():
    rng = np.random.default_rng(4)
    T, dk, dv = 5, 4, 3
    kk = rng.standard_normal(dk)
    kk /= np.linalg.norm(kk)
    k = np.tile(kk, (T, 1, 1))
    v = rng.standard_normal((T, 1, dv))
    S0 = rng.standard_normal((1, dk, dv))
    _, S = kda.forward(rng.standard_normal((T, 1, dk)), k, v, np.zeros((T, 1, dk)), np.ones((T, 1)), S0)
    expect = np.outer(kk, v[-1, 0]) + (np.eye(dk) - np.outer(kk, kk)) @ S0[0]
    assert np.allclose(S[0], expect, atol=1e-13)


def _loss(inputs, dO, dSf, S0):
    o, S = kda.forward(*inputs, S0)
    return np.sum(o * dO) + np.sum(S * dSf)


@pytest.mark.parametrize("ckpt", [2, 1000])
def test_backward_finite_differences(ckpt):
    rng = np.random.default_rng(5)
    T, H, dk, dv = 6, 2, 4, 3
    inputs = list(rand_inputs(rng, T, H, dk, dv, normalize=False))
    S0 = rng.standard_normal((H, dk, dv))
    dO = rng.standard_normal((T, H, dv))
    dSf = rng.standard_normal((H, dk, dv))
    grads = kda.backward(*inputs, dO, dSf, S0, ckpt=ckpt)
    h = 1e-6
    for which in range(6):
        base = inputs[which] if which < 5 else S0
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            def f(delta):
                b2 = base.copy()
                b2[idx] += delta
                ins = list(inputs)
                s0 = S0
                if which < 5:
                    ins[which] = b2
                else:
                    s0 = b2
                return _loss(ins, dO, dSf, s0)
            num[idx] = (f(h) - f(-h)) / (2 * h)
        err = np.abs(num - grads[which]).max() / (np.abs(num).max() + 1e-30)
        assert err < 1e-7, (which, err)


def test_backward_matches_autograd():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(6)
    T, H, dk, dv = 9, 2, 5, 4
    inputs = rand_inputs(rng, T, H, dk, dv)
    dO = rng.standard_normal((T, H, dv))
    dSf = rng.standard_normal((H, dk, dv))
    tq, tk, tv, tg, tb = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in inputs]
    S = torch.zeros(H, dk, dv, dtype=torch.float64)
    outs = []
    eye = torch.eye(dk, dtype=torch.float64)
    for t in range(T):
        kt = tk[t]
        P = eye[None] - tb[t][:, None, None] * kt[:, :, None] * kt[:, None, :]
        S = P @ (torch.exp(tg[t])[:, :, None] * S) + tb[t][:, None, None] * kt[:, :, None] * tv[t][:, None, :]
        outs.append(torch.einsum("hkv,hk->hv", S, tq[t]))
    L = (torch.stack(outs) * torch.tensor(dO)).sum() + (S * torch.tensor(dSf)).sum()
    L.backward()
    mine = kda.backward(*inputs, dO, dSf)
    for a, b in zip(mine[:5], (tq, tk, tv, tg, tb)):
        assert np.allclose(a, b.grad.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("C", [1, 2, 3, 5, 16, 64, 1000])
def test_chunkwise_equals_recurrent(C):
    rng = np.random.default_rng(7)
    T, H, dk, dv = 70, 2, 8, 6
    inputs = rand_inputs(rng, T, H, dk, dv)
    S0 = rng.standard_normal((H, dk, dv))
    o, S = kda.forward(*inputs, S0)
    oc, Sc = chunkwise.chunked_forward(*inputs, C, S0)
    rms = np.sqrt(np.mean(o ** 2))
    assert np.abs(oc - o).max() <= 1e-12 * rms
    assert np.abs(Sc - S).max() <= 1e-12 * np.sqrt(np.mean(S ** 2))


@pytest.mark.parametrize("cfg,C", [("fig1", 16), ("fig1", 5), ("agentic_small", 64)])
def test_tree_executor_equals_expanded(cfg, C):
    w = synth.workload(cfg)
    t = w.tree
    H, d = (w.H, w.dk) if cfg == "fig1" else (2, 16)
    inputs = synth.kda_inputs(w.seed, np.arange(t.n_rows), H, d, d, w.dtype)
    o_e, fin_e = kda.tree_forward(t, inputs)
    o_t, fin_t, _ = chunkwise.tree_execute(t, inputs, C)
    assert not np.isnan(o_t).any()
    assert np.abs(o_t - o_e).max() <= 1e-12 * np.sqrt(np.mean(o_e ** 2))
    assert np.abs(fin_t - fin_e).max() <= 1e-12 * np.sqrt(np.mean(fin_e ** 2))


def test_tree_backward_finite_differences():
    # tiny version of the Figure 1 tree; gradients w.r.t. unique rows sum over occurrences
    t = synth.Tree(np.array([-1, 0, 0, 1, 1], np.int32), np.array([3, 2, 2, 1, 2], np.int32))
    rng = np.random.default_rng(8)
    N, H, dk, dv = t.n_rows, 1, 3, 2
    inputs = list(rand_inputs(rng, N, H, dk, dv, normalize=False))
    d_o = rng.standard_normal((N, H, dv))
    dF = rng.standard_normal((len(t.leaves()), H, dk, dv))
    grads = kda.tree_backward(t, inputs, d_o, dF)

    def L(ins):
        o, fin = kda.tree_forward(t, ins)
        return np.sum(o * d_o) + np.sum(fin * dF)

    h = 1e-6
    for which in range(5):
        num = np.zeros_like(inputs[which])
        for idx in np.ndindex(num.shape):
            a = [x.copy() for x in inputs]
            b = [x.copy() for x in inputs]
            a[which][idx] += h
            b[which][idx] -= h
            num[idx] = (L(a) - L(b)) / (2 * h)
        assert np.abs(num - grads[which]).max() <= 1e-7 * np.abs(num).max(), which
