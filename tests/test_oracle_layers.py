"""Pins of the hybrid layer-group oracle (oracle.layers) against facts that do not come from it:
numerical derivatives, per-trajectory runs of the same group, closed forms of its pieces."""
import numpy as np
import torch

import synth
from oracle import layers as ol

TINY = ol.Dims(D=16, H=2, d_head=8, d_rope=4, d_latent=8)


def tiny_weights(seed, dims, n_kda, scale=0.3):
    rng = np.random.default_rng(seed)
    w = lambda o, i: rng.normal(0, scale, (o, i))
    return {"kda": [(w(dims.kda_proj, dims.D), w(dims.D, dims.D)) for _ in range(n_kda)],
            "mla": (w(dims.mla_proj, dims.D), w(2 * dims.D, dims.d_latent), w(dims.D, dims.D))}


def loss(tree, x, weights, dy, dims):
    y, _ = ol.group_forward(tree, x, weights, dims)
    return float((y * dy).sum())


def test_group_gradients_match_central_differences():
    """Directional derivatives of the fp64 group on the worked-example tree."""
    tree = synth.fig1_tree()
    rng = np.random.default_rng(1)
    N = tree.n_rows
    x = rng.normal(size=(N, TINY.D))
    dy = rng.normal(size=(N, TINY.D))
    weights = tiny_weights(2, TINY, n_kda=2)
    _, dx, dw, _ = ol.group_backward(tree, x, weights, dy, TINY)
    eps = 1e-5

    def check(analytic, perturb):
        u = rng.normal(size=analytic.shape)
        num = (loss(tree, *perturb(eps * u), dy, TINY) - loss(tree, *perturb(-eps * u), dy, TINY)) / (2 * eps)
        ana = float((analytic * u).sum())
        assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), (num, ana)

    check(dx, lambda d: (x + d, weights))
    for li in range(2):
        for wi in range(2):
            def pert(d, li=li, wi=wi):
                kda = [list(p) for p in weights["kda"]]
                kda[li][wi] = kda[li][wi] + d
                return x, {"kda": [tuple(p) for p in kda], "mla": weights["mla"]}
            check(dw["kda"][li][wi], pert)
    for wi in range(3):
        def pert(d, wi=wi):
            mla = list(weights["mla"])
            mla[wi] = mla[wi] + d
            return x, {"kda": weights["kda"], "mla": tuple(mla)}
        check(dw["mla"][wi], pert)


def test_tree_group_equals_each_trajectory_alone():
    """Running the group once on the tree gives every trajectory what it gets when run alone as a
    chain (HARTS Figure 1), and the tree's gradients are the sums of the trajectories' gradients
    under the expanded loss sum_j <y_j, R_j>."""
    tree = synth.fig1_tree()
    rng = np.random.default_rng(3)
    x = rng.normal(size=(tree.n_rows, TINY.D))
    weights = tiny_weights(4, TINY, n_kda=1)
    R = rng.normal(size=(tree.n_expanded(), TINY.D))
    y, dx, dw, _ = ol.group_backward(tree, x, weights, ol.occurrence_sum(tree, R), TINY)
    dx_sum = np.zeros_like(dx)
    dw_sum = None
    j = 0
    for leaf in tree.leaves():
        rows = tree.trajectory_rows(leaf)
        chain = synth.Tree(parent=np.array([-1], np.int32), length=np.array([len(rows)], np.int32))
        yt, dxt, dwt, _ = ol.group_backward(chain, x[rows], weights, R[j:j + len(rows)], TINY)
        j += len(rows)
        assert np.allclose(yt, y[rows], rtol=0, atol=1e-12)
        np.add.at(dx_sum, rows, dxt)
        flat = [w for p in dwt["kda"] for w in p] + list(dwt["mla"])
        dw_sum = flat if dw_sum is None else [a + b for a, b in zip(dw_sum, flat)]
    assert np.allclose(dx_sum, dx, rtol=0, atol=1e-10)
    for a, b in zip(dw_sum, [w for p in dw["kda"] for w in p] + list(dw["mla"])):
        assert np.allclose(a, b, rtol=0, atol=1e-9 * max(1.0, np.abs(b).max()))


def test_rmsnorm_closed_form():
    x = torch.tensor([[3.0, 4.0], [0.0, 0.0], [1e-3, -1e-3]], dtype=torch.float64)
    y = ol.rmsnorm(x, 1e-6)
    # mean square 12.5 -> y = x / sqrt(12.5 + 1e-6); a zero row stays zero
    assert torch.allclose(y[0], x[0] / np.sqrt(12.5 + 1e-6), rtol=1e-15)
    assert torch.equal(y[1], torch.zeros(2, dtype=torch.float64))
    assert torch.allclose(y[2], x[2] / np.sqrt(1e-6 + 1e-6), rtol=1e-15)


def test_rope_properties():
    pos = torch.tensor([0, 1, 7, 12345], dtype=torch.int64)
    rng = np.random.default_rng(5)
    a = torch.tensor(rng.normal(size=(4, 3, 64)))
    b = torch.tensor(rng.normal(size=(4, 3, 64)))
    ra = ol.rope(a, pos, 10000.0)
    assert torch.equal(ra[0], a[0])  # position 0 is the identity
    assert torch.allclose(ra.norm(dim=-1), a.norm(dim=-1), rtol=1e-14)  # a rotation
    # scores depend on the position difference only: <R(p) a, R(p') b> = <R(p - p') a, b>
    rb = ol.rope(b, pos.flip(0), 10000.0)
    lhs = (ra * rb).sum(-1)
    rel = ol.rope(a, pos - pos.flip(0), 10000.0)
    assert torch.allclose(lhs, (rel * b).sum(-1), rtol=1e-10, atol=1e-10)
    # the first pair turns by exactly pos radians, the last pair by pos * 10000^(-31/32)
    e = torch.zeros(2, 1, 64, dtype=torch.float64)
    e[:, 0, 0] = 1.0
    e[:, 0, 31] = 1.0
    r = ol.rope(e, torch.tensor([1, 2]), 10000.0)
    for i, p in enumerate((1, 2)):
        assert np.isclose(r[i, 0, 0], np.cos(p)) and np.isclose(r[i, 0, 32], np.sin(p))
        th = p * 10000.0 ** (-62.0 / 64.0)
        assert np.isclose(r[i, 0, 31], np.cos(th)) and np.isclose(r[i, 0, 63], np.sin(th))


def test_depth_positions_count_along_every_trajectory():
    for tree in (synth.fig1_tree(), synth.workload("agentic_small").tree):
        pos = ol.depth_positions(tree)
        for leaf in tree.leaves():
            rows = tree.trajectory_rows(leaf)
            assert np.array_equal(pos[rows], np.arange(len(rows)))


def test_kda_layer_gate_and_norm_values():
    """One-hot rows make each projection pick one weight column: the gate, beta and key norm
    then take known values (softplus(0) = ln 2, sigmoid(0) = 1/2, softplus(z) ~ z for large z)."""
    d = TINY
    tree = synth.Tree(parent=np.array([-1], np.int32), length=np.array([3], np.int32))
    x = np.zeros((3, d.D))
    x[:, 0] = 1.0
    s = 1.0 / np.sqrt(1.0 / d.D + d.eps)  # RMSNorm of a one-hot row
    w_in = np.zeros((d.kda_proj, d.D))
    z = np.array([0.0, 30.0, -30.0, 2.0])
    w_in[3 * d.D:3 * d.D + 4, 0] = z / s            # gate channels 0..3 of head 0
    w_in[4 * d.D:4 * d.D + 2, 0] = np.array([0.0, 3.0]) / s  # beta of heads 0, 1
    w_in[d.D:2 * d.D, 0] = np.arange(1, d.D + 1)    # key projections (any scale)
    parts = {}
    ol.kda_layer(tree, torch.tensor(x), torch.tensor(w_in), torch.zeros(d.D, d.D, dtype=torch.float64), d,
                 parts=parts)
    g = parts["g"][0, 0, :4].numpy()
    assert np.allclose(g, [-0.1 * np.log(2.0), -3.0, 0.0, -0.1 * np.log(1 + np.exp(2.0))], atol=1e-12)
    assert np.allclose(parts["beta"][0].numpy(), [0.5, 1 / (1 + np.exp(-3.0))], atol=1e-15)
    assert np.allclose(parts["k"].norm(dim=-1).numpy(), 1.0, atol=1e-9)


def test_mla_scores_equal_the_absorbed_latent_form():
    """Decompressed no-position scores q_h . k_h equal (W_uk,h^T q_h) . c: keys are a linear
    image of the latent, so the product can be taken in latent space."""
    d = TINY
    tree = synth.fig1_tree()
    rng = np.random.default_rng(6)
    x = torch.tensor(rng.normal(size=(tree.n_rows, d.D)))
    w = tiny_weights(7, d, 0)["mla"]
    parts = {}
    pos = torch.from_numpy(ol.depth_positions(tree))
    ol.mla_layer(tree, pos, x, *(torch.tensor(a) for a in w), d, parts=parts)
    c = parts["c"]
    for h in range(d.H):
        qn = parts["q"][:, h, :d.d_head]
        kn = parts["k"][:, h, :d.d_head]
        w_uk = torch.tensor(w[1][h * d.d_head:(h + 1) * d.d_head])
        assert torch.allclose(qn @ kn.T, (qn @ w_uk) @ c.T, rtol=1e-10, atol=1e-10)
        # every head sees the same rotary key
        assert torch.equal(parts["k"][:, h, d.d_head:], parts["kr"])
