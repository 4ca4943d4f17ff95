"""Tree-masked attention on the GPU against the per-trajectory causal softmax oracle."""
import numpy as np
import pytest

import synth
from kda_case import TOL, err_ratio
from oracle import attention as oat

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpc():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


@pytest.mark.parametrize("cfg,H", [("fig1", 2), ("agentic_small", 2)])
def test_tree_attention_matches_oracle(tpc, cfg, H):
    import torch
    tree = synth.workload(cfg).tree
    N = tree.n_rows
    seed = 31
    q = synth.normal_tensor(seed, 40, (N, H, 192), "bf16")
    k = synth.normal_tensor(seed, 41, (N, H, 192), "bf16")
    v = synth.normal_tensor(seed, 42, (N, H, 128), "bf16")
    d_o = synth.normal_tensor(seed, 43, (N, H, 128), "bf16")
    scale = 1.0 / np.sqrt(192.0)
    o_ref, lse_ref = oat.tree_forward(tree, q, k, v, scale)
    dq_ref, dk_ref, dv_ref = oat.tree_backward(tree, q, k, v, scale, d_o)
    plan = tpc.Plan(tree.parent, tree.length, 64).upload()
    st = tree.node_start()
    dev = lambda a: torch.tensor(plan.to_compact(a, st, tree.length), dtype=torch.float32).to(torch.bfloat16).cuda()
    comp = lambda a: plan.to_compact(a, st, tree.length)
    qd, kd, vd, gd = dev(q), dev(k), dev(v), dev(d_o)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = tpc.tpc_tree_attn_forward(plan, qd, kd, vd, scale, out_dtype=torch.float32, status=status)
    dq, dk, dv = tpc.tpc_tree_attn_backward(plan, qd, kd, vd, o, lse, gd, scale, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    errs = {"o": err_ratio(o.cpu().numpy(), comp(o_ref)), "lse": err_ratio(lse.cpu().numpy(), comp(lse_ref)),
            "dq": err_ratio(dq.cpu().numpy(), comp(dq_ref)), "dk": err_ratio(dk.cpu().numpy(), comp(dk_ref)),
            "dv": err_ratio(dv.cpu().numpy(), comp(dv_ref))}
    print(cfg, errs)
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
    # rotary positions: the depth of every row on its trajectories
    pos = tpc.tpc_rope_positions(plan).cpu().numpy()
    depth = np.concatenate([np.arange(int(sum(tree.length[u] for u in tree.path(v)[:-1])),
                                      int(sum(tree.length[u] for u in tree.path(v))))
                            for v in range(tree.n)])
    assert np.array_equal(pos, comp(depth))


def test_tree_attention_split_inputs(tpc):
    """q, k, v and dO given as fp32 values in bf16 hi/lo pairs: results match the oracle on the fp32
    values (no bf16 rounding of any input)."""
    import torch
    tree = synth.workload("agentic_small").tree
    N, H = tree.n_rows, 2
    seed = 32
    q = synth.normal_tensor(seed, 40, (N, H, 192), "f32")
    k = synth.normal_tensor(seed, 41, (N, H, 192), "f32")
    v = synth.normal_tensor(seed, 42, (N, H, 128), "f32")
    d_o = synth.normal_tensor(seed, 43, (N, H, 128), "f32")
    scale = 1.0 / np.sqrt(192.0)
    o_ref, lse_ref = oat.tree_forward(tree, q, k, v, scale)
    dq_ref, dk_ref, dv_ref = oat.tree_backward(tree, q, k, v, scale, d_o)
    plan = tpc.Plan(tree.parent, tree.length, 64).upload()
    st = tree.node_start()
    comp = lambda a: plan.to_compact(a, st, tree.length)
    f32 = lambda a: torch.tensor(comp(a), dtype=torch.float32).cuda()
    qh, ql = tpc.split_bf16(f32(q))
    kh, kl = tpc.split_bf16(f32(k))
    vh, vl = tpc.split_bf16(f32(v))
    gh, gl = tpc.split_bf16(f32(d_o))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = tpc.tpc_tree_attn_forward(plan, qh, kh, vh, scale, out_dtype=torch.float32, status=status, q_lo=ql,
                                       k_lo=kl, v_lo=vl)
    dq, dk, dv = tpc.tpc_tree_attn_backward(plan, qh, kh, vh, o, lse, gh, scale, status=status, q_lo=ql, k_lo=kl,
                                            v_lo=vl, d_o_lo=gl)
    torch.cuda.synchronize()
    assert status.item() == 0
    errs = {"o": err_ratio(o.cpu().numpy(), comp(o_ref)), "lse": err_ratio(lse.cpu().numpy(), comp(lse_ref)),
            "dq": err_ratio(dq.cpu().numpy(), comp(dq_ref)), "dk": err_ratio(dk.cpu().numpy(), comp(dk_ref)),
            "dv": err_ratio(dv.cpu().numpy(), comp(dv_ref))}
    print("split", errs)
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


EDGE_TREES = {
    # one row: a single key tile of one row, one query tile, rows past the tensor end read as zero
    "single_row": ([-1], [1]),
    # a chain of one- to three-row nodes: every key tile ragged, queries of later nodes see all
    "short_chain": ([-1, 0, 1, 2, 3], [1, 2, 3, 1, 2]),
    # a star of one-row leaves under a 130-row root (key tiles of 128 + 2 rows, ragged query tiles)
    "star": ([-1] + [0] * 9, [130] + [1] * 9),
    # a root whose length is an exact multiple of the tile sizes, two children of one row and 64
    "aligned": ([-1, 0, 0], [256, 1, 64]),
}


@pytest.mark.parametrize("name", sorted(EDGE_TREES))
@pytest.mark.parametrize("H,split", [(1, False), (3, True)])
def test_tree_attention_edge_cases(tpc, name, H, split):
    """Degenerate and ragged trees (single row, one-row nodes, tile-aligned lengths) in both input
    forms: outputs and all gradients against the oracle."""
    import torch
    parent, length = EDGE_TREES[name]
    tree = synth.Tree(parent=np.array(parent, np.int32), length=np.array(length, np.int32))
    N = tree.n_rows
    seed = 33
    dt = "f32" if split else "bf16"
    q = synth.normal_tensor(seed, 40, (N, H, 192), dt)
    k = synth.normal_tensor(seed, 41, (N, H, 192), dt)
    v = synth.normal_tensor(seed, 42, (N, H, 128), dt)
    d_o = synth.normal_tensor(seed, 43, (N, H, 128), dt)
    scale = 1.0 / np.sqrt(192.0)
    o_ref, lse_ref = oat.tree_forward(tree, q, k, v, scale)
    dq_ref, dk_ref, dv_ref = oat.tree_backward(tree, q, k, v, scale, d_o)
    plan = tpc.Plan(tree.parent, tree.length, 64).upload()
    st = tree.node_start()
    comp = lambda a: plan.to_compact(a, st, tree.length)
    f32 = lambda a: torch.tensor(comp(a), dtype=torch.float32).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if split:
        (qh, ql), (kh, kl), (vh, vl), (gh, gl) = (tpc.split_bf16(f32(a)) for a in (q, k, v, d_o))
        lo = dict(q_lo=ql, k_lo=kl, v_lo=vl)
        o, lse = tpc.tpc_tree_attn_forward(plan, qh, kh, vh, scale, out_dtype=torch.float32, status=status, **lo)
        dq, dk, dv = tpc.tpc_tree_attn_backward(plan, qh, kh, vh, o, lse, gh, scale, status=status, d_o_lo=gl, **lo)
    else:
        qd, kd, vd, gd = (f32(a).to(torch.bfloat16) for a in (q, k, v, d_o))
        o, lse = tpc.tpc_tree_attn_forward(plan, qd, kd, vd, scale, out_dtype=torch.float32, status=status)
        dq, dk, dv = tpc.tpc_tree_attn_backward(plan, qd, kd, vd, o, lse, gd, scale, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    errs = {"o": err_ratio(o.cpu().numpy(), comp(o_ref)), "lse": err_ratio(lse.cpu().numpy(), comp(lse_ref)),
            "dq": err_ratio(dq.cpu().numpy(), comp(dq_ref)), "dk": err_ratio(dk.cpu().numpy(), comp(dk_ref)),
            "dv": err_ratio(dv.cpu().numpy(), comp(dv_ref))}
    print(name, H, split, errs)
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
