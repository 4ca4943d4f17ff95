"""Compact top-k MoE routing with occurrence counts (HARTS abstract; Figure 1: q_B; Figure C.1(d)) on
the GPU against the expanded computation of the oracle: every trajectory position routed on its own.
The router logits and top-k decisions are bit-exact (both sides use the kernel's fixed-order fp32
sum), expert loads are exact integers, and the occurrence-weighted losses and logit gradients match
the position-by-position fp64 values to fp32 accuracy."""
import numpy as np
import pytest

import synth
from kda_case import err_ratio
from oracle import moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpc():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def bf16(x):
    return synth.round_to(x, "bf16").astype(np.float64)


@pytest.mark.parametrize("E,k", [(16, 2), (64, 8)])
def test_compact_routing_equals_expanded(tpc, E, k):
    import torch
    w = synth.workload("agentic_small")
    t = w.tree
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    N, NE, Dh = plan.info["n_unique"], plan.info["n_expanded"], 256
    h = bf16(synth.normal_tensor(61, synth.STREAM["h"], (N, Dh), "f32"))
    wr = bf16(synth.normal_tensor(61, synth.STREAM["w_vocab"], (E, Dh), "f32", 0.05))
    a, b = 0.7, 0.2
    routed = tpc.tpc_moe_route(plan, torch.tensor(h, dtype=torch.float32).to(torch.bfloat16).cuda(),
                               torch.tensor(wr, dtype=torch.float32).to(torch.bfloat16).cuda(), k)
    losses, dz = tpc.tpc_moe_router_loss(plan, routed, k, a, b)
    torch.cuda.synchronize()
    rows = plan.tables()["expanded_rows"]          # compact row of every trajectory position
    z, p, lse, idx, g = moe.route_expanded(h[rows], wr, k)
    load, P, l_aux, l_z, dz_pos = moe.losses_expanded(p, lse, idx, E, k, a, b)
    first = np.unique(rows, return_index=True)[1]  # one position per compact row
    assert np.array_equal(routed["logits"].cpu().numpy(), z[first])
    assert np.array_equal(routed["topk_idx"].cpu().numpy(), idx[first])
    assert np.array_equal(routed["expert_load"].cpu().numpy(), load)
    assert int(load.sum()) == k * NE
    errs = {"gate": err_ratio(routed["topk_gate"].cpu().numpy(), g[first]),
            "lse": err_ratio(routed["lse"].cpu().numpy(), lse[first]),
            "prob_sum": err_ratio(routed["prob_sum"].cpu().numpy(), P),
            "dlogits": err_ratio(dz.cpu().numpy(), moe.expanded_then_unique(dz_pos, rows, N))}
    lo = losses.cpu().numpy()
    errs["L_aux"] = abs(lo[0] - l_aux) / abs(l_aux)
    errs["L_z"] = abs(lo[1] - l_z) / abs(l_z)
    print("compact MoE routing vs expanded", N, "rows", NE, "positions", {k_: f"{v:.1e}" for k_, v in errs.items()})
    assert all(v <= 1e-5 for v in errs.values()), errs


def test_routing_full_wide_tree_sampled(tpc):
    """The wide tree (795,993 unique rows, 18.7 M positions), hidden 2048, 64 experts, top-2: sampled
    rows' logits and experts against the oracle, and expert loads summing to k x positions."""
    import torch
    import synth.gpu as sgpu
    w = synth.workload("wide")
    t = w.tree
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    N, NE, Dh, E, k = plan.info["n_unique"], plan.info["n_expanded"], 2048, 64, 2
    st = t.node_start()
    src_np = plan.compact_source_rows(st, t.length)
    src = torch.tensor(src_np, dtype=torch.int32, device="cuda")
    h = sgpu.normal_rows(41, synth.STREAM["h"], src, Dh, "bf16")
    wr = sgpu.normal_rows(41, synth.STREAM["w_vocab"], None, Dh, "bf16", 0.02, shape=(E,))
    routed = tpc.tpc_moe_route(plan, h, wr, k)
    torch.cuda.synchronize()
    assert int(routed["expert_load"].sum().item()) == k * NE
    pick = np.array([0, 1, 777, N // 3, N - 1])
    hs = synth.rows_normal(41, synth.STREAM["h"], src_np[pick], Dh, "bf16")
    z, _, _, idx, _ = moe.route_expanded(hs, wr.float().cpu().numpy(), k)
    assert np.array_equal(routed["logits"][torch.tensor(pick, device="cuda")].cpu().numpy(), z)
    assert np.array_equal(routed["topk_idx"][torch.tensor(pick, device="cuda")].cpu().numpy(), idx)
