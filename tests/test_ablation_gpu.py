"""The planner ablations on the GPU (HARTS Figure 4: node-wise linear attention; Figure 5: replay
against no replay): every mode computes the same recurrence within the bf16 bound, the node-wise and
minimum-call plans keep each trajectory's chunkwise numerical path bit for bit (chunk grids aligned
to trajectory positions, bounded replay), and the no-replay plan, whose side sequences start their
grid at the fork point, does not."""
import numpy as np
import pytest

import synth
from kda_case import Case, TOL, err_ratio, node_order, to_torch_compact
from oracle import kda as okda
from oracle import planner as P

pytestmark = pytest.mark.gpu

MODES = {"min_rounds": 0, "nodewise": 1, "noreplay": 2}


@pytest.fixture(scope="module")
def tpc():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def forward_backward(tpc, plan, x, out_dtype):
    o, fin, ws = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], out_dtype=out_dtype)
    gr = tpc.tpc_kda_backward(plan, ws, x["q"], x["k"], x["v"], x["g"], x["beta"], x["d_o"], x["d_final"],
                              out_dtype=out_dtype, want_d_init=False)
    return o, fin, gr, ws


def test_ablation_modes_parity_and_numerical_path(tpc):
    import torch
    w = synth.workload("agentic_small")
    t = w.tree
    case = Case(t, 2, 128, 64, "bf16", 31)
    o_ref, fin_ref = case.oracle_forward
    g_ref = case.oracle_backward
    tb0 = tpc.Plan(t.parent, t.length, 64).tables()
    lens = np.diff(tb0["traj_offset"]).astype(np.int32)
    eplan = tpc.Plan(np.full(len(lens), -1, np.int32), lens, 64).upload()
    outs = {}
    for mode, code in MODES.items():
        plan = tpc.Plan(t.parent, t.length, 64, code).upload()
        x = to_torch_compact(case, plan)
        o, fin, gr, ws = forward_backward(tpc, plan, x, torch.float32)
        torch.cuda.synchronize()
        tpc.tpc_status(plan, ws, case.H, case.d)
        errs = {"o": err_ratio(node_order(plan, case, o.cpu().numpy()), o_ref),
                "final": err_ratio(fin.cpu().numpy(), fin_ref)}
        for name, ref in zip(("dq", "dk", "dv", "dg", "dbeta"), g_ref[:5]):
            errs[name] = err_ratio(node_order(plan, case, gr[name].float().cpu().numpy()), ref)
        print(mode, "rounds", plan.info["n_rounds"], "replay rows", plan.info["replay_total"],
              "chunks", plan.info["n_chunks"], {k: f"{v:.2e}" for k, v in errs.items()})
        assert all(e <= TOL["bf16"] for e in errs.values()), (mode, errs)
        outs[mode] = (tpc.tpc_gather_expanded(plan, o), fin)
    # the trajectory-expanded run: one root per trajectory, chunk grid from position 0
    xe_plan = tpc.Plan(t.parent, t.length, 64).upload()
    x = to_torch_compact(case, xe_plan)
    xe = {k: tpc.tpc_gather_expanded(xe_plan, x[k]) for k in ("q", "k", "v", "g", "beta")}
    oe, fine, _ = tpc.tpc_kda_forward(eplan, xe["q"], xe["k"], xe["v"], xe["g"], xe["beta"], out_dtype=torch.float32)
    for mode in ("min_rounds", "nodewise"):
        assert torch.equal(outs[mode][0], oe), mode
        assert torch.equal(outs[mode][1], fine), mode
    assert not torch.equal(outs["noreplay"][0], oe)
    assert P.plan(t.parent, t.length, 64, "nodewise").n_rounds >= P.plan(t.parent, t.length, 64).n_rounds


def test_noreplay_error_by_handoff_depth(tpc):
    """Full agentic tree (H = 16, 64 leaves, 5 fork levels): forward outputs of the minimum-call
    plan (bounded replay) and of the no-replay plan against the oracle on the trajectories of two
    deepest leaves, max error over RMS binned by the handoff depth of each row (segment boundaries,
    i.e. boundary-state handoffs, on its path: 0 to 5).  Both stay inside the bf16 bound; the table
    is printed."""
    import torch
    import synth.gpu as sgpu
    w = synth.workload("agentic")
    t = w.tree
    heads = [0, 5]
    res = {}
    for mode in ("min_rounds", "noreplay"):
        plan = tpc.Plan(t.parent, t.length, 64, MODES[mode]).upload()
        st = t.node_start()
        src_np = plan.compact_source_rows(st, t.length)
        src = torch.tensor(src_np, dtype=torch.int32, device="cuda")
        x = dict(zip(("q", "k", "v", "g", "beta"), sgpu.kda_inputs(w.seed, src, w.H, w.dk, w.dv, "bf16")))
        o, _, ws = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], out_dtype=torch.float32,
                                       want_final=False)
        torch.cuda.synchronize()
        tpc.tpc_status(plan, ws, w.H, w.dk)
        inv = np.empty(len(src_np), np.int64)
        inv[src_np] = np.arange(len(src_np))
        res[mode] = (o, inv)
    depth = P.handoff_depth(t.parent)
    leaves = list(t.leaves())
    deepest = sorted(leaves, key=lambda l: (-depth[l], len(t.trajectory_rows(l))))[:2]
    st = t.node_start()
    errs = {m: {} for m in res}
    for leaf in deepest:
        rows = t.trajectory_rows(leaf)
        inp = synth.kda_inputs(w.seed, rows, w.H, w.dk, w.dv, "bf16", heads=heads)
        o_ref, _ = okda.forward(*inp)
        rms = np.sqrt(np.mean(o_ref ** 2))
        node_of_row = np.concatenate([np.full(t.length[v], v) for v in t.path(leaf)])
        for m, (o, inv) in res.items():
            got = o[torch.tensor(inv[rows], device="cuda")][:, heads].cpu().numpy()
            e = np.abs(got - o_ref).max(axis=(1, 2)) / rms
            for dd in np.unique(depth[node_of_row]):
                sel = depth[node_of_row] == dd
                errs[m][int(dd)] = max(errs[m].get(int(dd), 0.0), float(e[sel].max()))
    print("handoff depth | max err / RMS, bounded replay | no replay | excess")
    for dd in sorted(errs["noreplay"]):
        a, b = errs["min_rounds"][dd], errs["noreplay"][dd]
        print(f"{dd} | {a:.3e} | {b:.3e} | {100 * (b / a - 1):+.1f}%")
    assert max(errs["noreplay"]) == 5
    assert all(v <= TOL["bf16"] for m in errs for v in errs[m].values()), errs
