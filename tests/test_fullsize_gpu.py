"""Parity at the full workload sizes that bench.py times, on outputs the oracle can compute one by
one and on properties that hold at any size.

Inputs come from synth's device generator, which writes the same bits as its host generator
(tests/test_synth_gpu.py); sampled rows are regenerated on the host for the oracle, and the vocabulary
matrix (too large to draw on the host in seconds) is read back from the generator's device copy."""
import numpy as np
import pytest

import synth
from kda_case import TOL, err_ratio
from oracle import kda as okda
from oracle import logprob as olp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpc():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def single_fork_case(tpc):
    import torch
    import synth.gpu as sgpu
    w = synth.workload("single_fork")
    t = w.tree
    plan = tpc.Plan(t.parent, t.length, w.chunk).upload()
    st = t.node_start()
    src = torch.tensor(plan.compact_source_rows(st, t.length), dtype=torch.int32, device="cuda")
    x = dict(zip(("q", "k", "v", "g", "beta"), sgpu.kda_inputs(w.seed, src, w.H, w.dk, w.dv, w.dtype)))
    return w, t, plan, st, src, x


def test_single_fork_full_forward(tpc):
    """Full single-fork tree (N = 29,073, H = 16, d = 128, chunk 64, bf16 inputs): outputs of the
    first 256 tokens and of the first 64 tokens after one fork against the token-by-token oracle;
    every trajectory's outputs and final state bitwise equal to the trajectory-expanded run."""
    import torch
    w, t, plan, st, src, x = single_fork_case(tpc)
    o, fin, ws = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], out_dtype=torch.float32)
    torch.cuda.synchronize()
    tpc.tpc_status(plan, ws, w.H, w.dk)
    o_node = np.empty((t.n_rows, w.H, w.dv))
    o_node[plan.compact_source_rows(st, t.length)] = o.cpu().numpy()
    # prefix sample
    rows = np.arange(256)
    inp = synth.kda_inputs(w.seed, rows, w.H, w.dk, w.dv, w.dtype)
    ref, _ = okda.forward(*inp)
    e1 = err_ratio(o_node[rows], ref)
    # 64 tokens after the fork into branch 5: the oracle runs the whole prefix first
    b = 5
    rows = np.concatenate([np.arange(st[0], st[0] + t.length[0]), np.arange(st[b], st[b] + 64)])
    inp = synth.kda_inputs(w.seed, rows, w.H, w.dk, w.dv, w.dtype)
    ref, _ = okda.forward(*inp)
    e2 = err_ratio(o_node[rows[-64:]], ref[-64:])
    print("full single-fork samples", e1, e2)
    assert e1 <= TOL["bf16"] and e2 <= TOL["bf16"], (e1, e2)
    # tree == expanded, bitwise
    tb = plan.tables()
    lens = np.diff(tb["traj_offset"]).astype(np.int32)
    eplan = tpc.Plan(np.full(len(lens), -1, np.int32), lens, 64).upload()
    xe = {k: tpc.tpc_gather_expanded(plan, x[k]) for k in x}
    oe, fine, _ = tpc.tpc_kda_forward(eplan, xe["q"], xe["k"], xe["v"], xe["g"], xe["beta"], out_dtype=torch.float32)
    assert torch.equal(tpc.tpc_gather_expanded(plan, o), oe)
    assert torch.equal(fin, fine)


def test_single_fork_full_backward_equals_sum_over_trajectories(tpc):
    """Full size: the tree backward with the occurrence-summed upstream gradient equals the sum over
    trajectories of the trajectory-expanded backward (gradient accumulation into the shared
    prefix), for every input gradient."""
    import torch
    import synth.gpu as sgpu
    w, t, plan, st, src, x = single_fork_case(tpc)
    n_exp = plan.info["n_expanded"]
    d_o_exp = sgpu.normal_rows(w.seed, synth.STREAM["d_o_exp"], None, w.H * w.dv, "f32",
                               shape=(n_exp,)).view(n_exp, w.H, w.dv)
    d_o = tpc.tpc_reduce_expanded_to_unique(plan, d_o_exp)
    _, _, ws = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], out_dtype=torch.float32)
    gt = tpc.tpc_kda_backward(plan, ws, x["q"], x["k"], x["v"], x["g"], x["beta"], d_o.to(torch.bfloat16), None,
                              out_dtype=torch.float32)
    tb = plan.tables()
    lens = np.diff(tb["traj_offset"]).astype(np.int32)
    eplan = tpc.Plan(np.full(len(lens), -1, np.int32), lens, 64).upload()
    xe = {k: tpc.tpc_gather_expanded(plan, x[k]) for k in x}
    _, _, ews = tpc.tpc_kda_forward(eplan, xe["q"], xe["k"], xe["v"], xe["g"], xe["beta"], out_dtype=torch.float32)
    # the expanded run gets the same bf16-rounded gradient rows as the tree; bf16 d_o per row of the
    # tree is the rounded occurrence sum, so the expanded run carries it on the first occurrence only
    first = np.zeros(n_exp, bool)
    rows = tb["expanded_rows"]
    _, idx = np.unique(rows, return_index=True)
    first[idx] = True
    d_o_first = tpc.tpc_gather_expanded(plan, d_o.to(torch.bfloat16))
    d_o_first[torch.tensor(~first, device="cuda")] = 0
    ge = tpc.tpc_kda_backward(eplan, ews, xe["q"], xe["k"], xe["v"], xe["g"], xe["beta"], d_o_first, None,
                              out_dtype=torch.float32)
    torch.cuda.synchronize()
    errs = {}
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        red = tpc.tpc_reduce_expanded_to_unique(plan, ge[key].float())
        errs[key] = err_ratio(gt[key].float().cpu().numpy(), red.cpu().numpy())
    print("full single-fork backward, tree vs summed trajectories", errs)
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


def test_wide_tree_logprob_full_size_sampled_rows(tpc):
    """Full wide tree (795,993 unique rows, 18.7 M positions, V = 65,536, Dh = 2048) in bench.py's
    launch configuration (16,384-row logit chunks): lse, the log-probabilities of every occurrence
    and dh of sampled rows against the fp64 oracle restricted to those rows."""
    import torch
    import synth.gpu as sgpu
    w = synth.workload("wide")
    t = w.tree
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    st = t.node_start()
    info = plan.info
    N, NE, V, Dh, CR = info["n_unique"], info["n_expanded"], 65536, 2048, 16384
    seed = 41
    src_np = plan.compact_source_rows(st, t.length)
    src = torch.tensor(src_np, dtype=torch.int32, device="cuda")
    h = sgpu.normal_rows(seed, synth.STREAM["h"], src, Dh, "bf16")
    W = sgpu.normal_rows(seed, synth.STREAM["w_vocab"], None, Dh, "bf16", 0.02, shape=(V,))
    targets_np = synth.uniform_int(seed, synth.STREAM["targets"], np.arange(NE), V).astype(np.int32)
    dlogp_np = synth.normal_tensor(seed, synth.STREAM["d_logp"], (NE,), "f32")
    targets = torch.tensor(targets_np, device="cuda")
    dlogp = torch.tensor(dlogp_np, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scratch = tpc.logprob_scratch(V, CR)
    logp, lse = tpc.tpc_logprob_forward(plan, h, W, targets, chunk_rows=CR, scratch=scratch, status=status)
    dh, dW = tpc.tpc_logprob_backward(plan, h, W, targets, dlogp, lse, chunk_rows=CR, scratch=scratch, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    # sampled compact rows: the first, the last, a prefix row and rows deep in the tree
    exp_rows = plan.tables()["expanded_rows"]
    pick = np.array([0, 1, 20000, N // 2, N - 2, N - 1])
    node_rows = src_np[pick]
    h_s = synth.rows_normal(seed, synth.STREAM["h"], node_rows, Dh, "bf16")
    W_h = W.float().cpu().numpy().astype(np.float64)
    occ = [np.nonzero(exp_rows == r)[0] for r in pick]
    occ_row = np.concatenate([np.full(len(o_), i) for i, o_ in enumerate(occ)])
    occ_idx = np.concatenate(occ)
    logp_ref, lse_ref = olp.forward(h_s, W_h, occ_row, targets_np[occ_idx])
    dh_ref, _ = olp.backward(h_s, W_h, occ_row, targets_np[occ_idx], dlogp_np[occ_idx])
    errs = {"lse": err_ratio(lse.cpu().numpy()[pick], lse_ref),
            "logp": err_ratio(logp.cpu().numpy()[occ_idx], logp_ref),
            "dh": err_ratio(dh.cpu().numpy()[pick], dh_ref)}
    print("full wide-tree log-prob samples", errs, "occurrences", len(occ_idx))
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
