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


# ------------------------------------------------------------------------------------ windowed parity
def windowed_parity(tpc, tree, H, d, seed, heads, specs, label):
    """Full-size tree-packed forward + backward against the token-by-token oracle on windows.

    specs: list of dicts {leaf, windows: [(first, last + 1) node-order rows], d_final: bool}.  The
    upstream output gradient is non-zero (N(0, 1), bf16) only on the windows' rows and the final-state
    gradient only on the flagged leaves, so every input gradient equals the sum, over the specs'
    trajectories, of the oracle's backward of that trajectory (HARTS abstract: gradients of dependent
    work accumulate into the shared prefix), and rows on no such trajectory get exactly zero.  Heads
    are independent: the oracle runs on ``heads`` only.  Outputs and the flagged leaves' final states
    are compared over the whole trajectories."""
    import torch
    import synth.gpu as sgpu
    plan = tpc.Plan(tree.parent, tree.length, 64).upload()
    info = plan.info
    N = info["n_unique"]
    st = tree.node_start()
    src_np = plan.compact_source_rows(st, tree.length)
    inv = np.empty(N, np.int64)
    inv[src_np] = np.arange(N)
    src = torch.tensor(src_np, dtype=torch.int32, device="cuda")
    x = dict(zip(("q", "k", "v", "g", "beta"), sgpu.kda_inputs(seed, src, H, d, d, "bf16")))
    leaves = list(tree.leaves())
    d_o = torch.zeros(N, H, d, dtype=torch.bfloat16, device="cuda")
    d_fin = torch.zeros(len(leaves), H, d, d, dtype=torch.float32, device="cuda")
    win_rows = {}
    for sp in specs:
        rows = np.concatenate([np.arange(a, b) for a, b in sp["windows"]]) if sp["windows"] else np.zeros(0, np.int64)
        win_rows[sp["leaf"]] = rows
        if len(rows):
            vals = synth.rows_normal(seed, synth.STREAM["d_o"], rows, H * d, "bf16").reshape(len(rows), H, d)
            d_o[torch.tensor(inv[rows], device="cuda")] = torch.tensor(vals, dtype=torch.float32).to(
                torch.bfloat16).cuda()
        if sp["d_final"]:
            li = leaves.index(sp["leaf"])
            d_fin[li] = torch.tensor(synth.normal_tensor(seed, synth.STREAM["d_final"], (H, d, d), "f32",
                                                         first=li * H * d * d), dtype=torch.float32)
    o, fin, ws = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], out_dtype=torch.float32)
    gr = tpc.tpc_kda_backward(plan, ws, x["q"], x["k"], x["v"], x["g"], x["beta"], d_o, d_fin,
                              out_dtype=torch.float32, want_d_init=False)
    torch.cuda.synchronize()
    tpc.tpc_status(plan, ws, H, d)
    # the oracle, trajectory by trajectory, gradients summed per node-order row
    union = np.unique(np.concatenate([tree.trajectory_rows(sp["leaf"]) for sp in specs]))
    pos = {r: i for i, r in enumerate(union)}
    nh = len(heads)
    acc = {k: np.zeros((len(union), nh, d)) for k in ("dq", "dk", "dv", "dg")}
    acc["dbeta"] = np.zeros((len(union), nh))
    o_ref = np.zeros((len(union), nh, d))
    fin_ref = {}
    for sp in specs:
        rows = tree.trajectory_rows(sp["leaf"])
        inp = synth.kda_inputs(seed, rows, H, d, d, "bf16", heads=heads)
        dO = np.zeros((len(rows), nh, d))
        wr = win_rows[sp["leaf"]]
        if len(wr):
            vals = synth.rows_normal(seed, synth.STREAM["d_o"], wr, H * d, "bf16").reshape(len(wr), H, d)[:, heads]
            where = {r: i for i, r in enumerate(rows)}
            dO[[where[r] for r in wr]] = vals
        li = leaves.index(sp["leaf"])
        dF = None
        if sp["d_final"]:
            dF = synth.normal_tensor(seed, synth.STREAM["d_final"], (H, d, d), "f32", first=li * H * d * d)[heads]
        o_t, S_t = okda.forward(*inp)
        g_t = okda.backward(*inp, dO, dF)
        ix = np.array([pos[r] for r in rows])
        o_ref[ix] = o_t
        fin_ref[li] = S_t
        for key, val in zip(("dq", "dk", "dv", "dg", "dbeta"), g_t[:5]):
            np.add.at(acc[key], ix, val)
    cix = torch.tensor(inv[union], device="cuda")
    hix = torch.tensor(heads, device="cuda")
    pick = lambda t: t[cix][:, hix].float().cpu().numpy()
    errs = {"o": err_ratio(pick(o), o_ref)}
    for li, S in fin_ref.items():
        errs[f"final[{li}]"] = err_ratio(fin[li][hix].cpu().numpy(), S)
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        errs[key] = err_ratio(pick(gr[key]), acc[key])
    # rows on no checked trajectory: exactly zero gradient (all heads)
    off = torch.ones(N, dtype=torch.bool, device="cuda")
    off[cix] = False
    zero_off = {key: float(gr[key][off].abs().max().item()) if off.any() else 0.0
                for key in ("dq", "dk", "dv", "dg", "dbeta")}
    print(label, {k: f"{v:.2e}" for k, v in errs.items()}, "off-trajectory max |grad|", zero_off,
          "trajectory rows", len(union), "of", N)
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
    assert all(z == 0.0 for z in zero_off.values()), zero_off
    return plan


def test_single_fork_windowed_backward_vs_oracle(tpc):
    """Full single-fork tree (N = 29,073, H = 16): the upstream gradient on the last 64 rows of the
    longest branch (the reverse scan crosses the fork and the 128 prefix chunks) and the final-state
    gradient of a second leaf; outputs, both final states and all gradients of heads 0 and 9
    against the oracle."""
    w = synth.workload("single_fork")
    t = w.tree
    leaves = list(t.leaves())
    lens = [len(t.trajectory_rows(l)) for l in leaves]
    longest = leaves[int(np.argmax(lens))]
    other = leaves[0] if leaves[0] != longest else leaves[1]
    st = t.node_start()
    end = st[longest] + t.length[longest]
    specs = [dict(leaf=longest, windows=[(end - 64, end)], d_final=False),
             dict(leaf=other, windows=[], d_final=True)]
    windowed_parity(tpc, t, w.H, w.dk, w.seed, [0, 9], specs, "single-fork windowed")


def test_agentic_full_windowed_with_replay_vs_oracle(tpc):
    """Full agentic tree (64 leaves, 5 fork levels, H = 16, with replay rows): a trajectory whose path
    holds replay-started sequences, upstream gradient on the last 64 rows of its leaf and on 64 rows
    inside a replay-started node, plus its final-state gradient; outputs, final state and every
    gradient of heads 3 and 12 against the oracle."""
    w = synth.workload("agentic")
    t = w.tree
    plan = tpc.Plan(t.parent, t.length, 64)
    tb = plan.tables()
    assert plan.info["replay_total"] > 0
    best, best_n = None, -1
    for leaf in t.leaves():
        path = t.path(leaf)
        n_rep = sum(1 for v in path if tb["replay_len"][v] > 0)
        if n_rep > best_n or (n_rep == best_n and tb["round"][leaf] > tb["round"][best]):
            best, best_n = leaf, n_rep
    assert best_n >= 2
    st = t.node_start()
    path = t.path(best)
    rep = [v for v in path if tb["replay_len"][v] > 0][0]
    end = st[best] + t.length[best]
    windows = [(st[rep], st[rep] + min(64, int(t.length[rep])))] if rep != best else []
    windows.append((max(end - 64, st[best]), end))
    specs = [dict(leaf=best, windows=windows, d_final=True)]
    print("agentic leaf", best, "replay-started nodes on the path", best_n, "rounds", plan.info["n_rounds"])
    windowed_parity(tpc, t, w.H, w.dk, w.seed, [3, 12], specs, "agentic windowed")


def test_wide_tree_windowed_vs_oracle(tpc):
    """Full wide tree (32,768-token prefix = 512 sequential chunks, 512 leaves) as bench.py runs its
    KDA layer (one group of 8 of the 32 heads per call): upstream gradient on the last 64 rows of the
    prefix and of a depth-3 leaf, final-state gradient of that leaf; outputs, final state and all
    gradients of heads 1 and 6 against the oracle."""
    w = synth.workload("wide")
    t = w.tree
    leaves = list(t.leaves())
    lens = [len(t.trajectory_rows(l)) for l in leaves]
    leaf = leaves[int(np.argmax(lens))]
    st = t.node_start()
    pend = int(t.length[0])
    end = st[leaf] + t.length[leaf]
    windows = [(pend - 64, pend), (max(end - 64, st[leaf]), end)]
    specs = [dict(leaf=leaf, windows=windows, d_final=True)]
    windowed_parity(tpc, t, 8, w.dk, w.seed + 17, [1, 6], specs, "wide windowed (8-head group)")


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
    scratch = tpc.logprob_scratch(plan, V, CR)
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
