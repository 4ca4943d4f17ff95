"""GPU log-probability recovery (one logit row per unique row) against the fp64 oracle."""
import numpy as np
import pytest

import synth
from kda_case import TOL, err_ratio
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


def make(tree, Dh, V, seed):
    N, n_exp = tree.n_rows, tree.n_expanded()
    h = synth.normal_tensor(seed, synth.STREAM["h"], (N, Dh), "bf16")
    W = synth.normal_tensor(seed, synth.STREAM["w_vocab"], (V, Dh), "bf16", 0.1)
    targets = synth.uniform_int(seed, synth.STREAM["targets"], np.arange(n_exp), V)
    dlogp = synth.normal_tensor(seed, synth.STREAM["d_logp"], (n_exp,), "f32")
    occ_row = np.concatenate([tree.trajectory_rows(l) for l in tree.leaves()])
    return h, W, targets, dlogp, occ_row


@pytest.mark.parametrize("cfg,chunk", [("agentic_small", 512), ("fig1", 64)])
def test_logprob_matches_oracle(tpc, cfg, chunk):
    import torch
    tree = synth.workload(cfg).tree
    Dh, V = 64, 1000
    h, W, targets, dlogp, occ_row = make(tree, Dh, V, 7)
    logp_ref, lse_ref = olp.forward(h, W, occ_row, targets)
    dh_ref, dW_ref = olp.backward(h, W, occ_row, targets, dlogp)
    plan = tpc.Plan(tree.parent, tree.length, 16 if cfg == "fig1" else 64).upload()
    st = tree.node_start()
    hd = torch.tensor(plan.to_compact(h, st, tree.length), dtype=torch.float32).to(torch.bfloat16).cuda()
    Wd = torch.tensor(W, dtype=torch.float32).to(torch.bfloat16).cuda()
    td = torch.tensor(targets, dtype=torch.int32, device="cuda")
    dl = torch.tensor(dlogp, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    logp, lse = tpc.tpc_logprob_forward(plan, hd, Wd, td, chunk_rows=chunk, status=status)
    dh, dW = tpc.tpc_logprob_backward(plan, hd, Wd, td, dl, lse, chunk_rows=chunk, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    comp = lambda a: plan.to_compact(a, st, tree.length)
    errs = {"logp": err_ratio(logp.cpu().numpy(), logp_ref), "lse": err_ratio(lse.cpu().numpy(), comp(lse_ref)),
            "dh": err_ratio(dh.cpu().numpy(), comp(dh_ref)), "dW": err_ratio(dW.cpu().numpy(), dW_ref)}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
    # one logit row serves every occurrence: equal (row, target) pairs give identical values
    rows = plan.tables()["expanded_rows"]
    key = rows.astype(np.int64) * V + targets
    lp = logp.cpu().numpy()
    first = {}
    for j, k in enumerate(key):
        if k in first:
            assert lp[j] == lp[first[k]]
        else:
            first[k] = j
    print(cfg, errs)


def test_logprob_rejects_out_of_range_targets(tpc):
    import torch
    tree = synth.workload("fig1").tree
    plan = tpc.Plan(tree.parent, tree.length, 16).upload()
    hd = torch.zeros(tree.n_rows, 64, dtype=torch.bfloat16, device="cuda")
    Wd = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    td = torch.full((tree.n_expanded(),), 64, dtype=torch.int32, device="cuda")  # == V: out of range
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tpc.tpc_logprob_forward(plan, hd, Wd, td, chunk_rows=64, status=status)
    torch.cuda.synchronize()
    assert status.item() == 7
