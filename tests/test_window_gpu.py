"""Sharing windows across microbatches on the GPU (HARTS abstract: gradients of dependent
microbatches accumulate before one backward pass through the shared prefix; Figure 3): a producer
call's exported boundary states start several consumer calls; the consumers' backward passes run
first and their state gradients enter the producer's single backward.  Forward results equal the
whole-tree call bit for bit (same chunk grid, bounded replay); gradients match the whole-tree call
and the oracle within the bf16 bound."""
import numpy as np
import pytest

import synth
from kda_case import Case, TOL, err_ratio

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpc():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def test_sharing_window_equals_whole_tree(tpc):
    import torch
    from tree_packed_chunkwise_b200.window import Window
    w = synth.workload("agentic_small")
    t = w.tree
    H, d, seed = 2, 128, 41
    depth = np.zeros(t.n, int)
    for v in range(t.n):
        depth[v] = 0 if t.parent[v] < 0 else depth[t.parent[v]] + 1
    cut = [v for v in range(t.n) if depth[v] == 2]
    win = Window(t.parent, t.length, 64, cut)
    assert len(win.consumers) >= 3 and len(win.exports) < len(win.consumers)  # exports shared
    leaves = list(t.leaves())
    case = Case(t, H, d, 64, "bf16", seed)
    q, k, v, g, b = case.inputs
    d_o = case.d_o

    def tensors(mb, replay_rows=0):
        rows = mb.orig_rows
        x = {name: torch.tensor(arr[rows], dtype=torch.float32).to(torch.bfloat16).cuda()
             for name, arr in zip(("q", "k", "v", "g", "beta"), (q, k, v, g, b))}
        do = d_o[rows].copy()
        if replay_rows:
            do[np.isin(rows, mb.node_rows[0])] = 0.0  # replayed rows carry no output gradient
        x["d_o"] = torch.tensor(do, dtype=torch.float32).to(torch.bfloat16).cuda()
        # final-state gradients of the microbatch's leaves that are leaves of the whole tree
        sub_leaves = np.nonzero(~np.isin(np.arange(len(mb.parent)), mb.parent[mb.parent >= 0]))[0]
        dfin = np.zeros((len(sub_leaves), H, d, d))
        for i, sl in enumerate(sub_leaves):
            orig_first = mb.node_rows[sl][0]
            match = [li for li, l in enumerate(leaves) if t.node_start()[l] == orig_first]
            if match:
                dfin[i] = case.d_final[match[0]]
        x["d_final"] = torch.tensor(dfin, dtype=torch.float32).cuda()
        return x

    px = tensors(win.producer)
    cx = [tensors(mb, r) for mb, r in zip(win.consumers, win.replay_n)]
    fwd = win.forward(px, cx, out_dtype=torch.float32)
    pg, cg = win.backward(px, cx, fwd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    # assemble per original node-order row: producer rows, then each consumer's own (non-replayed) rows
    N = t.n_rows
    out = {key: np.full((N, H) + ((d,) if key != "dbeta" else ()), np.nan) for key in ("o", "dq", "dk", "dv", "dg", "dbeta")}
    po, co, _ = fwd
    sources = [(win.producer, po[0], pg, None)] + [(mb, co[i][0], cg[i], mb.node_rows[0] if win.replay_n[i] else None)
                                                    for i, mb in enumerate(win.consumers)]
    for mb, o, gr, rep in sources:
        own = np.ones(len(mb.orig_rows), bool) if rep is None else ~np.isin(mb.orig_rows, rep)
        rows = mb.orig_rows[own]
        out["o"][rows] = o.float().cpu().numpy()[own]
        for key in ("dq", "dk", "dv", "dg", "dbeta"):
            out[key][rows] = gr[key].float().cpu().numpy()[own]
    assert not np.isnan(out["o"]).any() and not np.isnan(out["dk"]).any()
    # the whole tree in one call
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    full = {}
    st = t.node_start()
    comp = lambda a: plan.to_compact(a, st, t.length)
    xf = {name: torch.tensor(comp(arr), dtype=torch.float32).to(torch.bfloat16).cuda()
          for name, arr in zip(("q", "k", "v", "g", "beta", "d_o"), (q, k, v, g, b, d_o))}
    o_f, fin_f, ws = tpc.tpc_kda_forward(plan, xf["q"], xf["k"], xf["v"], xf["g"], xf["beta"], out_dtype=torch.float32)
    g_f = tpc.tpc_kda_backward(plan, ws, xf["q"], xf["k"], xf["v"], xf["g"], xf["beta"], xf["d_o"],
                               torch.tensor(case.d_final, dtype=torch.float32).cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    src = plan.compact_source_rows(st, t.length)
    full["o"] = np.empty_like(out["o"])
    full["o"][src] = o_f.cpu().numpy()
    assert np.array_equal(full["o"], out["o"]), "window forward must equal the whole-tree call bit for bit"
    errs = {}
    g_ref = case.oracle_backward
    for key, ref in zip(("dq", "dk", "dv", "dg", "dbeta"), g_ref[:5]):
        fk = np.empty_like(out[key])
        fk[src] = g_f[key].float().cpu().numpy()
        errs[key] = (err_ratio(out[key], fk), err_ratio(out[key], ref))
    print("window vs whole tree / vs oracle", {k: f"{a:.1e} / {b_:.1e}" for k, (a, b_) in errs.items()})
    assert all(a <= TOL["bf16"] and b_ <= TOL["bf16"] for a, b_ in errs.values()), errs
