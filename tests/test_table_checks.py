"""Index and bounds mode: every index field of the plan's device tables is bounded before a call
that reads them launches anything (HARTS Figure 2(c): rounds, boundary-state slots, replayed rows).

CPU: the host evaluation of the same bounds (tpc_plan_check_host) passes every valid plan in every
planner mode, with and without sharing-window exports, and rejects a planted bad entry in each
table that the kernels index through.  GPU: the device check rejects a corrupted uploaded entry with
TPC_ERR_DEVICE_CHECK before any compute kernel is launched, and with the mode on results are
bitwise those of the mode off."""
import numpy as np
import pytest

import synth

ERR_BAD_SHAPE, ERR_DEVICE_CHECK = 2, 7
MODES = (0, 1, 2)  # minimum rounds, node-wise, no replay


@pytest.fixture(scope="module")
def tpc():
    from tree_packed_chunkwise_b200 import build
    build.build()
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def random_forest(rng):
    n = int(rng.integers(1, 30))
    parent = np.array([-1] + [(-1 if rng.random() < 0.05 else int(rng.integers(0, i))) for i in range(1, n)], np.int32)
    length = rng.integers(1, 150, size=n).astype(np.int32)
    return parent, length


def test_valid_plans_pass_host_checks(tpc):
    for cfg in ("fig1", "agentic_small", "agentic", "single_fork"):
        w = synth.workload(cfg)
        for mode in MODES:
            tpc.Plan(w.tree.parent, w.tree.length, w.chunk, mode).check_host()
    rng = np.random.default_rng(11)
    for _ in range(300):
        parent, length = random_forest(rng)
        for mode in MODES:
            tpc.Plan(parent, length, 64, mode).check_host()
    # sharing-window exports: consumers past the sequences of the plan
    w = synth.workload("agentic_small")
    t = w.tree
    s0 = np.zeros(t.n, np.int64)  # trajectory position of each node's first token
    for v in range(t.n):
        s0[v] = 0 if t.parent[v] < 0 else s0[t.parent[v]] + t.length[t.parent[v]]
    ex = []  # aligned positions inside non-root nodes (s < pos <= s + length)
    for v in range(t.n):
        pos = (s0[v] // 64 + 1) * 64
        if t.parent[v] >= 0 and pos <= s0[v] + t.length[v] and len(ex) < 4:
            ex.append((v, int(pos)))
    assert ex
    tpc.Plan(t.parent, t.length, 64, exports=ex).check_host()


def planted(pl, info):
    """(table, word, bad value, table name) entries that break one bound each."""
    N, R = info["n_unique"], info["replay_total"]
    ns, nsl = info["n_seqs"], info["n_slots"]
    d = pl.debug_tables()
    rep_chunk = int(np.nonzero(d["chunks"][:, 2] > 0)[0][0])
    out = [
        (0, 8 * 1 + 0, info["n_chunks"], "seqs"),              # chunk_begin past the chunks
        (0, 8 * 0 + 2, nsl, "seqs"),                          # import from a slot that does not exist
        (0, 8 * 0 + 2, -info["n_roots"] - 1, "seqs"),         # initial state of a root that does not exist
        (1, 8 * 3 + 3, N, "chunks"),                           # own rows run past N
        (1, 8 * 2 + 1, 0, "chunks"),                           # empty chunk
        (1, 8 * rep_chunk + 4, R, "chunks"),                   # replay rows past R
        (1, 8 * 0 + 0, ns, "chunks"),                          # chunk of a sequence that does not exist
        (3, 0, ns + info["n_exports"], "slot_cons"),          # consumer past the sequences
        (6, R - 1, N, "replay_rows"),                          # replayed row past N
        (6, 0, -1, "replay_rows"),
        (11, 5, N, "exp_rows"),                                # expanded position maps past N
        (12, 3, int(info["n_expanded"]) + 1, "occ_begin"),     # occurrence offsets past the list
        (13, 0, -1, "occ_list"),
        (16, 1, N + 1, "attn_ranges"),                         # ancestor range past N
        (17, 2, 129, "attn_qtiles"),                           # query tile wider than 128 rows
        (18, 0, pl.n_nodes, "attn_ktiles"),                    # key tile of a node that does not exist
    ]
    if nsl:
        out.append((2, 2, len(d["slot_cons"]) + 1, "slots"))  # consumer list past its table
    return out


def test_planted_bad_entries_fail_host_checks(tpc):
    w = synth.workload("agentic_small")  # replays, slots and several rounds
    pl = tpc.Plan(w.tree.parent, w.tree.length, w.chunk)
    info = pl.info
    assert info["replay_total"] > 0 and info["n_slots"] > 0
    for table, word, value, name in planted(pl, info):
        with pytest.raises(tpc.TpcError) as e:
            pl.check_host(table, word, value)
        assert e.value.code == ERR_DEVICE_CHECK, (table, word, value)
        assert name + "[" in str(e.value), (name, str(e.value))
    # an offset table out of order: occ_begin[2] = 0 < occ_begin[1] (every row occurs at least once)
    with pytest.raises(tpc.TpcError) as e:
        pl.check_host(12, 2, 0)
    assert e.value.code == ERR_DEVICE_CHECK and "occ_begin[1]: non-decreasing" in str(e.value), str(e.value)
    # words outside a table, and tables that do not exist, are refused on the host
    for table, word in ((1, 8 * info["n_chunks"]), (6, info["replay_total"]), (19, 0)):
        with pytest.raises(tpc.TpcError) as e:
            pl.check_host(table, word, 0)
        assert e.value.code == ERR_BAD_SHAPE


def test_checks_mode_switch(tpc):
    was = tpc.tpc_checks_enabled()
    try:
        tpc.tpc_checks_enable(True)
        assert tpc.tpc_checks_enabled()
        tpc.tpc_checks_enable(False)
        assert not tpc.tpc_checks_enabled()
    finally:
        tpc.tpc_checks_enable(was)


@pytest.mark.gpu
def test_device_check_rejects_corrupt_entry_before_launch(tpc):
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from kda_case import Case, to_torch_compact
    w = synth.workload("agentic_small")
    t = w.tree
    case = Case(t, 2, 128, 64, "bf16", 23)
    pl = tpc.Plan(t.parent, t.length, 64).upload()
    x = to_torch_compact(case, pl)
    pl.check_device()  # a valid upload passes, whatever the mode
    was = tpc.tpc_checks_enabled()
    try:
        tpc.tpc_checks_enable(False)
        o0, f0, _ = tpc.tpc_kda_forward(pl, x["q"], x["k"], x["v"], x["g"], x["beta"], x["init"])
        torch.cuda.synchronize()
        tpc.tpc_checks_enable(True)
        n0 = tpc.tpc_launch_count()
        o1, f1, _ = tpc.tpc_kda_forward(pl, x["q"], x["k"], x["v"], x["g"], x["beta"], x["init"])
        torch.cuda.synchronize()
        assert tpc.tpc_launch_count() > n0 + 1  # the check and the forward's kernels
        assert torch.equal(o0, o1) and torch.equal(f0, f1)
        N = pl.info["n_unique"]
        for table, word, value, name in ((1, 8 * 3 + 3, N + 1000, "chunks"), (6, 0, N, "replay_rows"),
                                         (0, 2, pl.info["n_slots"] + 7, "seqs")):
            old = pl.poke_table(table, word, value)
            n0 = tpc.tpc_launch_count()
            with pytest.raises(tpc.TpcError) as e:
                tpc.tpc_kda_forward(pl, x["q"], x["k"], x["v"], x["g"], x["beta"], x["init"])
            assert e.value.code == ERR_DEVICE_CHECK and name + "[" in str(e.value), str(e.value)
            assert tpc.tpc_launch_count() == n0 + 1  # the check kernel alone
            with pytest.raises(tpc.TpcError) as e:
                pl.check_device()
            assert e.value.code == ERR_DEVICE_CHECK
            assert pl.poke_table(table, word, old) == value
            pl.check_device()
        o2, _, _ = tpc.tpc_kda_forward(pl, x["q"], x["k"], x["v"], x["g"], x["beta"], x["init"])
        torch.cuda.synchronize()
        assert torch.equal(o0, o2)
    finally:
        tpc.tpc_checks_enable(was)
