"""Host-side checks of the C ABI library (no GPU needed): every declared symbol is
exported, and the C++ planner's tables equal the oracle planner's bit for bit."""
import os
import re

import numpy as np
import pytest

import synth
from oracle import planner as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tpc():
    from tree_packed_chunkwise_b200 import build
    build.build()
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(tpc_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(tpc):
    names = declared_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(tpc.lib(), n), n
    assert names <= set(tpc.SIGNATURES), names - set(tpc.SIGNATURES)


MODE_CODE = {"min_rounds": 0, "nodewise": 1, "noreplay": 2}


def compare(tpc, parent, length, C, mode="min_rounds"):
    ref = P.plan(parent, length, C, mode)
    pl = tpc.Plan(parent, length, C, MODE_CODE[mode])
    tb = pl.tables()
    assert pl.info["n_rounds"] == ref.n_rounds
    assert np.array_equal(tb["round"], ref.round)
    assert np.array_equal(tb["is_cont"], ref.cont)
    assert np.array_equal(tb["anchor"], ref.anchor)
    assert np.array_equal(tb["replay_start"], ref.replay_start)
    assert np.array_equal(tb["replay_len"], ref.replay_len)
    assert np.array_equal(tb["row_offset"], ref.row_offset)
    assert np.array_equal(tb["occurrence"], ref.occurrence)
    assert np.array_equal(tb["leaves"], ref.leaves)
    rows, offs = P.expanded_rows(ref)
    assert np.array_equal(tb["expanded_rows"], rows)
    assert np.array_equal(tb["traj_offset"], offs)
    assert pl.info["replay_total"] == ref.replay_total
    assert pl.info["n_slots"] == len(ref.slots)
    assert pl.info["n_seqs"] == len(ref.seqs)
    assert pl.info["n_chunks"] == P.chunk_count(ref)
    return pl


@pytest.mark.parametrize("cfg", ["fig1", "single_fork", "agentic", "agentic_small", "wide"])
def test_planner_bit_exact_on_workloads(tpc, cfg):
    w = synth.workload(cfg)
    compare(tpc, w.tree.parent, w.tree.length, w.chunk)


@pytest.mark.parametrize("C", [16, 32, 64])
def test_planner_bit_exact_random(tpc, C):
    rng = np.random.default_rng(C)
    for _ in range(400):
        n = int(rng.integers(1, 40))
        parent = [-1] + [(-1 if rng.random() < 0.05 else int(rng.integers(0, i))) for i in range(1, n)]
        length = rng.integers(1, 4 * C, size=n)
        compare(tpc, parent, length, C)


@pytest.mark.parametrize("mode", ["nodewise", "noreplay"])
@pytest.mark.parametrize("cfg", ["fig1", "single_fork", "agentic", "agentic_small", "wide"])
def test_ablation_planners_bit_exact_on_workloads(tpc, cfg, mode):
    w = synth.workload(cfg)
    compare(tpc, w.tree.parent, w.tree.length, w.chunk, mode)


@pytest.mark.parametrize("mode", ["nodewise", "noreplay"])
@pytest.mark.parametrize("C", [16, 64])
def test_ablation_planners_bit_exact_random(tpc, C, mode):
    rng = np.random.default_rng(100 + C + MODE_CODE[mode])
    for _ in range(300):
        n = int(rng.integers(1, 40))
        parent = [-1] + [(-1 if rng.random() < 0.05 else int(rng.integers(0, i))) for i in range(1, n)]
        length = rng.integers(1, 4 * C, size=n)
        compare(tpc, parent, length, C, mode)


def test_ablation_planners_on_fig1(tpc):
    """Fig. 1 tree (A 40 -> B 24, C 17; B -> D 9, E 31), chunk 16, worked by hand from the two
    ablation rules.  Node-wise: A in call 1; B, C start at 32 from A's state (8 replayed rows each)
    in call 2; D, E start at 64 from B's state in call 3; chunks 3 + 2 + 2 + 1 + 2 = 10.
    No replay: the minimum-call structure of the main plan (call 1 = A, B, D; call 2 = C, E) with
    C starting at 40 and no replayed row, so A-B-D is cut at 40 to export that state: chunks
    [0,16) [16,32) [32,40) [40,48) [48,64) [64,73), C [40,56) [56,57), E [64,80) [80,95) = 10."""
    w = synth.workload("fig1")
    t = w.tree
    nw = tpc.Plan(t.parent, t.length, 16, tpc.PLAN_NODEWISE)
    tb = nw.tables()
    assert nw.info["n_rounds"] == 3 and list(tb["round"]) == [1, 2, 2, 3, 3]
    assert list(tb["is_cont"]) == [0, 0, 0, 0, 0] and list(tb["replay_len"]) == [0, 8, 8, 0, 0]
    assert nw.info["n_chunks"] == 10 and nw.info["replay_total"] == 16 and nw.info["n_seqs"] == 5
    nr = tpc.Plan(t.parent, t.length, 16, tpc.PLAN_NO_REPLAY)
    tb = nr.tables()
    assert nr.info["n_rounds"] == 2 and list(tb["round"]) == [1, 1, 2, 1, 2]
    assert list(tb["replay_len"]) == [0, -1, 0, -1, 0] and list(tb["replay_start"]) == [0, -1, 40, -1, 64]
    assert list(tb["anchor"]) == [-1, 0, 0, 1, 1]
    assert nr.info["n_chunks"] == 10 and nr.info["replay_total"] == 0
    with pytest.raises(tpc.TpcError) as e:
        tpc.Plan(t.parent, t.length, 16, 7)
    assert e.value.code == 3


def test_fig1_chunk_table(tpc):
    w = synth.workload("fig1")
    pl = tpc.Plan(w.tree.parent, w.tree.length, 16)
    assert pl.info["n_chunks"] == 9 and pl.info["n_rounds"] == 2 and pl.info["replay_total"] == 8
    assert pl.info["n_unique"] == 121 and pl.info["n_expanded"] == 225


def test_invalid_inputs_return_status(tpc):
    with pytest.raises(tpc.TpcError) as e:
        tpc.Plan([-1, 2, 0], [1, 1, 1], 16)
    assert e.value.code == 1
    with pytest.raises(tpc.TpcError) as e:
        tpc.Plan([-1, 0], [4, 0], 16)
    assert e.value.code == 1
    with pytest.raises(tpc.TpcError) as e:
        tpc.Plan([-1], [4], 48)
    assert e.value.code == 3
    assert tpc.lib().tpc_plan_device_bytes(None) == 0


def check_device_tables(pl, n_leaves, n_roots, C):
    """Bounds every kernel relies on: rows, replay indices, slots, consumers, leaves and imports."""
    d = pl.debug_tables()
    i = pl.info
    N, R = i["n_unique"], i["replay_total"]
    ns, nc, nsl = i["n_seqs"], i["n_chunks"], i["n_slots"]
    for si, (cb, n_ch, imp, leaf, head, rnd, start, nrep) in enumerate(d["seqs"]):
        assert 0 <= cb and cb + n_ch <= nc and n_ch >= 1
        assert -1 <= leaf < n_leaves and 1 <= rnd <= i["n_rounds"] and 0 <= nrep < C
        assert (0 <= imp < nsl) or (-n_roots <= imp <= -1)
    for ci, (seq, n, nrep, row0, rbase, slot, pos0, idx) in enumerate(d["chunks"]):
        assert 0 <= seq < ns and 1 <= n <= C and 0 <= nrep <= n
        assert 0 <= row0 and row0 + (n - nrep) <= N
        assert nrep == 0 or (0 <= rbase and rbase + nrep <= R)
        assert -1 <= slot < nsl
    for prod, ech, cb, ncons in d["slots"]:
        assert 0 <= prod < ns and 0 <= ech < nc and d["chunks"][ech][5] >= 0
        assert all(0 <= c < ns + i["n_exports"] for c in d["slot_cons"][cb:cb + ncons])
    assert np.all((d["replay_rows"] >= 0) & (d["replay_rows"] < N))


@pytest.mark.parametrize("mode", ["min_rounds", "nodewise", "noreplay"])
def test_device_tables_within_bounds(tpc, mode):
    for cfg in ("fig1", "agentic_small", "agentic", "single_fork"):
        w = synth.workload(cfg)
        t = w.tree
        pl = tpc.Plan(t.parent, t.length, w.chunk, MODE_CODE[mode])
        check_device_tables(pl, len(t.leaves()), int((t.parent < 0).sum()), w.chunk)
    rng = np.random.default_rng(5)
    for _ in range(200):
        n = int(rng.integers(1, 30))
        parent = np.array([-1] + [(-1 if rng.random() < 0.05 else int(rng.integers(0, i))) for i in range(1, n)],
                          np.int32)
        length = rng.integers(1, 150, size=n).astype(np.int32)
        pl = tpc.Plan(parent, length, 64, MODE_CODE[mode])
        has_child = np.zeros(n, bool)
        has_child[parent[parent >= 0]] = True
        check_device_tables(pl, int((~has_child).sum()), int((parent < 0).sum()), 64)

