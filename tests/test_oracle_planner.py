"""Pins for the oracle round planner: the HARTS figures' worked examples,
brute-force minimality and layout invariants."""
import json
import os

import numpy as np
import pytest

import synth
from oracle import planner as P

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_figure1_calls_and_occurrence():
    gd = load("fig1_plan.json")
    pl = P.plan(gd["parent"], gd["length"], gd["chunk"])
    assert pl.n_rounds == len(gd["calls"])
    for r, nodes in enumerate(gd["calls"], start=1):
        assert sorted(np.nonzero(pl.round == r)[0].tolist()) == sorted(nodes)
    r2 = [sq["nodes"] for sq in pl.seqs if sq["round"] == 2]
    assert sorted(r2) == sorted(gd["sequences_in_call_2"])
    r1 = [sq["nodes"] for sq in pl.seqs if sq["round"] == 1]
    assert r1 == [gd["calls"][0]]
    assert pl.occurrence[1] == gd["occurrence_B"]
    assert len(pl.leaves) == gd["n_trajectories"]
    # C replays A's positions 32..39 from the boundary at 32; E starts exactly at 64
    assert (pl.replay_start[2], pl.replay_len[2]) == (32, 8)
    assert (pl.replay_start[4], pl.replay_len[4]) == (64, 0)
    assert pl.row_offset.tolist() == [0, 40, 104, 64, 73]


def test_figure2c_replay_started_in_round_one():
    gd = load("fig2c_plan.json")
    pl = P.plan(gd["parent"], gd["length"], gd["chunk"])
    assert pl.round.tolist() == gd["round"]
    assert pl.cont.tolist() == gd["continuation"]
    heads = {sq["head"]: sq for sq in pl.seqs}
    for v in gd["replay_started"]:
        assert v in heads and heads[v]["replay"] > 0
    assert heads[2]["round"] == 1 and heads[2]["import_kind"] == "init"
    assert heads[0]["nodes"] == gd["round1_chain"]


def random_tree(rng, nmax, C):
    n = int(rng.integers(1, nmax + 1))
    parent = [-1]
    for i in range(1, n):
        parent.append(-1 if rng.random() < 0.08 else int(rng.integers(0, i)))
    length = rng.integers(1, 3 * C + 1, size=n)
    return parent, length


@pytest.mark.parametrize("C", [2, 4, 16])
def test_dp_matches_brute_force(C):
    rng = np.random.default_rng(100 + C)
    for _ in range(3500):
        parent, length = random_tree(rng, 9, C)
        assert P.plan(parent, length, C).n_rounds == P.brute_force_min_rounds(parent, length, C)


def test_continuation_never_worse_than_none():
    # taking a continuation child is never worse than starting every child independently
    rng = np.random.default_rng(7)
    for _ in range(500):
        parent, length = random_tree(rng, 8, 4)
        pl = P.plan(parent, length, 4)
        conts = pl.cont_child.copy()
        for v in range(len(parent)):
            if conts[v] >= 0:
                c2 = conts.copy()
                c2[v] = -1
                assert P.rounds_for_choice(parent, length, 4, c2) >= pl.n_rounds


@pytest.mark.parametrize("cfg", ["fig1", "single_fork", "agentic", "agentic_small", "wide"])
def test_plan_invariants(cfg):
    w = synth.workload(cfg)
    t = w.tree
    pl = P.plan(t.parent, t.length, w.chunk)
    # sum of occurrence counts over rows = expanded tokens
    assert int(np.sum(pl.occurrence * pl.length)) == t.n_expanded()
    # layout: a permutation of rows, every chain contiguous
    rows = np.concatenate([np.arange(pl.row_offset[v], pl.row_offset[v] + pl.length[v]) for v in range(t.n)])
    assert np.array_equal(np.sort(rows), np.arange(t.n_rows))
    covered = np.zeros(t.n_rows, np.int64)
    for sq in pl.seqs:
        assert 0 <= sq["replay"] < w.chunk
        assert sq["start"] % w.chunk == 0
        nodes = sq["nodes"]
        for a, b in zip(nodes[:-1], nodes[1:]):
            assert pl.row_offset[b] == pl.row_offset[a] + pl.length[a]
        for u in nodes:
            covered[pl.row_offset[u]:pl.row_offset[u] + pl.length[u]] += 1
    # every row is computed outside replay exactly once
    assert np.all(covered == 1)
    assert len(pl.seqs) == len(pl.leaves)
    # an imported slot is produced in an earlier round
    for sl in pl.slots:
        pr = pl.seqs[sl["producer_seq"]]["round"]
        for c in sl["consumers"]:
            assert pl.seqs[c]["round"] == pr + 1
            assert pl.seqs[c]["start"] == sl["b"]


def test_expected_rounds_of_workloads():
    assert P.plan(*_tl("single_fork")).n_rounds == 2
    assert P.plan(*_tl("fig1")).n_rounds == 2
    assert P.plan(*_tl("agentic")).n_rounds <= 6


def _tl(cfg):
    w = synth.workload(cfg)
    return w.tree.parent, w.tree.length, w.chunk


def test_invalid_trees_rejected():
    with pytest.raises(P.InvalidTree):
        P.plan([-1, 2, 0], [1, 1, 1], 4)      # parent order
    with pytest.raises(P.InvalidTree):
        P.plan([-1, 0], [1, 0], 4)            # zero-length segment
    with pytest.raises(P.InvalidTree):
        P.plan([-1, 5], [1, 1], 4)            # parent out of range
