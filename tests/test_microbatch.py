"""L1 microbatch planner (HARTS abstract: compression-oriented microbatches; Figure 1(c); Table 4):
the C library against the oracle's step-by-step restatement, bit for bit, plus invariants, a worked
example and brute force on tiny forests.  CPU only."""
import numpy as np
import pytest

import synth
from oracle import microbatch as M


@pytest.fixture(scope="module")
def tpc():
    from tree_packed_chunkwise_b200 import build
    build.build()
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def leaves_of(parent):
    parent = np.asarray(parent)
    has_child = np.zeros(len(parent), bool)
    has_child[parent[parent >= 0]] = True
    return np.nonzero(~has_child)[0]


def compare(tpc, parent, length, budget):
    leaf_mb, mu, me, st = tpc.tpc_microbatch_plan(parent, length, budget)
    ref_mb, ref_u, ref_e = M.l1_plan(parent, length, budget)
    leaves = leaves_of(parent)
    assert [ref_mb[int(l)] for l in leaves] == list(leaf_mb)
    assert list(mu) == ref_u and list(me) == ref_e
    rs = M.stats(ref_u, ref_e)
    assert st["n_microbatches"] == rs["n_microbatches"] and st["unique_tokens"] == rs["unique"]
    assert st["expanded_tokens"] == rs["expanded"] and abs(st["compression"] - rs["compression"]) < 1e-12
    return leaf_mb, mu, me, st


def random_forest(rng, n_trees, max_nodes, max_len):
    parent, length = [], []
    for _ in range(n_trees):
        base = len(parent)
        m = int(rng.integers(1, max_nodes + 1))
        for i in range(m):
            parent.append(-1 if i == 0 else base + int(rng.integers(0, i)))
            length.append(int(rng.integers(1, max_len + 1)))
    return np.array(parent, np.int32), np.array(length, np.int32)


def test_l1_bit_exact_random(tpc):
    rng = np.random.default_rng(7)
    for _ in range(300):
        parent, length = random_forest(rng, int(rng.integers(1, 8)), 12, 200)
        budget = int(rng.integers(1, int(length.sum()) + 50))
        compare(tpc, parent, length, budget)


@pytest.mark.parametrize("budget", [20000, 65536, 250000])
def test_l1_bit_exact_many_agentic_trees(tpc, budget):
    trees = [synth.agentic_tree(seed=s) for s in range(10, 18)]
    parent, length = [], []
    for t in trees:
        base = len(parent)
        parent += [(-1 if p < 0 else base + int(p)) for p in t.parent]
        length += list(t.length)
    leaf_mb, mu, me, st = compare(tpc, np.array(parent, np.int32), np.array(length, np.int32), budget)
    # invariants: every microbatch within the budget unless it is one over-long trajectory; the union
    # accounting never compresses more than the whole forest would
    for m in range(st["n_microbatches"]):
        assert mu[m] <= budget or (leaf_mb == m).sum() == 1
    whole = sum(int(t.n_expanded()) for t in trees) / float(sum(int(t.n_rows) for t in trees))
    assert st["compression"] <= whole + 1e-12
    assert st["expanded_tokens"] == sum(int(t.n_expanded()) for t in trees)


def test_l1_worked_example(tpc):
    """Fig. 1 tree (A 40 -> B 24, C 17; B -> D 9, E 31: 121 unique, 225 expanded tokens) and a star
    (R 50 -> three children of 30: 140 unique, 240 expanded).  Budget 150: both fit whole, the
    140-token piece opens microbatch 0, the 121-token one cannot join it (261 > 150) and opens
    microbatch 1; compression 465 / 261.  Budget 100: the Fig. 1 tree is cut along its depth-first
    leaves D (A-B-D, 73), E (31 new tokens would make 104: new piece A-B-E, 95), C (17 new would
    make 112: new piece A-C, 57); the star into three pieces of 80; first fit of 95, 80, 80, 80, 73,
    57 under 100 gives six microbatches."""
    parent = np.array([-1, 0, 0, 1, 1, -1, 5, 5, 5], np.int32)
    length = np.array([40, 24, 17, 9, 31, 50, 30, 30, 30], np.int32)
    leaf_mb, mu, me, st = compare(tpc, parent, length, 150)
    assert st["n_microbatches"] == 2 and list(mu) == [140, 121] and list(me) == [240, 225]
    assert list(leaf_mb) == [1, 1, 1, 0, 0, 0]  # leaves 2, 3, 4 (tree 1) then 6, 7, 8 (the star)
    assert abs(st["compression"] - 465 / 261) < 1e-12
    leaf_mb, mu, me, st = compare(tpc, parent, length, 100)
    assert st["n_microbatches"] == 6 and sorted(mu) == [57, 73, 80, 80, 80, 95]


def test_l1_against_brute_force_on_tiny_forests(tpc):
    """The plan is a valid partition; its microbatch count is never below the true minimum, and on
    these tiny forests it reaches the minimum count in most cases (the rest are reported)."""
    rng = np.random.default_rng(11)
    hits = total = 0
    for _ in range(60):
        parent, length = random_forest(rng, int(rng.integers(1, 4)), 4, 40)
        if len(leaves_of(parent)) > 7:
            continue
        budget = int(rng.integers(1, int(length.sum()) + 10))
        _, mu, _, st = compare(tpc, parent, length, budget)
        best_n, best_u = M.brute_force(parent, length, budget)
        assert st["n_microbatches"] >= best_n
        assert st["n_microbatches"] > best_n or st["unique_tokens"] >= best_u
        total += 1
        hits += st["n_microbatches"] == best_n
    print(f"L1 reaches the minimum microbatch count on {hits} of {total} tiny forests")
    assert hits >= 0.7 * total


def test_l1_errors(tpc):
    with pytest.raises(tpc.TpcError) as e:
        tpc.tpc_microbatch_plan([-1, 0], [3, 4], 0)
    assert e.value.code == 2
    with pytest.raises(tpc.TpcError) as e:
        tpc.tpc_microbatch_plan([-1, 2, 0], [3, 4, 5], 10)
    assert e.value.code == 1


def test_microbatch_forest_extracts_paths(tpc):
    parent = np.array([-1, 0, 0, 1, 1, -1, 5], np.int32)
    length = np.array([5, 4, 3, 2, 1, 7, 6], np.int32)
    leaf_mb = np.array([0, 1, 0, 1])  # leaves 2, 3, 4, 6
    sp, sl, ids = tpc.microbatch_forest(parent, length, leaf_mb, 0)
    assert list(ids) == [0, 1, 2, 4] and list(sp) == [-1, 0, 0, 1] and list(sl) == [5, 4, 3, 1]
    sp, sl, ids = tpc.microbatch_forest(parent, length, leaf_mb, 1)
    assert list(ids) == [0, 1, 3, 5, 6] and list(sp) == [-1, 0, 1, -1, 3]
