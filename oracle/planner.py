"""Round planner for packed chunkwise linear-attention calls (oracle side).

HARTS pages: the abstract states that a linear-time planner reaches the
global minimum number of sequential linear-attention calls under the
packed chunkwise-call model; Figure 2 shows fork-free segments, direct
continuations (thick edges), replay-started side sequences and the rule
that a boundary state produced by a call can seed another sequence only
after that call returns; Figure 1 shows the resulting calls for its tree
(Call 1 = [A,B,D], Call 2 = [C] and [E]) and the occurrence count q_B = 2.

The pages give no algorithm.  The model used here (the plainest one that
fits the figures):
  * chunk grids are aligned to absolute trajectory positions (multiples of C);
  * a node v with start position s_v either continues its parent's
    sequence, or starts its own sequence at b_v = floor(s_v / C) * C from the
    boundary state after token b_v - 1 (produced by the anchor a(v), the node
    on v's path that holds that token; the initial state when b_v = 0),
    replaying tokens b_v .. s_v - 1 without writing outputs;
  * such a sequence runs one round after the anchor's round (round 1 when
    b_v = 0);
  * a sequence is a continuation chain; every internal node continues
    exactly one child.

Dynamic program: e(v) = (round an independent child sharing v's anchor
would get) - r(v), in {0, 1}.  For a child c of v, delta_c(e) = 1 when v
itself holds token b_c - 1, else e.  H(v, e) = extra rounds below v:
0 for a leaf, else min over the continued child c* of
max(H(c*, delta_c*(e)), max_{c != c*} delta_c(e) + H(c, 0)).
Ties: smaller H, then larger replay saved (s_c - b_c), then smaller id.

Ablation modes (HARTS Figure 4 compares node-wise linear attention, Figure 5 a variant without
replay; the pages describe neither further, so these are the plainest readings):
  * "nodewise": no node continues its parent; each node starts its own sequence at b_v from its
    anchor's boundary state (same bounded replay), one round after the anchor (round 1 if b_v = 0);
  * "noreplay": a side node starts exactly at s_v from the state after token s_v - 1 (its parent
    holds it), so b_v = s_v and a(v) = parent(v); the same dynamic program picks the continuations.
    Its producer must cut a chunk at s_v to export that state (chunk_count models the cuts).
"""
from __future__ import annotations

import dataclasses
import itertools
import numpy as np


class InvalidTree(ValueError):
    pass


def validate(parent, length):
    parent = np.asarray(parent)
    length = np.asarray(length)
    n = parent.shape[0]
    if length.shape[0] != n or n == 0:
        raise InvalidTree("empty tree or size mismatch")
    for i in range(n):
        if parent[i] != -1 and not (0 <= parent[i] < i):
            raise InvalidTree(f"node {i}: parent {parent[i]} must be -1 or < {i}")
        if length[i] < 1:
            raise InvalidTree(f"node {i}: length {length[i]} < 1")


def positions(parent, length):
    """s_v: absolute position of the first token of v on every trajectory through it."""
    n = len(parent)
    s = np.zeros(n, np.int64)
    for v in range(n):
        p = parent[v]
        s[v] = 0 if p < 0 else s[p] + length[p]
    return s


def anchors(parent, length, s, C):
    """b_v = floor(s_v/C)*C and a(v) = the node on v's path holding token b_v - 1 (-1 if b_v = 0)."""
    n = len(parent)
    b = (s // C) * C
    a = np.full(n, -1, np.int64)
    for v in range(n):
        if b[v] == 0:
            continue
        u = parent[v]
        while s[u] > b[v] - 1:
            u = parent[u]
        a[v] = u
    return b, a


@dataclasses.dataclass
class Plan:
    C: int
    parent: np.ndarray
    length: np.ndarray
    s: np.ndarray
    b: np.ndarray
    anchor: np.ndarray
    round: np.ndarray            # r(v), 1-based
    cont: np.ndarray             # 1 if v continues its parent's sequence
    cont_child: np.ndarray       # chosen continuation child, -1 for leaves
    replay_start: np.ndarray     # b_v for sequence heads (0 for roots), -1 for continuations
    replay_len: np.ndarray       # s_v - b_v for heads with b_v > 0 ... (0 for roots), -1 for continuations
    row_offset: np.ndarray       # compact-layout first row of v
    occurrence: np.ndarray       # number of trajectories (leaves) through v
    n_rounds: int
    seqs: list                   # list of dict(head, nodes, round, start, end, import_kind, import_id, leaf)
    slots: list                  # list of dict(anchor, b, producer_seq, consumers=[seq ids])
    leaves: np.ndarray

    @property
    def n_unique(self):
        return int(self.length.sum())

    @property
    def replay_total(self):
        return int(sum(sq["replay"] for sq in self.seqs))


def _children(parent):
    ch = [[] for _ in range(len(parent))]
    for i, p in enumerate(parent):
        if p >= 0:
            ch[p].append(i)
    return ch


MODES = ("min_rounds", "nodewise", "noreplay")


def plan(parent, length, C, mode="min_rounds") -> Plan:
    parent = np.asarray(parent, np.int64)
    length = np.asarray(length, np.int64)
    validate(parent, length)
    if mode not in MODES:
        raise ValueError(f"unknown mode {mode}")
    n = len(parent)
    ch = _children(parent)
    s = positions(parent, length)
    if mode == "noreplay":
        b = s.copy()                          # handoff exactly at the fork point
        a = np.where(parent >= 0, parent, -1)  # the parent holds token s_v - 1
    else:
        b, a = anchors(parent, length, s, C)

    def delta(v, c, e):
        return 1 if s[v] < b[c] else e

    # bottom-up DP over both values of e (children have larger ids)
    H = np.zeros((n, 2), np.int64)
    choice = np.full((n, 2), -1, np.int64)
    for v in range(n - 1, -1, -1):
        if not ch[v] or mode == "nodewise":
            continue
        for e in (0, 1):
            best = None
            for cs in ch[v]:
                h = H[cs, delta(v, cs, e)]
                for c in ch[v]:
                    if c != cs:
                        h = max(h, delta(v, c, e) + H[c, 0])
                key = (h, -(s[cs] - b[cs]), cs)
                if best is None or key < best:
                    best = key
            H[v, e] = best[0]
            choice[v, e] = best[2]

    # top-down assignment
    rnd = np.zeros(n, np.int64)
    ee = np.zeros(n, np.int64)
    cont = np.zeros(n, np.int64)
    cont_child = np.full(n, -1, np.int64)
    for v in range(n):
        if parent[v] < 0:
            rnd[v], ee[v] = 1, 0
        if mode == "nodewise":
            if parent[v] >= 0:
                rnd[v] = 1 if b[v] == 0 else rnd[a[v]] + 1
            continue
        if ch[v]:
            cs = choice[v, ee[v]]
            cont_child[v] = cs
            for c in ch[v]:
                if c == cs:
                    rnd[c] = rnd[v]
                    ee[c] = delta(v, c, ee[v])
                    cont[c] = 1
                else:
                    rnd[c] = rnd[v] + delta(v, c, ee[v])
                    ee[c] = 0
    roots = [v for v in range(n) if parent[v] < 0]
    n_rounds = int(rnd.max())
    if mode != "nodewise":
        assert n_rounds == int(1 + max(H[r, 0] for r in roots))

    # compact layout: DFS preorder, continuation child first, then others by id; roots by id
    row_offset = np.zeros(n, np.int64)
    nxt = 0
    stack = list(reversed(roots))
    while stack:
        v = stack.pop()
        row_offset[v] = nxt
        nxt += length[v]
        order = ([cont_child[v]] if cont_child[v] >= 0 else []) + [c for c in ch[v] if c != cont_child[v]]
        stack.extend(reversed(order))

    # occurrences
    occ = np.zeros(n, np.int64)
    for v in range(n - 1, -1, -1):
        if not ch[v]:
            occ[v] = 1
        if parent[v] >= 0:
            occ[parent[v]] += occ[v]

    # sequences: chains headed by roots and independent nodes, ordered by (round, head id)
    heads = [v for v in range(n) if parent[v] < 0 or not cont[v]]
    heads.sort(key=lambda v: (rnd[v], v))
    root_of = np.zeros(n, np.int64)
    for v in range(n):
        root_of[v] = v if parent[v] < 0 else root_of[parent[v]]
    replay_start = np.full(n, -1, np.int64)
    replay_len = np.full(n, -1, np.int64)
    seqs = []
    seq_of = np.full(n, -1, np.int64)
    for h in heads:
        nodes = [h]
        while cont_child[nodes[-1]] >= 0:
            nodes.append(cont_child[nodes[-1]])
        start = 0 if parent[h] < 0 else int(b[h])
        replay = int(s[h] - start)
        replay_start[h] = start
        replay_len[h] = replay
        sid = len(seqs)
        for u in nodes:
            seq_of[u] = sid
        last = nodes[-1]
        seqs.append(dict(head=int(h), nodes=[int(u) for u in nodes], round=int(rnd[h]), start=start,
                         end=int(s[last] + length[last]), replay=replay, leaf=int(last),
                         root=int(root_of[h]), import_kind=None, import_id=-1))

    # slots = distinct (anchor, b) over heads with b > 0; ordered by (producer round, producer seq, b)
    keyset = {}
    for sq in seqs:
        h = sq["head"]
        if parent[h] >= 0 and b[h] > 0:
            keyset.setdefault((int(a[h]), int(b[h])), []).append(sq)
    slot_keys = sorted(keyset, key=lambda k: (rnd[k[0]], seq_of[k[0]], k[1]))
    slots = []
    for sid, (an, bb) in enumerate(slot_keys):
        cons = sorted(keyset[(an, bb)], key=lambda sq: sq["head"])
        slots.append(dict(anchor=an, b=bb, producer_seq=int(seq_of[an]),
                          consumers=[seqs.index(c) for c in cons]))
        for c in cons:
            c["import_kind"] = "slot"
            c["import_id"] = sid
    for sq in seqs:
        if sq["import_kind"] is None:
            sq["import_kind"] = "init"
            sq["import_id"] = sq["root"]
    leaves = np.array([v for v in range(n) if not ch[v]], np.int64)
    return Plan(C=C, parent=parent, length=length, s=s, b=b, anchor=a, round=rnd, cont=cont,
                cont_child=cont_child, replay_start=replay_start, replay_len=replay_len,
                row_offset=row_offset, occurrence=occ, n_rounds=n_rounds, seqs=seqs, slots=slots,
                leaves=leaves)


def chunk_count(pl: Plan) -> int:
    """Chunks of the packed calls: each sequence is cut at multiples of C from its start and, in
    addition, wherever it exports a boundary state (only off the grid in no-replay plans)."""
    total = 0
    for si, sq in enumerate(pl.seqs):
        cuts = {sl["b"] for sl in pl.slots if sl["producer_seq"] == si}
        p0, start, end = sq["start"], sq["start"], sq["end"]
        while p0 < end:
            p1 = min(start + ((p0 - start) // pl.C + 1) * pl.C, end)
            later = [c for c in cuts if c > p0]
            if later:
                p1 = min(p1, min(later))
            total += 1
            p0 = p1
    return total


def handoff_depth(parent) -> np.ndarray:
    """Per node, the boundary-state handoffs on the way from the root to its first token: the
    segment boundaries on its path (its depth in the tree; the root is 0)."""
    parent = np.asarray(parent, np.int64)
    dep = np.zeros(len(parent), np.int64)
    for v in range(len(parent)):
        dep[v] = 0 if parent[v] < 0 else dep[parent[v]] + 1
    return dep


# ------------------------------------------------------------------ brute force
def rounds_for_choice(parent, length, C, conts):
    """Rounds implied by an arbitrary choice of continuation child per node (-1 = none)."""
    parent = np.asarray(parent, np.int64)
    length = np.asarray(length, np.int64)
    s = positions(parent, length)
    b, a = anchors(parent, length, s, C)
    n = len(parent)
    r = np.zeros(n, np.int64)
    for v in range(n):
        p = parent[v]
        if p < 0:
            r[v] = 1
        elif conts[p] == v:
            r[v] = r[p]
        else:
            r[v] = 1 if b[v] == 0 else r[a[v]] + 1
    return int(r.max())


def brute_force_min_rounds(parent, length, C):
    """Minimum number of rounds over every continuation choice, including 'no continuation'."""
    ch = _children(parent)
    internal = [v for v in range(len(parent)) if ch[v]]
    options = [[-1] + ch[v] for v in internal]
    best = None
    for combo in itertools.product(*options):
        conts = np.full(len(parent), -1, np.int64)
        for v, c in zip(internal, combo):
            conts[v] = c
        r = rounds_for_choice(parent, length, C, conts)
        best = r if best is None else min(best, r)
    return best


# ------------------------------------------------------------------ expanded maps
def expanded_rows(pl: Plan):
    """For every trajectory (leaves by id) the compact row of each position, concatenated."""
    out = []
    offs = [0]
    for leaf in pl.leaves:
        path = []
        v = int(leaf)
        while v >= 0:
            path.append(v)
            v = int(pl.parent[v])
        path = path[::-1]
        rows = np.concatenate([np.arange(pl.row_offset[u], pl.row_offset[u] + pl.length[u]) for u in path])
        out.append(rows)
        offs.append(offs[-1] + len(rows))
    return np.concatenate(out).astype(np.int64), np.array(offs, np.int64)
