"""L1 microbatch planner (oracle side): compression-oriented packing of many rollout trees.

HARTS pages: the abstract says a two-level planner first constructs compression-oriented
microbatches and then refines membership, sharing, placement and order; Figure 1(c) shows the first
level (L1) forming microbatches from whole trees; Table 4 reports L1's compression, balance and
planning time; the work of a microbatch is measured in unique non-replayed token rows.  The pages
give no algorithm.  The plainest one that fits them, written out step by step:

  1. Trees (connected components of the parent-pointer forest) in increasing root id; the leaves of
     a tree (its trajectories) in depth-first order, children by increasing id, so that neighbouring
     trajectories share the longest prefixes.
  2. Pieces.  A tree whose unique tokens fit the budget is one piece (its sharing is kept whole).  A
     larger tree is cut: walk its leaves in depth-first order and add each leaf's path to the current
     piece; the cost of the piece is the number of tokens of the union of its paths; close the piece
     before a leaf whose new tokens would take it over the budget (a trajectory longer than the
     budget becomes a piece of its own).
  3. Microbatches.  Pieces sorted by cost, largest first (ties: smaller first leaf id), go first-fit
     into microbatches of capacity `budget`, the cost of a microbatch being the sum of its pieces'
     costs (pieces of different trees share nothing).

Reported: the microbatch of every leaf, and per microbatch its unique tokens (union of its
trajectories' paths) and expanded tokens (sum of their lengths); compression = total expanded /
total unique, balance = mean unique / max unique.

This module is test infrastructure: only tests and the benchmark's CPU baseline use it.
"""
from __future__ import annotations

import numpy as np


def _children(parent):
    ch = [[] for _ in range(len(parent))]
    for i, p in enumerate(parent):
        if p >= 0:
            ch[p].append(i)
    return ch


def _path(parent, v):
    out = []
    while v >= 0:
        out.append(int(v))
        v = int(parent[v])
    return out[::-1]


def union_tokens(parent, length, leaves) -> int:
    """Tokens of the union of the root-to-leaf paths of `leaves`."""
    nodes = set()
    for l in leaves:
        nodes.update(_path(parent, l))
    return int(sum(int(length[v]) for v in nodes))


def expanded_tokens(parent, length, leaves) -> int:
    return int(sum(sum(int(length[v]) for v in _path(parent, l)) for l in leaves))


def dfs_leaves(parent, root):
    ch = _children(parent)
    out, stack = [], [root]
    while stack:
        v = stack.pop()
        if not ch[v]:
            out.append(v)
        stack.extend(reversed(ch[v]))
    return out


def l1_plan(parent, length, budget):
    """Returns (leaf_mb: dict leaf -> microbatch, mb_unique list, mb_expanded list)."""
    parent = np.asarray(parent, np.int64)
    length = np.asarray(length, np.int64)
    if budget < 1:
        raise ValueError("budget must be >= 1")
    n = len(parent)
    roots = [v for v in range(n) if parent[v] < 0]
    pieces = []  # (cost, leaves)
    for r in roots:
        leaves = dfs_leaves(parent, r)
        whole = union_tokens(parent, length, leaves)
        if whole <= budget:
            pieces.append((whole, leaves))
            continue
        cur, cur_nodes, cost = [], set(), 0
        for l in leaves:
            path = _path(parent, l)
            new = sum(int(length[v]) for v in path if v not in cur_nodes)
            if cur and cost + new > budget:
                pieces.append((cost, cur))
                cur, cur_nodes, cost = [], set(), 0
                new = sum(int(length[v]) for v in path)
            cur.append(l)
            cur_nodes.update(path)
            cost += new
        pieces.append((cost, cur))
    pieces.sort(key=lambda p: (-p[0], p[1][0]))
    bins = []  # [load, [leaves]]
    for cost, leaves in pieces:
        for b in bins:
            if b[0] + cost <= budget:
                b[0] += cost
                b[1].extend(leaves)
                break
        else:
            bins.append([cost, list(leaves)])
    leaf_mb = {}
    mb_u, mb_e = [], []
    for m, (_, leaves) in enumerate(bins):
        for l in leaves:
            leaf_mb[l] = m
        mb_u.append(union_tokens(parent, length, leaves))
        mb_e.append(expanded_tokens(parent, length, leaves))
    return leaf_mb, mb_u, mb_e


def stats(mb_u, mb_e):
    tu, te = sum(mb_u), sum(mb_e)
    return dict(n_microbatches=len(mb_u), unique=tu, expanded=te, compression=te / tu,
                balance=(tu / len(mb_u)) / max(mb_u))


def brute_force(parent, length, budget):
    """Over every partition of the leaves into groups whose union fits the budget (groups holding a
    single over-long trajectory allowed): the fewest groups, and among those the fewest unique
    tokens.  Exponential; for tiny forests only."""
    parent = np.asarray(parent, np.int64)
    length = np.asarray(length, np.int64)
    leaves = [v for v in range(len(parent)) if not _children(parent)[v]]
    best = None

    def partitions(items):
        if not items:
            yield []
            return
        first, rest = items[0], items[1:]
        for p in partitions(rest):
            for i in range(len(p)):
                yield p[:i] + [[first] + p[i]] + p[i + 1:]
            yield [[first]] + p

    for part in partitions(leaves):
        ok = all(union_tokens(parent, length, g) <= budget or len(g) == 1 for g in part)
        if not ok:
            continue
        key = (len(part), sum(union_tokens(parent, length, g) for g in part))
        if best is None or key < best:
            best = key
    return best
