"""Sharing windows across microbatches (HARTS abstract: within a sharing window, gradients from
dependent microbatches accumulate before one backward pass through the shared prefix computation;
Figure 3: the producer's backward runs inside the window's last consumer backward).

A rollout tree is cut at some nodes: the subtree under each cut node becomes a consumer
microbatch, the rest of the tree (the shared prefix) the producer microbatch.  A consumer starts at
the last chunk-aligned position b_c <= s_c of its cut node c and replays rows b_c .. s_c - 1 (its
own first segment, copied from the producer's rows, no output gradient), from the producer's
boundary state after token b_c - 1, which the producer's plan exports (tpc_plan_create_window).
Every trajectory therefore keeps its chunkwise numerical path: the forward results equal the
whole-tree run bit for bit.  Backward: every consumer first; their initial-state gradients are
summed per export (in consumer order) and enter the producer's single backward at the exported
boundaries; the consumers' replayed-row gradients are then added to the producer's rows.

Host logic and argument marshalling only: every arithmetic step runs in the library's kernels
(tpc_kda_forward / tpc_kda_backward_window / tpc_kda_export_states / tpc_gather_rows /
tpc_add_rows).  PyTorch provides device memory.
"""
from __future__ import annotations

import numpy as np

from . import (Plan, tpc_add_rows, tpc_gather_rows, tpc_kda_backward, tpc_kda_export_states, tpc_kda_forward)


def _starts(parent, length):
    s = np.zeros(len(parent), np.int64)
    for v in range(len(parent)):
        s[v] = 0 if parent[v] < 0 else s[parent[v]] + length[parent[v]]
    return s


def _node_rows(length):
    st = np.concatenate([[0], np.cumsum(length)[:-1]]).astype(np.int64)
    return st


class Microbatch:
    """One call's forest: parent/length, and for each of its compact rows the original node-order
    row of the whole tree it holds (after upload)."""

    def __init__(self, parent, length, node_rows, chunk, exports=None):
        self.parent = np.asarray(parent, np.int32)
        self.length = np.asarray(length, np.int32)
        self.node_rows = node_rows            # per node: original node-order rows of its tokens
        self.plan = Plan(self.parent, self.length, chunk, exports=exports)  # tables uploaded on first use
        own = self.plan.compact_source_rows(_node_rows(self.length), self.length)  # compact -> own node order
        flat = np.concatenate(node_rows) if node_rows else np.zeros(0, np.int64)
        self.orig_rows = flat[own]           # compact row -> original node-order row


class Window:
    def __init__(self, parent, length, chunk, cut_nodes):
        parent = np.asarray(parent, np.int64)
        length = np.asarray(length, np.int64)
        n = len(parent)
        self.C = chunk
        s = _starts(parent, length)
        st = _node_rows(length)
        rows_of = [np.arange(st[v], st[v] + length[v]) for v in range(n)]
        cut = sorted(int(c) for c in cut_nodes)
        in_sub = np.zeros(n, bool)
        owner = np.full(n, -1)
        for c in cut:
            if parent[c] < 0:
                raise ValueError(f"cut node {c} is a root")
        for v in range(n):  # parents before children
            if v in cut:
                if in_sub[parent[v]]:
                    raise ValueError(f"cut node {v} lies inside another cut subtree")
                in_sub[v], owner[v] = True, v
            elif parent[v] >= 0 and in_sub[parent[v]]:
                in_sub[v], owner[v] = True, owner[parent[v]]
        # producer: the nodes outside every cut subtree, renumbered by increasing id
        prod = np.nonzero(~in_sub)[0]
        pid = -np.ones(n, np.int64)
        pid[prod] = np.arange(len(prod))
        exports, self.cons_export = [], []
        for c in cut:
            b = (s[c] // chunk) * chunk
            if b == 0:
                self.cons_export.append(-1)
                continue
            u = parent[c]
            while s[u] > b - 1:
                u = parent[u]
            key = (int(pid[u]), int(b))
            if key not in exports:
                exports.append(key)
            self.cons_export.append(exports.index(key))
        self.producer = Microbatch(np.where(parent[prod] >= 0, pid[np.maximum(parent[prod], 0)], -1),
                                   length[prod], [rows_of[v] for v in prod], chunk, exports)
        self.exports = exports
        # consumers: [replayed segment b_c .. s_c - 1] -> the cut subtree
        self.consumers, self.replay_n = [], []
        for c in cut:
            nodes = [v for v in range(n) if owner[v] == c]
            b = (s[c] // chunk) * chunk
            rep = int(s[c] - b)
            path_rows = []
            u = c
            while parent[u] >= 0:
                u = parent[u]
                path_rows.append(u)
            traj = np.concatenate([rows_of[v] for v in reversed(path_rows)]) if path_rows else np.zeros(0, np.int64)
            rep_rows = traj[b:s[c]]
            cid = {v: i + (1 if rep else 0) for i, v in enumerate(nodes)}
            par = ([-1] if rep else []) + [(0 if rep else -1) if v == c else cid[int(parent[v])] for v in nodes]
            lens = ([rep] if rep else []) + [int(length[v]) for v in nodes]
            node_rows = ([rep_rows] if rep else []) + [rows_of[v] for v in nodes]
            self.consumers.append(Microbatch(par, lens, node_rows, chunk))
            self.replay_n.append(rep)
        # row maps: a consumer's replayed rows (compact rows of its first segment) -> producer rows
        inv = -np.ones(int(length.sum()), np.int64)
        inv[self.producer.orig_rows] = np.arange(len(self.producer.orig_rows))
        self.replay_src, self.replay_dst = [], []
        for mb, rep in zip(self.consumers, self.replay_n):
            mine = np.nonzero(np.isin(mb.orig_rows, mb.node_rows[0]))[0] if rep else np.zeros(0, np.int64)
            self.replay_src.append(mine)
            self.replay_dst.append(inv[mb.orig_rows[mine]])
        self._dev = None

    def _upload(self):
        import torch
        if self._dev is None:
            for mb in [self.producer] + self.consumers:
                mb.plan.upload()
            self._dev = ([torch.tensor(a, dtype=torch.int32, device="cuda") for a in self.replay_src],
                         [torch.tensor(a, dtype=torch.int32, device="cuda") for a in self.replay_dst])
        return self._dev

    # ------------------------------------------------------------------ calls
    def forward(self, prod_x, cons_x, out_dtype=None):
        """prod_x / cons_x[i]: dicts q, k, v, g, beta in each microbatch's compact order.  Returns
        (producer (o, final, ws), [consumer (o, final, ws)], exported states)."""
        self._upload()
        P = self.producer
        H, d = prod_x["q"].shape[1], prod_x["q"].shape[2]
        po = tpc_kda_forward(P.plan, prod_x["q"], prod_x["k"], prod_x["v"], prod_x["g"], prod_x["beta"],
                             out_dtype=out_dtype)
        states = tpc_kda_export_states(P.plan, po[2], H, d) if self.exports else None
        co = []
        for mb, x, e in zip(self.consumers, cons_x, self.cons_export):
            init = None if e < 0 else states[e:e + 1]
            co.append(tpc_kda_forward(mb.plan, x["q"], x["k"], x["v"], x["g"], x["beta"], init_state=init,
                                      out_dtype=out_dtype))
        return po, co, states

    def backward(self, prod_x, cons_x, fwd, out_dtype=None):
        """prod_x / cons_x[i] also hold d_o (zero on a consumer's replayed rows) and d_final.
        Consumers first; their initial-state gradients accumulate per export; then the producer's one
        backward; then the replayed-row gradients join the producer's rows.  Returns
        (producer grads, [consumer grads])."""
        import torch
        src_rows, dst_rows = self._upload()
        (po, co, states) = fwd
        H, d = prod_x["q"].shape[1], prod_x["q"].shape[2]
        cg = []
        export_grads = None
        if self.exports:
            export_grads = torch.zeros(len(self.exports), H, d, d, dtype=torch.float32, device="cuda")
        for i, (mb, x, e) in enumerate(zip(self.consumers, cons_x, self.cons_export)):
            init = None if e < 0 else states[e:e + 1]
            g = tpc_kda_backward(mb.plan, co[i][2], x["q"], x["k"], x["v"], x["g"], x["beta"], x["d_o"],
                                 x.get("d_final"), init_state=init, out_dtype=out_dtype, want_d_init=e >= 0)
            if e >= 0:  # gradient of the exported state: summed over the consumers, in consumer order
                tpc_add_rows(g["d_init"], torch.tensor([e], dtype=torch.int32, device="cuda"), export_grads)
            cg.append(g)
        pg = tpc_kda_backward(self.producer.plan, po[2], prod_x["q"], prod_x["k"], prod_x["v"], prod_x["g"],
                              prod_x["beta"], prod_x["d_o"], prod_x.get("d_final"), out_dtype=out_dtype,
                              export_grads=export_grads, want_d_init=False)
        for i, g in enumerate(cg):
            if self.replay_n[i] == 0:
                continue
            for key in ("dk", "dv", "dg", "dbeta"):
                if g[key].dtype != torch.float32 or pg[key].dtype != torch.float32:
                    raise TypeError("replayed-row gradients accumulate in fp32 (out_dtype float32)")
                tpc_add_rows(tpc_gather_rows(g[key], src_rows[i]), dst_rows[i], pg[key])
        return pg, cg
