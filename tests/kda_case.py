"""Test-case assembly for KDA parity: seeded inputs (synth), oracle results and the
same inputs in the library's compact layout."""
from __future__ import annotations

import functools

import numpy as np

import synth
from oracle import kda as okda


def err_ratio(gpu, ref, floor=1.0) -> float:
    """max |gpu - ref| / RMS(ref) over a whole tensor.

    A reference that is zero (e.g. the gate gradient of a single token read from the
    zero state, or dQ / dK of a row that attends to itself alone, where dP - delta
    cancels) has no meaningful RMS: the fp64 oracle leaves a cancellation residue of
    ~1e-17.  A reference whose RMS is below 1e-9 of ``floor`` counts as zero and its
    error is taken relative to ``floor`` (inputs and upstream gradients are O(1))."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    if not ref.size:
        return 0.0
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.max(np.abs(gpu - ref)) / (rms if rms > 1e-9 * floor else floor))


TOL = {"f32": 1e-5, "bf16": 2e-3}


class Case:
    def __init__(self, tree: synth.Tree, H, d, chunk, dtype, seed, with_init=False, expanded_do=False):
        self.tree, self.H, self.d, self.C, self.dtype, self.seed = tree, H, d, chunk, dtype, seed
        N = tree.n_rows
        self.inputs = synth.kda_inputs(seed, np.arange(N), H, d, d, dtype)
        leaves = tree.leaves()
        self.d_final = synth.normal_tensor(seed, synth.STREAM["d_final"], (len(leaves), H, d, d), "f32")
        if expanded_do:
            n_exp = tree.n_expanded()
            self.d_o_exp = synth.normal_tensor(seed, synth.STREAM["d_o_exp"], (n_exp, H, d), dtype)
            # occurrence sum (the definition of the gradient reaching a unique row)
            self.d_o = np.zeros((N, H, d))
            off = 0
            for leaf in leaves:
                rows = tree.trajectory_rows(leaf)
                np.add.at(self.d_o, rows, self.d_o_exp[off:off + len(rows)])
                off += len(rows)
        else:
            self.d_o_exp = None
            self.d_o = synth.normal_tensor(seed, synth.STREAM["d_o"], (N, H, d), dtype)
        roots = np.nonzero(tree.parent < 0)[0]
        self.init = None
        if with_init:
            self.init_roots = synth.normal_tensor(seed, synth.STREAM["init"], (len(roots), H, d, d), "f32", 0.5)
            self.init = np.zeros((tree.n, H, d, d))
            self.init[roots] = self.init_roots

    @functools.cached_property
    def oracle_forward(self):
        return okda.tree_forward(self.tree, self.inputs, self.init)

    @functools.cached_property
    def oracle_backward(self):
        return okda.tree_backward(self.tree, self.inputs, self.d_o, self.d_final, self.init)


def to_torch_compact(case: Case, plan, device="cuda"):
    """The case's node-order arrays in the plan's compact layout, as device tensors."""
    import torch
    t = case.tree
    st = t.node_start()
    dt = torch.bfloat16 if case.dtype == "bf16" else torch.float32
    comp = lambda a: plan.to_compact(a, st, t.length)
    q, k, v, g, b = (torch.tensor(comp(x), dtype=torch.float32).to(dt).to(device) for x in case.inputs)
    d_o = torch.tensor(comp(case.d_o), dtype=torch.float32).to(dt if case.d_o_exp is None else torch.float32).to(device)
    d_final = torch.tensor(case.d_final, dtype=torch.float32, device=device)
    init = None
    if case.init is not None:
        init = torch.tensor(case.init_roots, dtype=torch.float32, device=device)
    return dict(q=q, k=k, v=v, g=g, beta=b, d_o=d_o, d_final=d_final, init=init)


def node_order(plan, case: Case, arr):
    """Compact-order array -> node order."""
    t = case.tree
    tb = plan.tables()
    st = t.node_start()
    out = np.empty_like(arr)
    for v in range(t.n):
        out[st[v]:st[v] + t.length[v]] = arr[tb["row_offset"][v]:tb["row_offset"][v] + t.length[v]]
    return out
