"""The allocation-free forward (tpc_kda_forward_static) against the regular forward.

Some callers cannot allocate device memory (a host runtime whose pool owns the device, or a
latency-critical path that must not pay a cudaMalloc); they call tpc_kda_forward_static, which
keeps its tables and workspace in a device array built into the library.  This file is collected
last so that a run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest

import synth
from kda_case import Case, TOL, err_ratio, to_torch_compact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpc():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def _case(name):
    if name == "fig1":
        w = synth.workload("fig1")
        return Case(w.tree, w.H, w.dk, w.chunk, "f32", 21), None
    w = synth.workload("agentic_small")
    import torch
    return Case(w.tree, 2, 128, 64, "bf16", 22), torch.float32


def _compare(tpc, case, out_dtype):
    import torch
    t = case.tree
    plan = tpc.Plan(t.parent, t.length, case.C)
    x_plan = tpc.Plan(t.parent, t.length, case.C).upload()
    x = to_torch_compact(case, x_plan)
    o_s, f_s = tpc.tpc_kda_forward_static(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], out_dtype=out_dtype)
    o_r, f_r, _ = tpc.tpc_kda_forward(x_plan, x["q"], x["k"], x["v"], x["g"], x["beta"], out_dtype=out_dtype)
    torch.cuda.synchronize()
    tol = TOL[case.dtype]
    assert err_ratio(o_s.float().cpu().numpy(), o_r.float().cpu().numpy()) <= tol
    assert err_ratio(f_s.cpu().numpy(), f_r.cpu().numpy()) <= tol


def test_static_forward_matches_regular_forward_twice_in_a_row(tpc):
    # two different problems back to back, then the first again: the shared array's leftover
    # contents from the previous call must not leak into the next result
    for name in ("fig1", "agentic_small", "fig1"):
        case, out_dtype = _case(name)
        _compare(tpc, case, out_dtype)


def test_static_forward_rejects_oversized_problem(tpc):
    import torch
    w = synth.workload("single_fork")
    plan = tpc.Plan(w.tree.parent, w.tree.length, 64)
    N = plan.info["n_unique"]
    z = torch.zeros(N, 16, 128, dtype=torch.bfloat16, device="cuda")
    zb = torch.zeros(N, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tpc.TpcError) as e:
        tpc.tpc_kda_forward_static(plan, z, z, z, z, zb)
    assert e.value.code == 5 and "bytes" in str(e.value)


def test_static_forward_status_word_is_readable(tpc):
    """The allocation-free forward keeps its status word in the built-in array; its kernel-side gate
    check is read (and cleared) by tpc_kda_static_status."""
    import torch
    tree = synth.Tree(np.array([-1], np.int32), np.array([40], np.int32))
    case = Case(tree, 1, 32, 16, "f32", 3)
    case.inputs = list(case.inputs)
    case.inputs[3] = case.inputs[3] * 0 - 20.0  # decay 300 inside a 16-row sub-block: out of range
    plan = tpc.Plan(tree.parent, tree.length, 16)
    x = to_torch_compact(case, tpc.Plan(tree.parent, tree.length, 16).upload())
    tpc.tpc_kda_forward_static(plan, x["q"], x["k"], x["v"], x["g"], x["beta"])
    with pytest.raises(tpc.TpcError) as e:
        tpc.tpc_kda_static_status()
    assert e.value.code == 9
    tpc.tpc_kda_static_status()  # cleared
    ok = Case(tree, 1, 32, 16, "f32", 4)
    y = to_torch_compact(ok, tpc.Plan(tree.parent, tree.length, 16).upload())
    tpc.tpc_kda_forward_static(plan, y["q"], y["k"], y["v"], y["g"], y["beta"])
    tpc.tpc_kda_static_status()

