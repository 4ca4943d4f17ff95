"""GPU parity of the tree-packed KDA path against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest

import synth
from kda_case import Case, TOL, err_ratio, node_order, to_torch_compact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpc():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def run_case(tpc, case: Case, out_dtype=None, split=False):
    import torch
    t = case.tree
    plan = tpc.Plan(t.parent, t.length, case.C).upload()
    x = to_torch_compact(case, plan)
    if case.d_o_exp is not None:
        # the occurrence sum runs on the device (deterministic, trajectory order)
        tb = plan.tables()
        d_o_exp = torch.tensor(case.d_o_exp, dtype=torch.float32, device="cuda")
        x["d_o"] = tpc.tpc_reduce_expanded_to_unique(plan, d_o_exp)
        assert np.allclose(x["d_o"].cpu().numpy(), plan.to_compact(case.d_o, t.node_start(), t.length), atol=1e-5)
    out_dtype = out_dtype or torch.float32
    o, fin, ws = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], x["init"], out_dtype=out_dtype,
                                     split=split)
    gr = tpc.tpc_kda_backward(plan, ws, x["q"], x["k"], x["v"], x["g"], x["beta"], x["d_o"], x["d_final"],
                              x["init"], out_dtype=out_dtype, split=split)
    torch.cuda.synchronize()
    tpc.tpc_status(plan, ws, case.H, case.d)
    res = dict(o=o, final=fin, **gr)
    res = {k: (v.float().cpu().numpy() if v is not None else None) for k, v in res.items()}
    for k in ("o", "dq", "dk", "dv", "dg", "dbeta"):
        res[k] = node_order(plan, case, res[k])
    return plan, res


def check(case, res, tol):
    o_ref, fin_ref = case.oracle_forward
    g_ref = case.oracle_backward
    errs = {"o": err_ratio(res["o"], o_ref), "final": err_ratio(res["final"], fin_ref)}
    for name, ref in zip(("dq", "dk", "dv", "dg", "dbeta"), g_ref[:5]):
        errs[name] = err_ratio(res[name], ref)
    if case.init is not None:
        roots = np.nonzero(case.tree.parent < 0)[0]
        errs["d_init"] = err_ratio(res["d_init"], g_ref[5][roots])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, (errs, tol)
    return errs


def test_fig1_fp32(tpc):
    w = synth.workload("fig1")
    case = Case(w.tree, w.H, w.dk, w.chunk, "f32", w.seed, expanded_do=True)
    plan, res = run_case(tpc, case)
    errs = check(case, res, TOL["f32"])
    print("fig1 errors", errs)


def test_fig1_fp32_with_initial_state(tpc):
    w = synth.workload("fig1")
    case = Case(w.tree, w.H, w.dk, w.chunk, "f32", 11, with_init=True)
    check(case, run_case(tpc, case)[1], TOL["f32"])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_forest_fp32(tpc, seed):
    # ragged segments (1..70 tokens), several roots, deep chains, partial chunks everywhere
    rng = np.random.default_rng(seed)
    n = 14
    parent = [-1] + [(-1 if rng.random() < 0.15 else int(rng.integers(0, i))) for i in range(1, n)]
    length = rng.integers(1, 70, size=n).astype(np.int32)
    tree = synth.Tree(np.array(parent, np.int32), length)
    case = Case(tree, 2, 32, 16, "f32", 100 + seed, with_init=(seed == 1))
    check(case, run_case(tpc, case)[1], TOL["f32"])


@pytest.mark.parametrize("H", [1, 3, 6])
def test_tensor_core_path_head_counts(tpc, H):
    """bf16 at chunk 64 / d 128 on a ragged forest (replays, several roots, partial chunks) with head
    counts that the chunk kernels split differently over their CTAs: one head per CTA (H = 1, 3)
    and two heads per CTA over an odd number of CTAs per chunk (H = 6)."""
    rng = np.random.default_rng(40 + H)
    n = 9
    parent = [-1] + [(-1 if rng.random() < 0.15 else int(rng.integers(0, i))) for i in range(1, n)]
    length = rng.integers(1, 150, size=n).astype(np.int32)
    tree = synth.Tree(np.array(parent, np.int32), length)
    case = Case(tree, H, 128, 64, "bf16", 300 + H, with_init=(H == 3))
    errs = check(case, run_case(tpc, case)[1], TOL["bf16"])
    print("head count", H, errs)


def test_single_segment_and_short_tree(tpc):
    for tree in (synth.Tree(np.array([-1], np.int32), np.array([1], np.int32)),
                 synth.Tree(np.array([-1, 0, 0], np.int32), np.array([16, 16, 1], np.int32))):
        case = Case(tree, 1, 32, 16, "f32", 5)
        check(case, run_case(tpc, case)[1], TOL["f32"])


def test_agentic_small_bf16(tpc):
    w = synth.workload("agentic_small")
    case = Case(w.tree, 4, 128, 64, "bf16", w.seed)
    errs = check(case, run_case(tpc, case)[1], TOL["bf16"])
    print("agentic_small errors", errs)


def test_agentic_small_fp32_split_inputs_on_tensor_cores(tpc):
    """fp32 inputs given as TPC_F32_SPLIT at d = 128, chunk 64 take the tensor-core kernels with
    bf16 hi/lo operands: the products carry about 16 significant bits, so the bound is the bf16 one."""
    w = synth.workload("agentic_small")
    case = Case(w.tree, 4, 128, 64, "f32", w.seed + 7)
    errs = check(case, run_case(tpc, case, split=True)[1], TOL["bf16"])
    print("agentic_small fp32-split errors", errs)


def test_agentic_small_fp32_exact_at_d128(tpc):
    """Plain fp32 inputs at d = 128, chunk 64 (with replay rows) take the fp32 CUDA-core kernels and
    meet the fp32 bound, 1e-5 of the RMS, for outputs, final states and every gradient."""
    w = synth.workload("agentic_small")
    case = Case(w.tree, 2, 128, 64, "f32", w.seed + 8, with_init=True)
    errs = check(case, run_case(tpc, case)[1], TOL["f32"])
    print("agentic_small fp32 exact errors", errs)


def test_kda_wrappers_reject_bad_tensors_before_launch(tpc):
    """Row count, shape, dtype, contiguity and device are checked before any kernel is launched."""
    import torch
    w = synth.workload("fig1")
    plan = tpc.Plan(w.tree.parent, w.tree.length, 16).upload()
    N = plan.info["n_unique"]
    good = lambda: torch.zeros(N, 2, 32, device="cuda")
    beta = torch.zeros(N, 2, device="cuda")
    n0 = tpc.tpc_launch_count()
    bad_cases = {
        "short": (torch.zeros(N - 1, 2, 32, device="cuda"), beta),
        "strided": (torch.zeros(N, 2, 64, device="cuda")[:, :, :32], beta),
        "dtype": (good().to(torch.bfloat16), beta),
        "host": (torch.zeros(N, 2, 32), beta),
        "beta_shape": (good(), torch.zeros(N, 3, device="cuda")),
    }
    for name, (kk, bb) in bad_cases.items():
        with pytest.raises(tpc.TpcError) as e:
            tpc.tpc_kda_forward(plan, good(), kk, good(), good(), bb)
        assert e.value.code == 2, name
    with pytest.raises(tpc.TpcError) as e:
        tpc.tpc_kda_forward_static(plan, good(), good(), good(), good(), beta[:5])
    assert e.value.code == 2
    assert tpc.tpc_launch_count() == n0


def test_tree_forward_bitwise_equals_expanded(tpc):
    """Same chunk grid -> same arithmetic: every trajectory's outputs and final state are
    bitwise equal between the tree-packed call and the trajectory-expanded call."""
    import torch
    w = synth.workload("agentic_small")
    t = w.tree
    case = Case(t, 2, 128, 64, "bf16", 9)
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    x = to_torch_compact(case, plan)
    o, fin, _ = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], out_dtype=torch.float32)
    tb = plan.tables()
    lens = np.diff(tb["traj_offset"]).astype(np.int32)
    eplan = tpc.Plan(np.full(len(lens), -1, np.int32), lens, 64).upload()
    xe = {k: tpc.tpc_gather_expanded(plan, x[k]) for k in ("q", "k", "v", "g", "beta")}
    oe, fine, _ = tpc.tpc_kda_forward(eplan, xe["q"], xe["k"], xe["v"], xe["g"], xe["beta"], out_dtype=torch.float32)
    o_exp_from_tree = tpc.tpc_gather_expanded(plan, o)
    assert torch.equal(o_exp_from_tree, oe)
    assert torch.equal(fin, fine)


def test_gate_range_is_reported(tpc):
    import torch
    tree = synth.Tree(np.array([-1], np.int32), np.array([40], np.int32))
    case = Case(tree, 1, 32, 16, "f32", 3)
    case.inputs = list(case.inputs)
    case.inputs[3] = case.inputs[3] * 0 - 20.0  # 16 rows of -20 per channel: decay 300 inside a sub-block
    plan = tpc.Plan(tree.parent, tree.length, 16).upload()
    x = to_torch_compact(case, plan)
    _, _, ws = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"])
    with pytest.raises(tpc.TpcError) as e:
        tpc.tpc_status(plan, ws, 1, 32)
    assert e.value.code == 9
    tpc.tpc_status(plan, ws, 1, 32)  # the status word was cleared


def test_occurrence_counts_and_abi_errors(tpc):
    import torch
    w = synth.workload("fig1")
    plan = tpc.Plan(w.tree.parent, w.tree.length, 16)
    with pytest.raises(tpc.TpcError) as e:  # tables not uploaded yet
        tpc.tpc_occurrence_counts(plan)
    assert e.value.code == 10
    plan.upload()
    cnt = tpc.tpc_occurrence_counts(plan).cpu().numpy()
    tb = plan.tables()
    expect = np.zeros(plan.info["n_unique"], np.int64)
    for v in range(w.tree.n):
        expect[tb["row_offset"][v]:tb["row_offset"][v] + w.tree.length[v]] = tb["occurrence"][v]
    assert np.array_equal(cnt, expect)
    q = torch.zeros(121, 2, 32, device="cuda")
    with pytest.raises(tpc.TpcError) as e:  # workspace too small
        tpc.tpc_kda_forward(plan, q, q, q, q, torch.zeros(121, 2, device="cuda"), ws=torch.zeros(256, dtype=torch.uint8,
                                                                                                  device="cuda"))
    assert e.value.code == 5


def test_bounded_device_wait_reports_timeout(tpc):
    """A bounded mbarrier wait that runs out (nothing arrives; 1 ms limit) records TPC_ERR_TIMEOUT
    and returns; the context stays usable for the next launch."""
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tpc.tpc_debug_wait_timeout(status, 1_000_000)
    torch.cuda.synchronize()
    assert status.item() == 8
    status.zero_()
    assert torch.ones(4, device="cuda").sum().item() == 4.0



@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_outputs_written_exactly_inside_nan_canaries(tpc, out):
    """Every output of the forward and backward is a view into a NaN-filled buffer with 4096 NaN
    elements on both sides: afterwards the padding is still all NaN (no write outside an output) and
    the outputs hold no NaN (every element written).  Tensor-core path, replay rows, initial states."""
    import torch
    w = synth.workload("agentic_small")
    t = w.tree
    case = Case(t, 2, 128, 64, "bf16", w.seed + 31, with_init=True)
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    x = to_torch_compact(case, plan)
    N, H, d = x["q"].shape
    pad = 4096
    odt = torch.float32 if out == "f32" else torch.bfloat16
    bufs = []

    def canary(shape, dtype):
        n = int(np.prod(shape))
        buf = torch.full((pad + n + pad,), float("nan"), dtype=dtype, device="cuda")
        bufs.append((buf, n))
        return buf[pad:pad + n].view(shape)

    o = canary((N, H, d), odt)
    fin = canary((plan.info["n_leaves"], H, d, d), torch.float32)
    _, _, ws = tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], x["init"], out_dtype=odt,
                                   o=o, final_state=fin)
    grads = dict(dq=canary((N, H, d), odt), dk=canary((N, H, d), odt), dv=canary((N, H, d), odt),
                 dg=canary((N, H, d), torch.float32), dbeta=canary((N, H), torch.float32),
                 d_init=canary((plan.info["n_roots"], H, d, d), torch.float32))
    tpc.tpc_kda_backward(plan, ws, x["q"], x["k"], x["v"], x["g"], x["beta"], x["d_o"], x["d_final"], x["init"],
                         out_dtype=odt, grads=grads)
    torch.cuda.synchronize()
    tpc.tpc_status(plan, ws, H, d)
    for i, (buf, n) in enumerate(bufs):
        assert torch.isnan(buf[:pad]).all() and torch.isnan(buf[pad + n:]).all(), f"write outside output {i}"
        assert not torch.isnan(buf[pad:pad + n]).any(), f"output {i} not fully written"
