"""Benchmark: tree-packed KDA forward + backward on one or more B200s.

One step = the whole hot path (planned rounds: forward and backward of the
tree-packed chunkwise KDA layer) over one synthetic rollout tree: the
single-fork tree (8192-token prefix -> 16 branches of U[512, 2048] tokens),
H = 16, d_k = d_v = 128, chunk 64, bf16 inputs with fp32 state.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tpc|reference]

N > 1 runs under torchrun: each rank processes its own tree (weak scaling, no
data-path collective); the time is the max over ranks.  Rank 0 prints one
JSON line.  ``--impl reference`` times the fp64 CPU oracle on bounded samples
of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "tree-packed KDA fwd+bwd tokens/s (unique & expanded); % of TC/HBM roofline"
WORKLOAD = "single_fork"

# algorithmic FLOP per processed token-head of each kernel (chunk C, head dim d): the matrix
# products of the chunkwise form, 2 C d per token for each product within a chunk and 2 d^2 for each
# product with a d x d state; forward kernels 10 C d + 6 d^2 in all, backward 18 C d + 14 d^2.  The
# reverse scan carries M^T dS and the output's state gradient Qbar^T dO - W^T (P^T dO) (one product
# with Qeff = Qbar - P W); the dq kernel forms P^T dO.
def kernel_flops(name, C, d):
    Cd, dd = C * d, d * d
    name = name[:-3] if name.endswith("_tc") else name
    return {"kda_fwd_prep": 6 * Cd, "kda_fwd_scan": 4 * dd, "kda_fwd_out": 4 * Cd + 2 * dd,
            "kda_bwd_scan": 8 * dd, "kda_bwd_dq": 8 * Cd + 4 * dd,
            "kda_bwd_dkv": 10 * Cd + 2 * dd}.get(name, 0)


# algorithmic HBM bytes per processed token-head of each kernel: the bytes of the layer's own
# tensors (q, k, v, g, beta, dO in; o, dq, dk, dv, dg, dbeta out; bf16 except dg/dbeta fp32) that
# the kernel must read or write; workspace traffic (chunk states, W, U, partials) is not counted
def kernel_bytes(name, d):
    name = name[:-3] if name.endswith("_tc") else name
    return {"kda_fwd_prep": 6 * d + 2, "kda_fwd_out": 8 * d, "kda_bwd_dq": 10 * d,
            "kda_bwd_dkv": 14 * d + 6}.get(name, 0)


# algorithmic HBM bytes per token-head of the whole step (bf16 I/O): forward reads q,k,v,g (8d)
# + beta (2) and writes o (2d); backward reads those and dO and writes dq,dk,dv (6d), dg (4d), dbeta (4)
def step_bytes_per_token_head(d):
    return (8 * d + 2 + 2 * d) + (8 * d + 2 + 2 * d + 6 * d + 4 * d + 4)


def step_flops_per_token_head(C, d):
    return 3 * (10 * C * d + 6 * d * d)


def _flat_numbers(j, prefix=""):
    """{dotted.key: number} of a nested JSON object."""
    out = {}
    if isinstance(j, dict):
        for k, v in j.items():
            out.update(_flat_numbers(v, f"{prefix}{k}."))
    elif isinstance(j, (int, float)) and not isinstance(j, bool):
        out[prefix[:-1].lower()] = float(j)
    return out


def _pick(nums, must, avoid=()):
    for k, v in nums.items():
        if all(m in k for m in must) and not any(a in k for a in avoid) and v > 0:
            return v
    return None


def load_peaks():
    """Measured HBM copy bandwidth (GB/s) and bf16 dense throughput (TFLOP/s, burst and sustained) of
    this machine's B200s from MEASURED_PEAKS.json when present (keys located by name: hbm_gbs,
    bf16_tflops, bf16_tflops_sustained or the like); the pool's earlier measurement otherwise."""
    fb = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, sustained=1400.0, sm_max_mhz=1965.0, source="fallback")
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        return fb
    try:
        with open(p) as f:
            nums = _flat_numbers(json.load(f))
    except (OSError, ValueError):
        return fb
    hbm = nums.get("hbm_gbs") or _pick(nums, ("hbm",), ("util", "frac", "pct"))
    bf16 = nums.get("bf16_tflops") or _pick(nums, ("bf16",), ("sustain", "util", "frac", "pct", "mhz", "clock"))
    sus = nums.get("bf16_tflops_sustained") or _pick(nums, ("bf16", "sustain"), ("mhz", "clock", "util", "frac"))
    if not hbm or not bf16:
        return fb
    return dict(hbm_gbs=hbm, bf16_tflops=bf16, sustained=sus, sm_max_mhz=nums.get("sm_max_mhz", 1965.0),
                source="measured")


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except FileNotFoundError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def setup_dist():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    """The maximum of x over the ranks (a scalar all-reduce outside the data path)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def source_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "tree_packed_chunkwise_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


TRAFFIC_SOURCES = ["kda_tc.cuh", "tc.cuh", "common.cuh"]


def committed_traffic(kernel):
    """dram bytes per launch from a committed ncu capture, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(kernel)
    if not e or e.get("source_hash") != source_hash(TRAFFIC_SOURCES):
        return None
    return e["bytes_per_launch"]


# ------------------------------------------------------------------------------------ CPU oracle
def oracle_sample(w, n_tokens, seed):
    """fp64 oracle fwd+bwd on a bounded sample: the first n_tokens of the first trajectory."""
    from oracle import kda as okda
    t = w.tree
    rows = t.trajectory_rows(t.leaves()[0])[:n_tokens]
    inp = synth.kda_inputs(seed, rows, w.H, w.dk, w.dv, w.dtype)
    d_o = synth.rows_normal(seed, synth.STREAM["d_o"], rows, w.H * w.dv, w.dtype).reshape(len(rows), w.H, w.dv)
    t0 = time.perf_counter()
    okda.forward(*inp)
    okda.backward(*inp, d_o)
    return time.perf_counter() - t0, len(rows)


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return 1


def run_reference(args, ws, rank):
    w = synth.workload(args.workload)
    if rank != 0:
        return
    n_tok = args.ref_tokens
    oracle_sample(w, 8, w.seed)  # warm caches / imports
    for _ in range(args.warmup):
        oracle_sample(w, 16, w.seed)
    tot_t, tot_n = 0.0, 0
    for _ in range(args.steps):
        dt, n = oracle_sample(w, n_tok, w.seed)
        tot_t += dt
        tot_n += n
    rate = tot_n / tot_t
    sample = f"first {n_tok} tokens of trajectory 0 (H={w.H}, d={w.dk}) fwd+bwd per step, fp64 numpy"
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "sample_tokens_per_step": n_tok},
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------ hybrid layer group
GROUP_WORKLOAD = "agentic"


def group_flops_per_row(depth):
    """Algorithmic FLOP of one unique row in the 3 KDA + 1 MLA group (forward + backward, the
    recomputation not counted): projections 2 D (4 D + H) + 2 D^2 per KDA layer, 2 D (3648) +
    2 (512)(2 D) + 2 D^2 for MLA, times 3 (backward = 2 x forward); attention 2 H (192 + 128)
    (depth + 1) times 3.5 (backward = 2.5 x forward); KDA core 3 (10 C d + 6 d^2) per head."""
    D, H, d, C = 2048, 16, 128, 64
    kda_proj = 2 * D * (4 * D + H) + 2 * D * D
    mla_proj = 2 * D * 3648 + 2 * 512 * 2 * D + 2 * D * D
    gemm = 3 * (3 * kda_proj + mla_proj)
    attn = 3.5 * 2 * H * (192 + 128) * (depth + 1)
    core = 3 * H * 3 * (10 * C * d + 6 * d * d)
    return gemm, attn, core


def measure_group(args, world, rank, tpc, torch, peaks):
    import synth.gpu as sgpu
    w = synth.workload(args.group_workload)
    t = w.tree
    seed = 3 + 1000 * rank
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    info = plan.info
    N, NE = info["n_unique"], info["n_expanded"]
    st = t.node_start()
    src_rows = torch.tensor(plan.compact_source_rows(st, t.length), dtype=torch.int32, device="cuda")
    D = 2048
    x = sgpu.normal_rows(seed, synth.STREAM["group_x"], src_rows, D, "f32")
    R = sgpu.normal_rows(seed, synth.STREAM["group_r"], None, D, "f32", shape=(NE,))
    shapes = synth.group_weight_shapes(3)
    W = {"kda": [tuple(sgpu.normal_rows(seed, synth.group_weight_stream(l, m), None, shp[1], "bf16", 0.02,
                                        shape=(shp[0],)) for m, shp in enumerate(pair))
                 for l, pair in enumerate(shapes["kda"])],
         "mla": tuple(sgpu.normal_rows(seed, synth.group_weight_stream(15, m), None, shp[1], "bf16", 0.02,
                                       shape=(shp[0],)) for m, shp in enumerate(shapes["mla"]))}
    ws = tpc.group_workspace(plan, 3)
    h = torch.empty(3, N, D, dtype=torch.float32, device="cuda")
    y = torch.empty(N, D, dtype=torch.float32, device="cuda")
    dx = torch.empty(N, D, dtype=torch.float32, device="cuda")
    grads = {"kda": [tuple(torch.empty(m.shape, dtype=torch.float32, device="cuda") for m in pair) for pair in W["kda"]],
             "mla": tuple(torch.empty(m.shape, dtype=torch.float32, device="cuda") for m in W["mla"])}
    stream = torch.cuda.current_stream()

    def step():
        tpc.tpc_group_forward(plan, W, x, ws, h=h, y=y)
        dy = tpc.tpc_reduce_expanded_to_unique(plan, R)
        tpc.tpc_group_backward(plan, W, x, h, dy, ws, dx=dx, grads=grads, reuse_forward=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    code = tpc.tpc_group_status(plan, ws, 3)
    K = max(1, args.group_steps)
    n0 = tpc.tpc_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = (tpc.tpc_launch_count() - n0) / K
    ms = max_over_ranks(e0.elapsed_time(e1), world) / K
    # per-kernel shares (separate pass, events around every launch)
    tpc.tpc_profile_enable(True)
    step()
    torch.cuda.synchronize()
    prof = tpc.tpc_profile_read()
    tpc.tpc_profile_enable(False)
    tot = sum(v[1] for v in prof.values())
    kern = {k: {"launches": n, "ms": v, "share": v / tot} for k, (n, v) in prof.items()}
    depth = np.concatenate([np.arange(a, a + l) for a, l in
                            zip([sum(int(t.length[u]) for u in t.path(v)[:-1]) for v in range(t.n)], t.length)])
    occ = depth  # rows in node order; the per-row count does not depend on the order
    gemm_f, attn_f, core_f = group_flops_per_row(occ)
    flops = float(N * gemm_f + attn_f.sum() + N * core_f)
    tflops = flops / (ms / 1e3) / 1e12
    peak = peaks["sustained"] or peaks["bf16_tflops"]
    gemm_ms = sum(v["ms"] for k, v in kern.items() if k.startswith("gemm"))
    attn_ms = sum(v["ms"] for k, v in kern.items() if k.startswith("attn"))
    return {"workload": w.name + " (hybrid group: 3 KDA + 1 MLA, D=2048)", "n_unique": N, "n_expanded": NE,
            "ms_per_step": ms, "unique_tokens_per_s": world * N / (ms / 1e3),
            "expanded_tokens_per_s": world * NE / (ms / 1e3), "status": code, "launches_per_step": launches,
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                         "algorithmic_tflop_per_step": flops / 1e12,
                         "gemm_tflop_per_step": float(N * gemm_f) / 1e12,
                         "attention_tflop_per_step": float(attn_f.sum()) / 1e12,
                         "peak_source": "bf16 sustained, " + peaks["source"]},
            "gemm_achieved_tflops": float(N * gemm_f) / 1e12 / (gemm_ms / 1e3) if gemm_ms else None,
            "attention_achieved_tflops": float(attn_f.sum()) / 1e12 / (attn_ms / 1e3) if attn_ms else None,
            "kernels": kern,
            "precision": "bf16 weights; fp32 activations and gradients, tensor-core products from bf16 hi/lo pairs"}


# ------------------------------------------------------------------------------------ wide tree + log-probs
def measure_wide(args, world, rank, tpc, torch, peaks):
    """The wide tree (512 trajectories on a 32,768-token prefix, two fork levels of 8): one KDA layer
    with H = 32 run as four independent groups of 8 heads (the heads of a KDA layer do not interact;
    one group's workspace fits the GPU, all 32 heads' would not), then per-position log-probability
    recovery with hidden 2048 and vocabulary 65,536, forward and backward."""
    import synth.gpu as sgpu
    w = synth.workload(args.wide_workload)
    t = w.tree
    seed = w.seed + 1000 * rank
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    info = plan.info
    N, NE, d, HG = info["n_unique"], info["n_expanded"], w.dk, 8
    groups = w.H // HG
    st = t.node_start()
    src_rows = torch.tensor(plan.compact_source_rows(st, t.length), dtype=torch.int32, device="cuda")
    bf = torch.bfloat16
    ins = []
    for gi in range(groups):
        sg = seed + 17 * (gi + 1)
        x = dict(zip(("q", "k", "v", "g", "beta"), sgpu.kda_inputs(sg, src_rows, HG, d, d, "bf16")))
        x["d_o"] = sgpu.normal_rows(sg, synth.STREAM["d_o"], src_rows, HG * d, "bf16").view(N, HG, d)
        x["d_final"] = sgpu.normal_rows(sg, synth.STREAM["d_final"], None, HG * d * d, "f32",
                                        shape=(info["n_leaves"],)).view(info["n_leaves"], HG, d, d)
        ins.append(x)
    shape = tpc.kda_shape(HG, d, tpc.TPC_BF16, tpc.TPC_BF16)
    wsb = tpc.alloc_workspace(plan, shape)
    outs = [dict(o=torch.empty(N, HG, d, dtype=bf, device="cuda"),
                 final=torch.empty(info["n_leaves"], HG, d, d, dtype=torch.float32, device="cuda"))
            for _ in range(groups)]
    grads = dict(dq=torch.empty(N, HG, d, dtype=bf, device="cuda"), dk=torch.empty(N, HG, d, dtype=bf, device="cuda"),
                 dv=torch.empty(N, HG, d, dtype=bf, device="cuda"),
                 dg=torch.empty(N, HG, d, dtype=torch.float32, device="cuda"),
                 dbeta=torch.empty(N, HG, dtype=torch.float32, device="cuda"), d_init=None)
    V, Dh, CR = 65536, 2048, 16384
    hid = sgpu.normal_rows(seed, synth.STREAM["h"], src_rows, Dh, "bf16")
    Wv = sgpu.normal_rows(seed, synth.STREAM["w_vocab"], None, Dh, "bf16", 0.02, shape=(V,))
    targets = torch.randint(0, V, (NE,), dtype=torch.int32, device="cuda",
                            generator=torch.Generator(device="cuda").manual_seed(seed))
    dlogp = sgpu.normal_rows(seed, synth.STREAM["d_logp"], None, 1, "f32", shape=(NE,)).view(NE)
    scratch = tpc.logprob_scratch(plan, V, CR)
    stream = torch.cuda.current_stream()

    def kda_part():
        for gi in range(groups):
            x, o = ins[gi], outs[gi]
            tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], ws=wsb, o=o["o"],
                                final_state=o["final"], out_dtype=bf)
            tpc.tpc_kda_backward(plan, wsb, x["q"], x["k"], x["v"], x["g"], x["beta"], x["d_o"], x["d_final"],
                                 out_dtype=bf, grads=grads)

    def logprob_part():
        logp, lse = tpc.tpc_logprob_forward(plan, hid, Wv, targets, chunk_rows=CR, scratch=scratch)
        tpc.tpc_logprob_backward(plan, hid, Wv, targets, dlogp, lse, chunk_rows=CR, scratch=scratch)

    def timed(fn, k):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(e0.elapsed_time(e1), world) / k

    for _ in range(args.warmup):
        kda_part()
        logprob_part()
    torch.cuda.synchronize()
    K = max(1, args.wide_steps)
    kda_ms = timed(kda_part, K)
    lp_ms = timed(logprob_part, K)
    tpc.tpc_profile_enable(True)
    logprob_part()
    torch.cuda.synchronize()
    prof = tpc.tpc_profile_read()
    tpc.tpc_profile_enable(False)
    gemm_ms = prof.get("gemm_bf16_tc", (0, 0.0))[1]
    lp_flops = 3 * 2.0 * Dh * V * N  # logits, dh, dW (the backward's recomputed logits not counted)
    kda_flops = 3.0 * w.H * (10 * 64 * d + 6 * d * d) * info["n_seq_tokens"]
    step_ms = kda_ms + lp_ms
    tflops = (lp_flops + kda_flops) / (step_ms / 1e3) / 1e12
    peak = peaks["sustained"] or peaks["bf16_tflops"]
    return {"workload": w.name + " + log-prob recovery (Dh 2048, V 65536)", "n_unique": N, "n_expanded": NE,
            "heads": w.H, "head_groups": groups, "ms_per_step": step_ms, "kda_ms": kda_ms, "logprob_ms": lp_ms,
            "unique_tokens_per_s": world * N / (step_ms / 1e3), "expanded_tokens_per_s": world * NE / (step_ms / 1e3),
            "logprob_kernels": {k: {"launches": n, "ms": v} for k, (n, v) in prof.items()},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                         "algorithmic_tflop_per_step": (lp_flops + kda_flops) / 1e12,
                         "logprob_gemm_achieved_tflops": (lp_flops + 2.0 * Dh * V * N) / 1e12 / (gemm_ms / 1e3)
                         if gemm_ms else None,
                         "peak_source": "bf16 sustained, " + peaks["source"]}}


# ------------------------------------------------------------------------------------ agentic tree (config 2)
def kda_step_timer(tpc, torch, plan, x, H, d, world, steps, warmup):
    """ms per tree-packed forward + backward (bf16 in / out, fp32 state) of one plan, device-timed."""
    bf = torch.bfloat16
    info = plan.info
    N = info["n_unique"]
    shape = tpc.kda_shape(H, d, tpc.TPC_BF16, tpc.TPC_BF16)
    ws = tpc.alloc_workspace(plan, shape)
    o = torch.empty(N, H, d, dtype=bf, device="cuda")
    fin = torch.empty(info["n_leaves"], H, d, d, dtype=torch.float32, device="cuda")
    gr = dict(dq=torch.empty(N, H, d, dtype=bf, device="cuda"), dk=torch.empty(N, H, d, dtype=bf, device="cuda"),
              dv=torch.empty(N, H, d, dtype=bf, device="cuda"),
              dg=torch.empty(N, H, d, dtype=torch.float32, device="cuda"),
              dbeta=torch.empty(N, H, dtype=torch.float32, device="cuda"), d_init=None)

    def step():
        tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], ws=ws, o=o, final_state=fin, out_dtype=bf)
        tpc.tpc_kda_backward(plan, ws, x["q"], x["k"], x["v"], x["g"], x["beta"], x["d_o"], x["d_final"],
                             out_dtype=bf, grads=gr)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    tpc.tpc_status(plan, ws, H, d)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    del ws
    return ms


def measure_agentic(args, world, rank, tpc, torch):
    """Config 2: the agentic tree (64 leaves, 5 fork levels, bounded replay), tree-packed forward +
    backward against the trajectory-expanded run of the same kernels; the planner's rounds; the two
    planner ablations (node-wise, no replay); a sharing window (producer + consumer microbatches)."""
    import synth.gpu as sgpu
    w = synth.workload("agentic")
    t = w.tree
    H, d = w.H, w.dk
    seed = w.seed + 1000 * rank
    out = {"workload": w.name}
    st = t.node_start()
    K, W = max(2, args.steps // 4), max(3, args.warmup)
    for mode, name in ((tpc.PLAN_MIN_ROUNDS, "tree"), (tpc.PLAN_NODEWISE, "nodewise"), (tpc.PLAN_NO_REPLAY, "noreplay")):
        plan = tpc.Plan(t.parent, t.length, 64, mode).upload()
        info = plan.info
        src = torch.tensor(plan.compact_source_rows(st, t.length), dtype=torch.int32, device="cuda")
        x = dict(zip(("q", "k", "v", "g", "beta"), sgpu.kda_inputs(seed, src, H, d, d, "bf16")))
        x["d_o"] = sgpu.normal_rows(seed, synth.STREAM["d_o"], src, H * d, "bf16").view(-1, H, d)
        x["d_final"] = sgpu.normal_rows(seed, synth.STREAM["d_final"], None, H * d * d, "f32",
                                        shape=(info["n_leaves"],)).view(info["n_leaves"], H, d, d)
        ms = kda_step_timer(tpc, torch, plan, x, H, d, world, K, W)
        rec = {"rounds": info["n_rounds"], "replay_rows": info["replay_total"], "chunks": info["n_chunks"],
               "sequences": info["n_seqs"], "ms_per_step": ms,
               "unique_tokens_per_s": world * info["n_unique"] / (ms / 1e3),
               "expanded_tokens_per_s": world * info["n_expanded"] / (ms / 1e3)}
        if name == "tree":
            out.update(n_unique=info["n_unique"], n_expanded=info["n_expanded"], **rec)
            # trajectory-expanded comparator: the same kernels, one sequence per trajectory
            tb = plan.tables()
            lens = np.diff(tb["traj_offset"]).astype(np.int32)
            eplan = tpc.Plan(np.full(len(lens), -1, np.int32), lens, 64).upload()
            xe = {k: tpc.tpc_gather_expanded(plan, x[k]) for k in ("q", "k", "v", "g", "beta", "d_o")}
            xe["d_final"] = x["d_final"]
            del x
            ems = kda_step_timer(tpc, torch, eplan, xe, H, d, world, 2, 2)
            out["expanded_path"] = {"ms_per_step": ems, "speedup_tree_vs_expanded": ems / ms,
                                    "target_speedup": info["n_expanded"] / info["n_seq_tokens"],
                                    "chunk_ratio": eplan.info["n_chunks"] / info["n_chunks"],
                                    "expanded_chunks": eplan.info["n_chunks"]}
            del xe
        else:
            out[name] = rec
        torch.cuda.empty_cache()
    return out


def measure_extras(args, world, rank, tpc, torch):
    """The L1 microbatch planner on a step of many trees, and compact MoE routing on the wide tree."""
    import synth.gpu as sgpu
    res = {}
    trees = [synth.agentic_tree(seed=s) for s in range(100, 132)]
    parent, length = [], []
    for tr in trees:
        base = len(parent)
        parent += [(-1 if p < 0 else base + int(p)) for p in tr.parent]
        length += list(tr.length)
    parent, length = np.array(parent, np.int32), np.array(length, np.int32)
    budget = 262144
    t0 = time.perf_counter()
    leaf_mb, mu, me, stats = tpc.tpc_microbatch_plan(parent, length, budget)
    dt = time.perf_counter() - t0
    whole = float(sum(int(tr.n_expanded()) for tr in trees)) / float(length.sum())
    res["microbatch_l1"] = {"trees": len(trees), "trajectories": int(len(leaf_mb)), "budget_unique_rows": budget,
                            "microbatches": stats["n_microbatches"], "compression": stats["compression"],
                            "compression_whole_trees": whole, "balance": stats["balance"], "plan_ms": dt * 1e3}
    w = synth.workload("wide")
    t = w.tree
    plan = tpc.Plan(t.parent, t.length, 64).upload()
    src = torch.tensor(plan.compact_source_rows(t.node_start(), t.length), dtype=torch.int32, device="cuda")
    Dh, E, k = 2048, 64, 2
    h = sgpu.normal_rows(41, synth.STREAM["h"], src, Dh, "bf16")
    wr = sgpu.normal_rows(41, synth.STREAM["w_vocab"], None, Dh, "bf16", 0.02, shape=(E,))
    routed = tpc.tpc_moe_route(plan, h, wr, k)
    tpc.tpc_moe_router_loss(plan, routed, k)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        routed = tpc.tpc_moe_route(plan, h, wr, k, scratch=routed["scratch"])
        tpc.tpc_moe_router_loss(plan, routed, k)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 3
    res["moe_routing"] = {"workload": w.name, "hidden": Dh, "experts": E, "top_k": k,
                          "unique_rows": plan.info["n_unique"], "positions": plan.info["n_expanded"],
                          "ms_route_and_loss": ms, "rows_per_s": plan.info["n_unique"] / (ms / 1e3),
                          "load_sum_equals_k_positions": int(routed["expert_load"].sum().item()) == k * plan.info["n_expanded"]}
    return res


# ------------------------------------------------------------------------------------ GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="tpc", choices=["tpc", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=192)
    ap.add_argument("--cpu-tokens", type=int, default=2048, help="oracle sample for cpu_baseline (about 10-15 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-expanded", action="store_true")
    ap.add_argument("--no-group", action="store_true", help="skip the hybrid layer group (3 KDA + 1 MLA) measurement")
    ap.add_argument("--group-steps", type=int, default=3)
    ap.add_argument("--group-workload", default=GROUP_WORKLOAD, help="tree of the hybrid group (agentic by default)")
    ap.add_argument("--no-wide", action="store_true", help="skip the wide tree with log-prob recovery")
    ap.add_argument("--wide-steps", type=int, default=2)
    ap.add_argument("--wide-workload", default="wide", help="tree of the log-prob measurement (a smaller one for profiling)")
    ap.add_argument("--workload", default=WORKLOAD, help="single_fork (default), agentic, agentic_small")
    ap.add_argument("--no-agentic", action="store_true", help="skip the agentic tree (config 2) and its ablations")
    ap.add_argument("--no-extras", action="store_true", help="skip the L1 microbatch planner and MoE routing")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "tpc" else args.warmup

    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, ws, rank)
        return

    import torch
    import tree_packed_chunkwise_b200 as tpc

    world, rank, local = setup_dist()
    w = synth.workload(args.workload)
    t = w.tree
    seed = w.seed + 1000 * rank
    plan = tpc.Plan(t.parent, t.length, w.chunk).upload()
    info = plan.info
    N, H, d = info["n_unique"], w.H, w.dk
    st = t.node_start()
    # inputs drawn on the device by the generator twin (same bits as synth's host generator)
    import synth.gpu as sgpu
    src_rows = torch.tensor(plan.compact_source_rows(st, t.length), dtype=torch.int32, device="cuda")
    bf = torch.bfloat16
    dev = dict(zip(("q", "k", "v", "g", "beta"), sgpu.kda_inputs(seed, src_rows, H, d, d, w.dtype)))
    dev["d_o"] = sgpu.normal_rows(seed, synth.STREAM["d_o"], src_rows, H * d, w.dtype).view(N, H, d)
    dev["d_final"] = sgpu.normal_rows(seed, synth.STREAM["d_final"], None, H * d * d, "f32",
                                      shape=(info["n_leaves"],)).view(info["n_leaves"], H, d, d)
    host = {k: v.cpu().pin_memory() for k, v in dev.items()}
    shape = tpc.kda_shape(H, d, tpc.TPC_BF16, tpc.TPC_BF16)
    wsb = tpc.alloc_workspace(plan, shape)
    outs = dict(o=torch.empty(N, H, d, dtype=bf, device="cuda"),
                final=torch.empty(info["n_leaves"], H, d, d, dtype=torch.float32, device="cuda"))
    grads = dict(dq=torch.empty(N, H, d, dtype=bf, device="cuda"), dk=torch.empty(N, H, d, dtype=bf, device="cuda"),
                 dv=torch.empty(N, H, d, dtype=bf, device="cuda"),
                 dg=torch.empty(N, H, d, dtype=torch.float32, device="cuda"),
                 dbeta=torch.empty(N, H, dtype=torch.float32, device="cuda"), d_init=None)
    stream = torch.cuda.current_stream()

    def step(x):
        tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], ws=wsb, o=outs["o"],
                            final_state=outs["final"], out_dtype=bf)
        tpc.tpc_kda_backward(plan, wsb, x["q"], x["k"], x["v"], x["g"], x["beta"], x["d_o"], x["d_final"],
                             out_dtype=bf, grads=grads)

    for _ in range(args.warmup):
        step(dev)
    torch.cuda.synchronize()
    tpc.tpc_status(plan, wsb, H, d)

    # ---- timed region: K steps, inputs + workspace (> 1 GB) far larger than L2
    n0 = tpc.tpc_launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step(dev)
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    launches = tpc.tpc_launch_count() - n0
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    ms_step = ms / args.steps
    value = world * N / (ms_step / 1e3)
    value_exp = world * info["n_expanded"] / (ms_step / 1e3)

    # ---- per-kernel durations (CUDA events around each launch, separate pass)
    tpc.tpc_profile_enable(True)
    for _ in range(args.steps):
        step(dev)
    torch.cuda.synchronize()
    prof = tpc.tpc_profile_read()
    tpc.tpc_profile_enable(False)
    tokens_proc = info["n_seq_tokens"]
    kern = {}
    for name, (n, tot) in prof.items():
        per = tot / n
        units = tokens_proc * H * args.steps / n  # token-heads one launch processes (averaged over launches)
        kern[name] = {"launches_per_step": n / args.steps, "ms_per_launch": per, "share": 0.0,
                      "gflop_per_launch": kernel_flops(name, w.chunk, d) * units / 1e9,
                      "gb_per_launch": kernel_bytes(name, d) * units / 1e9}
    total_ms = sum(v["ms_per_launch"] * v["launches_per_step"] for v in kern.values())
    for v in kern.values():
        v["share"] = v["ms_per_launch"] * v["launches_per_step"] / total_ms
    dom = max(kern, key=lambda k: kern[k]["share"])
    peaks = load_peaks()
    clocks = clk.summary()
    dk = kern[dom]
    # the KDA kernels sit below the B200 ridge point (tens of FLOP per algorithmic byte): HBM-bound
    achieved = dk["gb_per_launch"] / dk["ms_per_launch"] * 1e3  # GB/s
    tc_achieved = dk["gflop_per_launch"] / dk["ms_per_launch"]  # TFLOP/s
    roofline = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": committed_traffic(dom),
                "algorithmic_gb_per_launch": dk["gb_per_launch"],
                "tensor_frac": tc_achieved / peaks["bf16_tflops"], "tensor_achieved_tflops": tc_achieved,
                "peak_source": "measured HBM copy bandwidth (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
                else "fallback 6650 GB/s"}
    step_bytes = step_bytes_per_token_head(d) * tokens_proc * H
    step_flops = step_flops_per_token_head(w.chunk, d) * tokens_proc * H
    step_roof = {"hbm_frac": (step_bytes / (ms_step / 1e3)) / (peaks["hbm_gbs"] * 1e9),
                 "tc_frac": (step_flops / (ms_step / 1e3)) / (peaks["bf16_tflops"] * 1e12),
                 "algorithmic_bytes": step_bytes, "algorithmic_flops": step_flops, "peak_source": peaks["source"]}

    # ---- trajectory-expanded comparator: the same kernels, one sequence per trajectory
    expanded = None
    if not args.no_expanded:
        tb = plan.tables()
        lens = np.diff(tb["traj_offset"]).astype(np.int32)
        eplan = tpc.Plan(np.full(len(lens), -1, np.int32), lens, w.chunk).upload()
        xe = {k: tpc.tpc_gather_expanded(plan, dev[k]) for k in ("q", "k", "v", "g", "beta", "d_o")}
        xe["d_final"] = dev["d_final"]
        NE = eplan.info["n_unique"]
        ews = tpc.alloc_workspace(eplan, shape)
        eo = torch.empty(NE, H, d, dtype=bf, device="cuda")
        ef = torch.empty(eplan.info["n_leaves"], H, d, d, dtype=torch.float32, device="cuda")
        eg = {k: torch.empty_like(xe["q"]) for k in ("dq", "dk", "dv")}
        eg.update(dg=torch.empty(NE, H, d, dtype=torch.float32, device="cuda"),
                  dbeta=torch.empty(NE, H, dtype=torch.float32, device="cuda"), d_init=None)

        def estep():
            tpc.tpc_kda_forward(eplan, xe["q"], xe["k"], xe["v"], xe["g"], xe["beta"], ws=ews, o=eo, final_state=ef,
                                out_dtype=bf)
            tpc.tpc_kda_backward(eplan, ews, xe["q"], xe["k"], xe["v"], xe["g"], xe["beta"], xe["d_o"], xe["d_final"],
                                 out_dtype=bf, grads=eg)

        for _ in range(2):
            estep()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ek = max(2, args.steps // 4)
        e0.record(stream)
        for _ in range(ek):
            estep()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world) / ek
        # (the kernels work in whole chunks, so the chunk-count ratio bounds the speed-up they can reach)
        expanded = {"ms_per_step": ems, "expanded_tokens_per_s": world * info["n_expanded"] / (ems / 1e3),
                    "speedup_tree_vs_expanded": ems / ms_step,
                    "target_speedup": info["n_expanded"] / info["n_seq_tokens"],
                    "chunk_ratio": eplan.info["n_chunks"] / info["n_chunks"]}
        del ews, xe, eg

    # ---- end to end through the C ABI with host buffers: every step uploads its inputs from pinned
    # host memory and downloads its results, streamed: a copy stream uploads step i + 1's inputs
    # and downloads step i - 1's results while step i computes (two device buffer sets)
    e2e = None
    if not args.no_e2e:
        sets = [dev, {k: torch.empty_like(v) for k, v in dev.items()}]
        res = [dict(o=outs["o"], final=outs["final"], **{k: grads[k] for k in ("dq", "dk", "dv", "dg", "dbeta")}),
               None]
        res[1] = {k: torch.empty_like(v) for k, v in res[0].items()}
        hout = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in res[0].items()}
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(v.numel() * v.element_size() for v in hout.values())
        copy, down = torch.cuda.Stream(), torch.cuda.Stream()  # uploads and downloads (PCIe is duplex)
        ev = lambda: torch.cuda.Event()

        def run_one(x, r):
            tpc.tpc_kda_forward(plan, x["q"], x["k"], x["v"], x["g"], x["beta"], ws=wsb, o=r["o"],
                                final_state=r["final"], out_dtype=bf)
            gr = dict(r)
            gr["d_init"] = None
            tpc.tpc_kda_backward(plan, wsb, x["q"], x["k"], x["v"], x["g"], x["beta"], x["d_o"], x["d_final"],
                                 out_dtype=bf, grads=gr)

        def stream_steps(n):
            up = [None, None]     # set b's inputs have arrived
            done = [None, None]   # set b's compute (and so its inputs / results) is finished
            for b in range(min(2, n)):
                up[b] = ev()
                with torch.cuda.stream(copy):
                    for k in host:
                        sets[b][k].copy_(host[k], non_blocking=True)
                    up[b].record(copy)
            for i in range(n):
                b = i % 2
                stream.wait_event(up[b])
                run_one(sets[b], res[b])
                done[b] = ev()
                done[b].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(done[b])
                    for k in hout:
                        hout[k].copy_(res[b][k], non_blocking=True)
                    drained = ev()
                    drained.record(down)
                if i + 2 < n:  # next use of set b: step i + 2, after its inputs are consumed and results read
                    with torch.cuda.stream(copy):
                        copy.wait_event(done[b])
                        copy.wait_event(drained)
                        for k in host:
                            sets[b][k].copy_(host[k], non_blocking=True)
                        up[b] = ev()
                        up[b].record(copy)
            stream.wait_stream(copy)
            stream.wait_stream(down)

        stream_steps(3)
        torch.cuda.synchronize()
        barrier(world)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        stream_steps(args.steps)
        a1.record(stream)
        torch.cuda.synchronize()
        ams = max_over_ranks(a0.elapsed_time(a1), world) / args.steps
        e2e = {"value": world * N / (ams / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ams,
               "how": "per step: H2D of all inputs from pinned host memory, forward + backward through the C ABI, "
                      "D2H of all results; uploads and downloads run on two copy streams overlapping each "
                      "other and the neighbouring steps' compute (two device buffer sets); the timed region "
                      "spans all copies"}
        del sets, res

    # ---- the agentic tree (config 2), its planner ablations; L1 planner and MoE routing
    del wsb, outs, grads, dev
    torch.cuda.empty_cache()
    agentic = None if args.no_agentic else measure_agentic(args, world, rank, tpc, torch)
    extras = None if args.no_extras else measure_extras(args, world, rank, tpc, torch)
    torch.cuda.empty_cache()

    # ---- hybrid layer group on the agentic tree (KDA buffers released first)
    group = None
    if not args.no_group:
        torch.cuda.empty_cache()
        group = measure_group(args, world, rank, tpc, torch, peaks)
        torch.cuda.empty_cache()

    # ---- wide tree: KDA (H = 32) and log-probability recovery
    wide = None
    if not args.no_wide:
        torch.cuda.empty_cache()
        wide = measure_wide(args, world, rank, tpc, torch, peaks)
        torch.cuda.empty_cache()

    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, n = oracle_sample(w, args.cpu_tokens, seed)
        try:  # the same oracle with its BLAS pool held to one thread
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                dt1, n1 = oracle_sample(w, max(64, args.cpu_tokens // 4), seed)
            one = n1 / dt1
        except Exception:
            one = None
        cpu = {"value": n / dt, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
               "cpu_model": cpu_model(), "host_cpus": os.cpu_count(), "value_one_thread": one,
               "sample": f"first {n} tokens of trajectory 0 (H={H}, d={d}) fwd+bwd, fp64 numpy, {dt:.1f} s"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16 in/out, fp32 state and accumulation", "data": "synthetic",
                "config": {"workload": w.name, "n_unique": N, "n_expanded": info["n_expanded"],
                           "replay_rows": info["replay_total"], "rounds": info["n_rounds"], "chunk": w.chunk,
                           "heads": H, "head_dim": d, "parallelism": f"dp{world} (independent trees)",
                           "l2": "inputs+workspace > 1 GB per step, larger than L2"},
                "value_expanded": value_exp, "roofline": roofline, "step_roofline": step_roof,
                "kernels": kern, "gpu_launches": launches, "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu,
                "expanded_path": expanded, "agentic": agentic, "hybrid_group": group, "wide_logprob": wide,
                **(extras or {})}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
