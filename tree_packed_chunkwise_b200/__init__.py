"""Python binding of ``libtpc.so``: tree-packed chunkwise KDA on B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  PyTorch provides device memory and streams.  The
functions keep the C names of ``include/tpc.h``.  There is no CPU fallback:
without the built library or a CUDA device the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtpc.so")

TPC_F32, TPC_BF16, TPC_F32_SPLIT = 0, 1, 2
_STATUS = {0: "TPC_OK", 1: "TPC_ERR_INVALID_TREE", 2: "TPC_ERR_BAD_SHAPE", 3: "TPC_ERR_UNSUPPORTED",
           4: "TPC_ERR_NULL", 5: "TPC_ERR_WORKSPACE", 6: "TPC_ERR_CUDA", 7: "TPC_ERR_DEVICE_CHECK",
           8: "TPC_ERR_TIMEOUT", 9: "TPC_ERR_RANGE", 10: "TPC_ERR_STATE"}

i32p = ctypes.POINTER(ctypes.c_int32)
i64p = ctypes.POINTER(ctypes.c_int64)


class TpcError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{_STATUS.get(code, code)}: {msg}")
        self.code = code


class PlanInfo(ctypes.Structure):
    _fields_ = [("n_unique", ctypes.c_int64), ("n_expanded", ctypes.c_int64), ("replay_total", ctypes.c_int64),
                ("n_seq_tokens", ctypes.c_int64), ("n_nodes", ctypes.c_int32), ("n_rounds", ctypes.c_int32),
                ("n_seqs", ctypes.c_int32), ("n_chunks", ctypes.c_int32), ("n_slots", ctypes.c_int32),
                ("n_leaves", ctypes.c_int32), ("n_roots", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("max_seq_chunks", ctypes.c_int32), ("n_replay_targets", ctypes.c_int32),
                ("n_exports", ctypes.c_int32)]


class PlanTables(ctypes.Structure):
    _fields_ = [("round", i32p), ("is_cont", i32p), ("anchor", i32p), ("replay_start", i32p),
                ("replay_len", i32p), ("row_offset", i64p), ("occurrence", i32p), ("leaves", i32p),
                ("expanded_rows", i64p), ("traj_offset", i64p)]


class MicrobatchStats(ctypes.Structure):
    _fields_ = [("n_microbatches", ctypes.c_int32), ("unique_tokens", ctypes.c_int64),
                ("expanded_tokens", ctypes.c_int64), ("max_unique", ctypes.c_int64),
                ("compression", ctypes.c_double), ("balance", ctypes.c_double)]


class KdaShape(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32)]


class AttnShape(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32), ("scale", ctypes.c_float),
                ("io_dtype", ctypes.c_int32)]


class KdaFwdIO(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("g", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("init_state", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("final_state", ctypes.c_void_p)]


class KdaBwdIO(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("g", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("init_state", ctypes.c_void_p), ("d_o", ctypes.c_void_p),
                ("d_final", ctypes.c_void_p), ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p),
                ("dv", ctypes.c_void_p), ("dg", ctypes.c_void_p), ("dbeta", ctypes.c_void_p),
                ("d_init", ctypes.c_void_p)]


# exported symbols of include/tpc.h: name -> (restype, argtypes)
_V, _P = ctypes.c_void_p, ctypes.POINTER
GROUP_MAX_KDA = 8


class AttnLo(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("d_o", ctypes.c_void_p)]


class GroupShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("D", "H", "d_head", "d_rope", "d_latent", "n_kda", "reuse_forward")]


class GroupWeights(ctypes.Structure):
    _fields_ = [("kda", (ctypes.c_void_p * 2) * GROUP_MAX_KDA), ("mla", ctypes.c_void_p * 3)]


class GroupGrads(ctypes.Structure):
    _fields_ = [("kda", (ctypes.c_void_p * 2) * GROUP_MAX_KDA), ("mla", ctypes.c_void_p * 3)]


SIGNATURES = {
    "tpc_last_error": (ctypes.c_char_p, []),
    "tpc_version": (ctypes.c_char_p, []),
    "tpc_plan_create": (ctypes.c_int, [i32p, i32p, ctypes.c_int32, ctypes.c_int32, _P(_V)]),
    "tpc_plan_destroy": (None, [_V]),
    "tpc_microbatch_plan": (ctypes.c_int, [i32p, i32p, ctypes.c_int32, ctypes.c_int64, i32p, i64p, i64p,
                                           ctypes.c_int32, _P(MicrobatchStats)]),
    "tpc_plan_create_mode": (ctypes.c_int, [i32p, i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P(_V)]),
    "tpc_plan_create_window": (ctypes.c_int, [i32p, i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.c_int32, i32p, i64p, _P(_V)]),
    "tpc_kda_export_states": (ctypes.c_int, [_V, _P(KdaShape), _V, _V, _V]),
    "tpc_kda_backward_window": (ctypes.c_int, [_V, _P(KdaShape), _P(KdaBwdIO), _V, _V, ctypes.c_size_t, _V]),
    "tpc_gather_rows": (ctypes.c_int, [_V, _V, _V, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, _V]),
    "tpc_add_rows": (ctypes.c_int, [_V, _V, _V, ctypes.c_int64, ctypes.c_int64, _V]),
    "tpc_plan_get_info": (ctypes.c_int, [_V, _P(PlanInfo)]),
    "tpc_plan_export": (ctypes.c_int, [_V, _P(PlanTables)]),
    "tpc_plan_device_bytes": (ctypes.c_size_t, [_V]),
    "tpc_plan_debug_tables": (ctypes.c_int, [_V, _V, _V, _V, _V, _V]),
    "tpc_plan_upload": (ctypes.c_int, [_V, _V, ctypes.c_size_t, _V]),
    "tpc_kda_workspace_bytes": (ctypes.c_size_t, [_V, _P(KdaShape)]),
    "tpc_kda_forward": (ctypes.c_int, [_V, _P(KdaShape), _P(KdaFwdIO), _V, ctypes.c_size_t, _V]),
    "tpc_kda_backward": (ctypes.c_int, [_V, _P(KdaShape), _P(KdaBwdIO), _V, ctypes.c_size_t, _V]),
    "tpc_status": (ctypes.c_int, [_V, _P(KdaShape), _V, _V]),
    "tpc_reduce_expanded_to_unique": (ctypes.c_int, [_V, _V, _V, ctypes.c_int64, _V]),
    "tpc_gather_expanded": (ctypes.c_int, [_V, _V, _V, ctypes.c_int64, ctypes.c_int32, _V]),
    "tpc_occurrence_counts": (ctypes.c_int, [_V, _V, _V]),
    "tpc_kda_forward_static": (ctypes.c_int, [_V, _P(KdaShape), _P(KdaFwdIO), _V]),
    "tpc_kda_static_status": (ctypes.c_int, [_V]),
    "tpc_gemm_bf16": (ctypes.c_int, [_V, _V, _V, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_float, ctypes.c_float, _V, _V]),
    "tpc_gemm_split": (ctypes.c_int, [_V, _V, _V, _V, _V, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_float, ctypes.c_float, _V, _V]),
    "tpc_logprob_scratch_bytes": (ctypes.c_size_t, [_V, ctypes.c_int64, ctypes.c_int32]),
    "tpc_logprob_forward": (ctypes.c_int, [_V, _V, _V, ctypes.c_int64, ctypes.c_int64, _V, _V, _V, _V, ctypes.c_size_t,
                                           ctypes.c_int32, _V, _V]),
    "tpc_logprob_backward": (ctypes.c_int, [_V, _V, _V, ctypes.c_int64, ctypes.c_int64, _V, _V, _V, _V, _V, _V,
                                            ctypes.c_size_t, ctypes.c_int32, _V, _V]),
    "tpc_tree_attn_forward": (ctypes.c_int, [_V, _V, _V, _V, _V, _V, _V, _V, _V, _V]),
    "tpc_tree_attn_backward": (ctypes.c_int, [_V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V]),
    "tpc_rope_positions": (ctypes.c_int, [_V, _V, _V]),
    "tpc_moe_scratch_bytes": (ctypes.c_size_t, [_V, ctypes.c_int32]),
    "tpc_moe_route": (ctypes.c_int, [_V, _V, _V, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _V, _V, _V, _V, _V,
                                     _V, _V, ctypes.c_size_t, _V]),
    "tpc_moe_router_loss": (ctypes.c_int, [_V, _V, _V, _V, _V, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                           ctypes.c_float, _V, _V, _V, ctypes.c_size_t, _V]),
    "tpc_group_workspace_bytes": (ctypes.c_size_t, [_V, _P(GroupShape)]),
    "tpc_group_forward": (ctypes.c_int, [_V, _P(GroupShape), _P(GroupWeights), _V, _V, _V, _V, ctypes.c_size_t, _V]),
    "tpc_group_backward": (ctypes.c_int, [_V, _P(GroupShape), _P(GroupWeights), _V, _V, _V, _V, _P(GroupGrads), _V,
                                          ctypes.c_size_t, _V]),
    "tpc_group_status": (ctypes.c_int, [_V, _P(GroupShape), _V, _V]),
    "tpc_profile_enable": (None, [ctypes.c_int]),
    "tpc_profile_read": (ctypes.c_int, [ctypes.c_char_p, ctypes.c_size_t]),
    "tpc_launch_count": (ctypes.c_longlong, []),
    "tpc_debug_wait_timeout": (ctypes.c_int, [_V, ctypes.c_int64, _V]),
    "tpc_checks_enable": (None, [ctypes.c_int]),
    "tpc_checks_enabled": (ctypes.c_int, []),
    "tpc_plan_check_device": (ctypes.c_int, [_V, _V]),
    "tpc_plan_check_host": (ctypes.c_int, [_V, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32]),
    "tpc_debug_poke_table": (ctypes.c_int, [_V, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                            _P(ctypes.c_int32), _V]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run tree_packed_chunkwise_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc):
    if rc != 0:
        raise TpcError(rc, lib().tpc_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------------------------ plan
PLAN_MIN_ROUNDS, PLAN_NODEWISE, PLAN_NO_REPLAY = 0, 1, 2


class Plan:
    """Round plan of a rollout tree (host object; ``upload`` places its tables on the device).
    mode: PLAN_MIN_ROUNDS (default), or the ablations PLAN_NODEWISE / PLAN_NO_REPLAY."""

    def __init__(self, parent, length, chunk: int, mode: int = PLAN_MIN_ROUNDS, exports=None):
        """exports: optional [(node, position)] boundary states to export (tpc_plan_create_window)."""
        parent = np.ascontiguousarray(parent, np.int32)
        length = np.ascontiguousarray(length, np.int32)
        h = ctypes.c_void_p()
        ex = list(exports or [])
        en = np.ascontiguousarray([e[0] for e in ex] or [0], np.int32)
        ep = np.ascontiguousarray([e[1] for e in ex] or [0], np.int64)
        _check(lib().tpc_plan_create_window(parent.ctypes.data_as(i32p), length.ctypes.data_as(i32p),
                                            int(parent.shape[0]), int(chunk), int(mode), len(ex),
                                            en.ctypes.data_as(i32p), ep.ctypes.data_as(i64p), ctypes.byref(h)))
        self.mode = int(mode)
        self._h = h
        self.n_nodes = int(parent.shape[0])
        info = PlanInfo()
        _check(lib().tpc_plan_get_info(self._h, ctypes.byref(info)))
        self.info = {f: getattr(info, f) for f, _ in PlanInfo._fields_}
        self.dev_tables = None

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.tpc_plan_destroy(self._h)
            self._h = None

    @property
    def handle(self):
        return self._h

    def tables(self) -> dict:
        n, nl, ne = self.n_nodes, self.info["n_leaves"], self.info["n_expanded"]
        out = {k: np.zeros(n, np.int32) for k in ("round", "is_cont", "anchor", "replay_start", "replay_len",
                                                  "occurrence")}
        out["row_offset"] = np.zeros(n, np.int64)
        out["leaves"] = np.zeros(nl, np.int32)
        out["expanded_rows"] = np.zeros(ne, np.int64)
        out["traj_offset"] = np.zeros(nl + 1, np.int64)
        t = PlanTables(**{k: v.ctypes.data_as(i64p if v.dtype == np.int64 else i32p) for k, v in out.items()})
        _check(lib().tpc_plan_export(self._h, ctypes.byref(t)))
        return out

    def debug_tables(self) -> dict:
        """The device-facing sequence / chunk / slot tables (tpc_plan_debug_tables) as int32 arrays."""
        i = self.info
        seqs = np.zeros((i["n_seqs"], 8), np.int32)
        chunks = np.zeros((i["n_chunks"], 8), np.int32)
        slots = np.zeros((i["n_slots"], 4), np.int32)
        ncons = 0
        _check(lib().tpc_plan_debug_tables(self._h, None, None, slots.ctypes.data, None, None))
        ncons = int(slots[:, 3].sum()) if len(slots) else 0
        cons = np.zeros(max(ncons, 1), np.int32)
        rep = np.zeros(max(i["replay_total"], 1), np.int32)
        _check(lib().tpc_plan_debug_tables(self._h, seqs.ctypes.data, chunks.ctypes.data, slots.ctypes.data,
                                           cons.ctypes.data, rep.ctypes.data))
        return dict(seqs=seqs, chunks=chunks, slots=slots, slot_cons=cons[:ncons], replay_rows=rep[:i["replay_total"]])

    def upload(self, device="cuda", stream=None):
        import torch
        nbytes = int(lib().tpc_plan_device_bytes(self._h))
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _check(lib().tpc_plan_upload(self._h, _ptr(buf), nbytes, _stream_ptr(stream)))
        self.dev_tables = buf
        return self

    def check_device(self, stream=None):
        """Bounds every index field of the uploaded tables on the device (tpc_plan_check_device); raises
        TpcError(TPC_ERR_DEVICE_CHECK) naming the first bad entry."""
        _check(lib().tpc_plan_check_device(self._h, _stream_ptr(stream)))

    def check_host(self, table: int = -1, word: int = 0, value: int = 0):
        """The device-table checks on the host copy of the tables, with one word replaced when table >= 0."""
        _check(lib().tpc_plan_check_host(self._h, int(table), int(word), int(value)))

    def poke_table(self, table: int, word: int, value: int, stream=None) -> int:
        """Test hook: overwrites one int32 word of an uploaded table; returns the previous value."""
        old = ctypes.c_int32(0)
        _check(lib().tpc_debug_poke_table(self._h, int(table), int(word), int(value), ctypes.byref(old),
                                          _stream_ptr(stream)))
        return int(old.value)

    def compact_source_rows(self, node_start: np.ndarray, length: np.ndarray) -> np.ndarray:
        """For every compact row, the node-order row (rows of node 0, node 1, ...) it holds."""
        tb = self.tables()
        perm = np.empty(int(length.sum()), np.int64)
        for v in range(self.n_nodes):
            perm[tb["row_offset"][v]:tb["row_offset"][v] + length[v]] = np.arange(node_start[v], node_start[v] + length[v])
        return perm

    def to_compact(self, node_rows_array: np.ndarray, node_start: np.ndarray, length: np.ndarray) -> np.ndarray:
        """Reorders a node-order row array to the compact layout."""
        return node_rows_array[self.compact_source_rows(node_start, length)]


# ------------------------------------------------------------------------------------ microbatches
def tpc_microbatch_plan(parent, length, budget: int):
    """L1 microbatches of a forest: (leaf_mb [n_leaves] int32 in leaf-id order, mb_unique, mb_expanded,
    stats dict).  Host only."""
    parent = np.ascontiguousarray(parent, np.int32)
    length = np.ascontiguousarray(length, np.int32)
    n = int(parent.shape[0])
    has_child = np.zeros(n, bool)
    has_child[parent[parent >= 0]] = True
    n_leaves = int((~has_child).sum())
    leaf_mb = np.zeros(max(n_leaves, 1), np.int32)
    mu = np.zeros(max(n_leaves, 1), np.int64)
    me = np.zeros(max(n_leaves, 1), np.int64)
    st = MicrobatchStats()
    _check(lib().tpc_microbatch_plan(parent.ctypes.data_as(i32p), length.ctypes.data_as(i32p), n, int(budget),
                                     leaf_mb.ctypes.data_as(i32p), mu.ctypes.data_as(i64p), me.ctypes.data_as(i64p),
                                     len(mu), ctypes.byref(st)))
    m = st.n_microbatches
    return leaf_mb[:n_leaves], mu[:m], me[:m], {f: getattr(st, f) for f, _ in MicrobatchStats._fields_}


def microbatch_forest(parent, length, leaf_mb, m):
    """(parent, length, node ids) of the sub-forest holding microbatch m's trajectories (the nodes on
    their paths, renumbered in increasing original id)."""
    parent = np.asarray(parent, np.int64)
    n = len(parent)
    has_child = np.zeros(n, bool)
    has_child[parent[parent >= 0]] = True
    leaves = np.nonzero(~has_child)[0]
    keep = np.zeros(n, bool)
    for l in leaves[np.asarray(leaf_mb) == m]:
        v = int(l)
        while v >= 0 and not keep[v]:
            keep[v] = True
            v = int(parent[v])
    ids = np.nonzero(keep)[0]
    new = -np.ones(n, np.int64)
    new[ids] = np.arange(len(ids))
    sub_parent = np.where(parent[ids] >= 0, new[np.maximum(parent[ids], 0)], -1).astype(np.int32)
    return sub_parent, np.asarray(length)[ids].astype(np.int32), ids


# ------------------------------------------------------------------------------------ KDA
def _dtype_code(t, split=False):
    import torch
    if t.dtype == torch.bfloat16:
        return TPC_BF16
    return TPC_F32_SPLIT if split else TPC_F32


def _check_kda_tensors(plan: Plan, named: dict, d_final=None, init_state=None):
    """Raises TpcError (TPC_ERR_BAD_SHAPE) before any launch unless every per-row tensor has the
    plan's n_unique rows, shape [N, H, d] ([N, H] for beta), one dtype (bf16 or fp32), is
    contiguous and lives on the current CUDA device; the state tensors must be fp32 [n, H, d, d]."""
    import torch
    N = plan.info["n_unique"]
    q = named["q"]
    if q.dim() != 3:
        raise TpcError(2, f"q must be [N, H, d], got {tuple(q.shape)}")
    _, H, d = q.shape
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else None
    for name, t in named.items():
        want = (N, H) if name == "beta" else (N, H, d)
        if tuple(t.shape) != want:
            raise TpcError(2, f"{name} has shape {tuple(t.shape)}, expected {want} (n_unique = {N})")
        if t.dtype != q.dtype or t.dtype not in (torch.bfloat16, torch.float32):
            raise TpcError(2, f"{name} has dtype {t.dtype}; all inputs must share one dtype, bf16 or fp32")
        if not t.is_contiguous():
            raise TpcError(2, f"{name} is not contiguous")
        if t.device != dev:
            raise TpcError(2, f"{name} is on {t.device}, not the current device {dev}")
    for name, t, n in (("d_final", d_final, plan.info["n_leaves"]), ("init_state", init_state, plan.info["n_roots"])):
        if t is None:
            continue
        if tuple(t.shape) != (n, H, d, d) or t.dtype != torch.float32 or not t.is_contiguous() or t.device != dev:
            raise TpcError(2, f"{name} must be a contiguous fp32 [{n}, {H}, {d}, {d}] tensor on {dev}")


def kda_shape(H, d, in_dtype, out_dtype) -> KdaShape:
    return KdaShape(H, d, d, in_dtype, out_dtype)


def tpc_kda_workspace_bytes(plan: Plan, shape: KdaShape) -> int:
    return int(lib().tpc_kda_workspace_bytes(plan.handle, ctypes.byref(shape)))


def alloc_workspace(plan: Plan, shape: KdaShape, device="cuda"):
    import torch
    n = tpc_kda_workspace_bytes(plan, shape)
    if n == 0:
        raise TpcError(3, "unsupported shape for this plan")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def tpc_kda_forward(plan: Plan, q, k, v, g, beta, init_state=None, out_dtype=None, ws=None, o=None,
                    final_state=None, want_final=True, stream=None, split=False):
    """Tree-packed forward.  Tensors in compact row order; returns (o, final_state, ws).
    split: fp32 inputs on the tensor-core kernels as bf16 hi/lo pairs (TPC_F32_SPLIT) instead of
    the exact fp32 CUDA-core kernels."""
    import torch
    _check_kda_tensors(plan, dict(q=q, k=k, v=v, g=g, beta=beta), init_state=init_state)
    N, H, d = q.shape
    out_dtype = out_dtype or q.dtype
    shape = kda_shape(H, d, _dtype_code(q, split), TPC_BF16 if out_dtype == torch.bfloat16 else TPC_F32)
    if ws is None:
        ws = alloc_workspace(plan, shape, q.device)
    if o is None:
        o = torch.empty(N, H, d, dtype=out_dtype, device=q.device)
    if final_state is None and want_final:
        final_state = torch.empty(plan.info["n_leaves"], H, d, d, dtype=torch.float32, device=q.device)
    io = KdaFwdIO(_ptr(q).value, _ptr(k).value, _ptr(v).value, _ptr(g).value, _ptr(beta).value,
                  None if init_state is None else init_state.data_ptr(), o.data_ptr(),
                  None if final_state is None else final_state.data_ptr())
    _check(lib().tpc_kda_forward(plan.handle, ctypes.byref(shape), ctypes.byref(io), _ptr(ws), ws.numel(),
                                 _stream_ptr(stream)))
    return o, final_state, ws


def tpc_kda_forward_static(plan: Plan, q, k, v, g, beta, init_state=None, out_dtype=None, o=None,
                           final_state=None, want_final=True, stream=None):
    """Forward that allocates nothing on the device: tables and workspace live in the library's
    built-in scratch array (see include/tpc.h).  Returns (o, final_state)."""
    import torch
    _check_kda_tensors(plan, dict(q=q, k=k, v=v, g=g, beta=beta), init_state=init_state)
    N, H, d = q.shape
    out_dtype = out_dtype or q.dtype
    shape = kda_shape(H, d, _dtype_code(q), TPC_BF16 if out_dtype == torch.bfloat16 else TPC_F32)
    if o is None:
        o = torch.empty(N, H, d, dtype=out_dtype, device=q.device)
    if final_state is None and want_final:
        final_state = torch.empty(plan.info["n_leaves"], H, d, d, dtype=torch.float32, device=q.device)
    io = KdaFwdIO(q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(),
                  None if init_state is None else init_state.data_ptr(), o.data_ptr(),
                  None if final_state is None else final_state.data_ptr())
    _check(lib().tpc_kda_forward_static(plan.handle, ctypes.byref(shape), ctypes.byref(io), _stream_ptr(stream)))
    return o, final_state


def tpc_kda_static_status(stream=None):
    """Raises TpcError if a kernel-side check of the allocation-free forward failed (then clears it)."""
    _check(lib().tpc_kda_static_status(_stream_ptr(stream)))


def tpc_kda_export_states(plan: Plan, ws, H, d, stream=None):
    """The plan's exported boundary states after tpc_kda_forward: fp32 [n_exports, H, d, d]."""
    import torch
    out = torch.empty(plan.info["n_exports"], H, d, d, dtype=torch.float32, device=ws.device)
    shape = kda_shape(H, d, 0, 0)
    _check(lib().tpc_kda_export_states(plan.handle, ctypes.byref(shape), _ptr(ws), _ptr(out), _stream_ptr(stream)))
    return out


def tpc_gather_rows(src, rows, stream=None):
    """dst[i] = src[rows[i]] for a [R, ...] tensor (2- or 4-byte elements) and int32 device rows."""
    import torch
    width = int(np.prod(src.shape[1:]))
    out = torch.empty((rows.numel(),) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    _check(lib().tpc_gather_rows(_ptr(src), _ptr(rows), _ptr(out), rows.numel(), width, src.element_size(),
                                 _stream_ptr(stream)))
    return out


def tpc_add_rows(src, rows, dst, stream=None):
    """dst[rows[i]] += src[i] (fp32; distinct rows)."""
    width = int(np.prod(src.shape[1:]))
    _check(lib().tpc_add_rows(_ptr(src), _ptr(rows), _ptr(dst), rows.numel(), width, _stream_ptr(stream)))


def tpc_kda_backward(plan: Plan, ws, q, k, v, g, beta, d_o, d_final=None, init_state=None, out_dtype=None,
                     want_d_init=True, grads=None, stream=None, split=False, export_grads=None):
    """Backward; returns dict(dq, dk, dv, dg, dbeta, d_init).  split: as tpc_kda_forward (must match
    the forward that filled ws)."""
    import torch
    _check_kda_tensors(plan, dict(q=q, k=k, v=v, g=g, beta=beta, d_o=d_o), d_final=d_final, init_state=init_state)
    N, H, d = q.shape
    out_dtype = out_dtype or q.dtype
    shape = kda_shape(H, d, _dtype_code(q, split), TPC_BF16 if out_dtype == torch.bfloat16 else TPC_F32)
    if grads is None:
        dev = q.device
        grads = dict(dq=torch.empty(N, H, d, dtype=out_dtype, device=dev),
                     dk=torch.empty(N, H, d, dtype=out_dtype, device=dev),
                     dv=torch.empty(N, H, d, dtype=out_dtype, device=dev),
                     dg=torch.empty(N, H, d, dtype=torch.float32, device=dev),
                     dbeta=torch.empty(N, H, dtype=torch.float32, device=dev),
                     d_init=torch.empty(plan.info["n_roots"], H, d, d, dtype=torch.float32, device=dev)
                     if want_d_init else None)
    io = KdaBwdIO(q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(),
                  None if init_state is None else init_state.data_ptr(), d_o.data_ptr(),
                  None if d_final is None else d_final.data_ptr(),
                  grads["dq"].data_ptr(), grads["dk"].data_ptr(), grads["dv"].data_ptr(), grads["dg"].data_ptr(),
                  grads["dbeta"].data_ptr(), None if grads.get("d_init") is None else grads["d_init"].data_ptr())
    _check(lib().tpc_kda_backward_window(plan.handle, ctypes.byref(shape), ctypes.byref(io), _ptr(export_grads),
                                         _ptr(ws), ws.numel(), _stream_ptr(stream)))
    return grads


def tpc_status(plan: Plan, ws, H, d, stream=None):
    shape = kda_shape(H, d, 0, 0)
    _check(lib().tpc_status(plan.handle, ctypes.byref(shape), _ptr(ws), _stream_ptr(stream)))


def tpc_reduce_expanded_to_unique(plan: Plan, x_exp, stream=None):
    import torch
    width = int(np.prod(x_exp.shape[1:]))
    out = torch.empty((plan.info["n_unique"],) + tuple(x_exp.shape[1:]), dtype=torch.float32, device=x_exp.device)
    _check(lib().tpc_reduce_expanded_to_unique(plan.handle, _ptr(x_exp), _ptr(out), width, _stream_ptr(stream)))
    return out


def tpc_gather_expanded(plan: Plan, x_unique, stream=None):
    import torch
    width = int(np.prod(x_unique.shape[1:]))
    out = torch.empty((plan.info["n_expanded"],) + tuple(x_unique.shape[1:]), dtype=x_unique.dtype,
                      device=x_unique.device)
    _check(lib().tpc_gather_expanded(plan.handle, _ptr(x_unique), _ptr(out), width, x_unique.element_size(),
                                     _stream_ptr(stream)))
    return out


def tpc_occurrence_counts(plan: Plan, device="cuda", stream=None):
    import torch
    out = torch.empty(plan.info["n_unique"], dtype=torch.int32, device=device)
    _check(lib().tpc_occurrence_counts(plan.handle, _ptr(out), _stream_ptr(stream)))
    return out


# ------------------------------------------------------------------------------------ diagnostics
def tpc_profile_enable(on: bool):
    lib().tpc_profile_enable(1 if on else 0)


def tpc_profile_read() -> dict:
    """{kernel name: (launches, total ms)} of the launches recorded since the last read."""
    buf = ctypes.create_string_buffer(1 << 16)
    _check(lib().tpc_profile_read(buf, len(buf)))
    out = {}
    for line in buf.value.decode().splitlines():
        name, n, ms = line.split()
        out[name] = (int(n), float(ms))
    return out


def tpc_launch_count() -> int:
    return int(lib().tpc_launch_count())


def tpc_checks_enable(on: bool) -> None:
    """Index and bounds mode: every call that reads plan tables checks them on the device first."""
    lib().tpc_checks_enable(1 if on else 0)


def tpc_checks_enabled() -> bool:
    return bool(lib().tpc_checks_enabled())


def tpc_debug_wait_timeout(status, timeout_ns=1_000_000, stream=None):
    """Runs the library's bounded device wait on a barrier nothing arrives on; status (int32 device
    tensor) receives TPC_ERR_TIMEOUT."""
    _check(lib().tpc_debug_wait_timeout(_ptr(status), int(timeout_ns), _stream_ptr(stream)))


# ------------------------------------------------------------------------------------ dense products
def tpc_gemm_bf16(a, b, c=None, a_mn=False, b_mn=False, out_dtype=None, alpha=1.0, beta=0.0, status=None, stream=None):
    """C = alpha op(A) op(B) + beta C on tensor cores.  a: [M, K] (or [K, M] with a_mn), b: [N, K] (or [K, N]
    with b_mn), bf16, last dimension contiguous.  Returns C [M, N] (fp32 unless out_dtype is bf16)."""
    import torch
    M = a.shape[1] if a_mn else a.shape[0]
    K = a.shape[0] if a_mn else a.shape[1]
    N = b.shape[1] if b_mn else b.shape[0]
    if c is None:
        c = torch.empty(M, N, dtype=out_dtype or torch.float32, device=a.device)
    code = TPC_BF16 if c.dtype == torch.bfloat16 else TPC_F32
    _check(lib().tpc_gemm_bf16(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, a.stride(0), b.stride(0),
                               c.stride(0), int(a_mn), int(b_mn), code, float(alpha), float(beta),
                               None if status is None else status.data_ptr(), _stream_ptr(stream)))
    return c


def split_bf16(x):
    """(hi, lo) bf16 pair of an fp32 tensor: hi = bf16(x), lo = bf16(x - hi) (host-side helper for tests)."""
    import torch
    hi = x.to(torch.bfloat16)
    lo = (x - hi.float()).to(torch.bfloat16)
    return hi, lo


def tpc_gemm_split(a, a_lo, b, b_lo, c=None, a_mn=False, b_mn=False, alpha=1.0, beta=0.0, status=None, stream=None):
    """C = alpha (A B + A_lo B + A B_lo) + beta C; a_lo / b_lo may be None.  fp32 C."""
    import torch
    M = a.shape[1] if a_mn else a.shape[0]
    K = a.shape[0] if a_mn else a.shape[1]
    N = b.shape[1] if b_mn else b.shape[0]
    if c is None:
        c = torch.empty(M, N, dtype=torch.float32, device=a.device)
    _check(lib().tpc_gemm_split(a.data_ptr(), None if a_lo is None else a_lo.data_ptr(), b.data_ptr(),
                                None if b_lo is None else b_lo.data_ptr(), c.data_ptr(), M, N, K, a.stride(0),
                                b.stride(0), c.stride(0), int(a_mn), int(b_mn), TPC_F32, float(alpha), float(beta),
                                None if status is None else status.data_ptr(), _stream_ptr(stream)))
    return c


# ------------------------------------------------------------------------------------ log-probabilities
def logprob_scratch(plan: Plan, V, chunk_rows, device="cuda"):
    import torch
    n = int(lib().tpc_logprob_scratch_bytes(plan.handle, V, chunk_rows))
    return torch.empty(n, dtype=torch.uint8, device=device)


def tpc_logprob_forward(plan: Plan, h, W, targets, chunk_rows=2048, scratch=None, status=None, stream=None):
    """Per-occurrence log-probabilities (fp32 [n_expanded]) and per-row lse (fp32 [N_unique])."""
    import torch
    V, Dh = W.shape
    chunk_rows = min(chunk_rows, plan.info["n_unique"])
    scratch = scratch if scratch is not None else logprob_scratch(plan, V, chunk_rows, h.device)
    logp = torch.empty(plan.info["n_expanded"], dtype=torch.float32, device=h.device)
    lse = torch.empty(plan.info["n_unique"], dtype=torch.float32, device=h.device)
    _check(lib().tpc_logprob_forward(plan.handle, _ptr(h), _ptr(W), V, Dh, _ptr(targets), _ptr(logp), _ptr(lse),
                                     _ptr(scratch), scratch.numel(), chunk_rows, _ptr(status), _stream_ptr(stream)))
    return logp, lse


def tpc_logprob_backward(plan: Plan, h, W, targets, dlogp, lse, chunk_rows=2048, scratch=None, status=None,
                         stream=None):
    """Gradients (fp32) of sum(dlogp * logp) w.r.t. h [N_unique, Dh] and W [V, Dh]."""
    import torch
    V, Dh = W.shape
    chunk_rows = min(chunk_rows, plan.info["n_unique"])
    scratch = scratch if scratch is not None else logprob_scratch(plan, V, chunk_rows, h.device)
    dh = torch.empty(plan.info["n_unique"], Dh, dtype=torch.float32, device=h.device)
    dW = torch.empty(V, Dh, dtype=torch.float32, device=h.device)
    _check(lib().tpc_logprob_backward(plan.handle, _ptr(h), _ptr(W), V, Dh, _ptr(targets), _ptr(dlogp), _ptr(lse),
                                      _ptr(dh), _ptr(dW), _ptr(scratch), scratch.numel(), chunk_rows, _ptr(status),
                                      _stream_ptr(stream)))
    return dh, dW


# ------------------------------------------------------------------------------------ tree attention
def _attn_shape(q, v, scale, io_dtype):
    import torch
    return AttnShape(q.shape[1], q.shape[2], v.shape[2], float(scale),
                     TPC_BF16 if io_dtype == torch.bfloat16 else TPC_F32)


def _attn_lo(q_lo=None, k_lo=None, v_lo=None, d_o_lo=None):
    if q_lo is None and k_lo is None and v_lo is None and d_o_lo is None:
        return None
    dp = lambda t: None if t is None else t.data_ptr()
    return ctypes.byref(AttnLo(dp(q_lo), dp(k_lo), dp(v_lo), dp(d_o_lo)))


def tpc_tree_attn_forward(plan: Plan, q, k, v, scale, out_dtype=None, status=None, stream=None, q_lo=None, k_lo=None,
                          v_lo=None, o=None, lse=None):
    """Tree-masked attention forward; returns (o, lse).  *_lo: optional bf16 low parts (hi/lo pairs)."""
    import torch
    out_dtype = out_dtype or torch.float32
    N, H, _ = q.shape
    o = o if o is not None else torch.empty(N, H, v.shape[2], dtype=out_dtype, device=q.device)
    lse = lse if lse is not None else torch.empty(N, H, dtype=torch.float32, device=q.device)
    sh = _attn_shape(q, v, scale, o.dtype)
    _check(lib().tpc_tree_attn_forward(plan.handle, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v),
                                       _attn_lo(q_lo, k_lo, v_lo), _ptr(o), _ptr(lse), _ptr(status),
                                       _stream_ptr(stream)))
    return o, lse


def tpc_tree_attn_backward(plan: Plan, q, k, v, o, lse, d_o, scale, status=None, stream=None, q_lo=None, k_lo=None,
                           v_lo=None, d_o_lo=None):
    """Gradients (dq, dk, dv) in o's dtype.  *_lo: optional bf16 low parts (hi/lo pairs)."""
    import torch
    N, H, _ = q.shape
    dq = torch.empty(q.shape, dtype=o.dtype, device=q.device)
    dk = torch.empty(k.shape, dtype=o.dtype, device=q.device)
    dv = torch.empty(v.shape, dtype=o.dtype, device=q.device)
    delta = torch.empty(N, H, dtype=torch.float32, device=q.device)
    sh = _attn_shape(q, v, scale, o.dtype)
    _check(lib().tpc_tree_attn_backward(plan.handle, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v),
                                        _attn_lo(q_lo, k_lo, v_lo, d_o_lo), _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq),
                                        _ptr(dk), _ptr(dv), _ptr(delta), _ptr(status), _stream_ptr(stream)))
    return dq, dk, dv


def tpc_rope_positions(plan: Plan, device="cuda", stream=None):
    import torch
    pos = torch.empty(plan.info["n_unique"], dtype=torch.int32, device=device)
    _check(lib().tpc_rope_positions(plan.handle, _ptr(pos), _stream_ptr(stream)))
    return pos


# ------------------------------------------------------------------------------------ compact MoE routing
def tpc_moe_route(plan: Plan, h, w_router, k, scratch=None, stream=None):
    """Routes every unique row once (include/tpc.h).  Returns dict(logits, lse, topk_idx, topk_gate,
    expert_load, prob_sum, scratch)."""
    import torch
    N, Dh = h.shape
    E = w_router.shape[0]
    dev = h.device
    n = int(lib().tpc_moe_scratch_bytes(plan.handle, E))
    scratch = scratch if scratch is not None else torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
    out = dict(logits=torch.empty(N, E, dtype=torch.float32, device=dev),
               lse=torch.empty(N, dtype=torch.float32, device=dev),
               topk_idx=torch.empty(N, k, dtype=torch.int32, device=dev),
               topk_gate=torch.empty(N, k, dtype=torch.float32, device=dev),
               expert_load=torch.empty(E, dtype=torch.int64, device=dev),
               prob_sum=torch.empty(E, dtype=torch.float32, device=dev), scratch=scratch)
    _check(lib().tpc_moe_route(plan.handle, _ptr(h), _ptr(w_router), Dh, E, k, _ptr(out["logits"]), _ptr(out["lse"]),
                               _ptr(out["topk_idx"]), _ptr(out["topk_gate"]), _ptr(out["expert_load"]),
                               _ptr(out["prob_sum"]), _ptr(scratch), scratch.numel(), _stream_ptr(stream)))
    return out


def tpc_moe_router_loss(plan: Plan, routed: dict, k, a=1.0, b=1.0, stream=None):
    """(losses fp32 [2] = (L_aux, L_z), dlogits fp32 [N, E]) of the routing result."""
    import torch
    N, E = routed["logits"].shape
    losses = torch.empty(2, dtype=torch.float32, device=routed["logits"].device)
    dz = torch.empty_like(routed["logits"])
    sc = routed["scratch"]
    _check(lib().tpc_moe_router_loss(plan.handle, _ptr(routed["logits"]), _ptr(routed["lse"]),
                                     _ptr(routed["expert_load"]), _ptr(routed["prob_sum"]), E, k, float(a), float(b),
                                     _ptr(losses), _ptr(dz), _ptr(sc), sc.numel(), _stream_ptr(stream)))
    return losses, dz


# ------------------------------------------------------------------------------------ hybrid layer group
GROUP_DIMS = {"D": 2048, "H": 16, "d_head": 128, "d_rope": 64, "d_latent": 512}


def group_shape(n_kda: int = 3, reuse_forward: bool = False) -> GroupShape:
    d = GROUP_DIMS
    return GroupShape(d["D"], d["H"], d["d_head"], d["d_rope"], d["d_latent"], n_kda, int(reuse_forward))


def group_weight_shapes(n_kda: int = 3):
    """{"kda": [(w_in, w_o) shapes] * n_kda, "mla": (w_a, w_b, w_o) shapes}, [out][in] row-major."""
    d = GROUP_DIMS
    D, H = d["D"], d["H"]
    kda = (4 * D + H, D), (D, D)
    mla = (H * (d["d_head"] + d["d_rope"]) + d["d_latent"] + d["d_rope"], D), (2 * D, d["d_latent"]), (D, D)
    return {"kda": [kda] * n_kda, "mla": mla}


def _group_ptrs(struct_cls, tensors):
    s = struct_cls()
    for i, pair in enumerate(tensors["kda"]):
        for j, t in enumerate(pair):
            s.kda[i][j] = t.data_ptr()
    for j, t in enumerate(tensors["mla"]):
        s.mla[j] = t.data_ptr()
    return s


def tpc_group_workspace_bytes(plan: Plan, n_kda: int = 3) -> int:
    sh = group_shape(n_kda)
    return int(lib().tpc_group_workspace_bytes(plan.handle, ctypes.byref(sh)))


def group_workspace(plan: Plan, n_kda: int = 3, device="cuda"):
    import torch
    return torch.empty(tpc_group_workspace_bytes(plan, n_kda), dtype=torch.uint8, device=device)


def tpc_group_forward(plan: Plan, weights, x, ws, h=None, y=None, stream=None):
    """Forward of the layer group on compact rows x (fp32 [N][2048]); returns (y, h)."""
    import torch
    n_kda = len(weights["kda"])
    N, D = x.shape
    h = h if h is not None else torch.empty(max(n_kda, 1), N, D, dtype=torch.float32, device=x.device)
    y = y if y is not None else torch.empty_like(x)
    sh = group_shape(n_kda)
    w = _group_ptrs(GroupWeights, weights)
    _check(lib().tpc_group_forward(plan.handle, ctypes.byref(sh), ctypes.byref(w), _ptr(x), _ptr(h), _ptr(y),
                                   _ptr(ws), ws.numel(), _stream_ptr(stream)))
    return y, h


def tpc_group_backward(plan: Plan, weights, x, h, dy, ws, dx=None, grads=None, stream=None, reuse_forward=False):
    """Backward (with recomputation) of sum <dy, y>; returns (dx, grads) with fp32 weight gradients.
    reuse_forward: ws still holds tpc_group_forward's result on the same inputs (the last layer is then
    not recomputed)."""
    import torch
    n_kda = len(weights["kda"])
    dx = dx if dx is not None else torch.empty_like(dy)
    if grads is None:
        grads = {"kda": [tuple(torch.empty(w.shape, dtype=torch.float32, device=x.device) for w in pair)
                         for pair in weights["kda"]],
                 "mla": tuple(torch.empty(w.shape, dtype=torch.float32, device=x.device) for w in weights["mla"])}
    sh = group_shape(n_kda, reuse_forward)
    w = _group_ptrs(GroupWeights, weights)
    g = _group_ptrs(GroupGrads, grads)
    _check(lib().tpc_group_backward(plan.handle, ctypes.byref(sh), ctypes.byref(w), _ptr(x), _ptr(h), _ptr(dy),
                                    _ptr(dx), ctypes.byref(g), _ptr(ws), ws.numel(), _stream_ptr(stream)))
    return dx, grads


def tpc_group_status(plan: Plan, ws, n_kda: int = 3, stream=None) -> int:
    sh = group_shape(n_kda)
    return int(lib().tpc_group_status(plan.handle, ctypes.byref(sh), _ptr(ws), _stream_ptr(stream)))
