"""Device twin of the synth generators (same Philox definition, same bits), for sizes the
host generator would take minutes on.  Tensors are written at the rows given by a map from
destination row to node-order row."""
from __future__ import annotations

import ctypes
import os
import subprocess

from . import STREAM

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libsynth.so")
SRC = os.path.join(HERE, "csrc", "synth_gen.cu")
_lib = None


def build(force=False):
    if force or not os.path.exists(LIB) or os.path.getmtime(SRC) > os.path.getmtime(LIB):
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-Xcompiler", "-fPIC", "-shared", "-o", LIB + ".tmp", SRC], check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} not built (synth.gpu.build())")
        L = ctypes.CDLL(LIB)
        V = ctypes.c_void_p
        L.synth_normal_rows.argtypes = [ctypes.c_uint64, ctypes.c_uint32, V, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_double, ctypes.c_int, V, V]
        L.synth_kda_inputs.argtypes = [ctypes.c_uint64, V, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, V, V, V, V, V, V]
        _lib = L
    return _lib


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def kda_inputs(seed, rows, H, dk, dv, dtype):
    """rows: int32 cuda tensor of node-order row ids (destination order). Returns q, k, v, g, beta."""
    import torch
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    n = rows.numel()
    q = torch.empty(n, H, dk, dtype=dt, device="cuda")
    k = torch.empty_like(q)
    g = torch.empty_like(q)
    v = torch.empty(n, H, dv, dtype=dt, device="cuda")
    b = torch.empty(n, H, dtype=dt, device="cuda")
    rc = lib().synth_kda_inputs(seed, rows.data_ptr(), n, H, dk, dv, 1 if dtype == "bf16" else 0, q.data_ptr(),
                                k.data_ptr(), v.data_ptr(), g.data_ptr(), b.data_ptr(), _stream())
    assert rc == 0, rc
    return q, k, v, g, b


def normal_rows(seed, stream, rows, width, dtype, scale=1.0, shape=None):
    """[len(rows), width] normals of a [*, width] tensor (rows None -> 0..n-1 given by shape)."""
    import torch
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    if rows is None:
        n = shape[0]
        ptr = None
    else:
        n = rows.numel()
        ptr = rows.data_ptr()
    out = torch.empty(n, width, dtype=dt, device="cuda")
    rc = lib().synth_normal_rows(seed, stream, ptr, n, width, float(scale), 1 if dtype == "bf16" else 0,
                                 out.data_ptr(), _stream())
    assert rc == 0, rc
    return out
