"""Seeded synthetic inputs for the tree-packed chunkwise KDA path.

This module is shared by the fp64 oracle (``oracle/``) and by the GPU
harness.  It holds no arithmetic of the method itself: it only draws
rollout trees and tensors.

Random numbers come from Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
"Parallel random numbers: as easy as 1, 2, 3", SC'11), a counter-based
generator, so any element can be regenerated on its own: the host
(numpy, here) and the device (``synth/csrc/synth_gen.cu``) implement the
same definition and produce the same bits.  Each element of a tensor is
addressed by (seed, stream, flat index); its counter is
``(idx_lo, idx_hi, stream, 0)`` and its key ``(seed_lo, seed_hi ^ 0x5EED)``.
A standard normal is made from the four 32-bit outputs by Box-Muller with
53-bit uniforms, in fp64; rounding to the storage type is fp64 -> fp32
(round to nearest even), and for bf16 then fp32 -> bf16 (round to nearest
even).

Tensor layout is *node order*: the rows of node 0, then node 1, ... (node
ids are topological, parent < child).  Each side maps node order to its
own layout.

Value distributions (per token row and head), as the workload states:
q, v ~ N(0,1); k ~ N(0,1) then L2-normalised per (row, head) in fp64;
beta = sigmoid(N(0,1)); g = log(alpha) = -0.1 * softplus(N(0,1)) per
channel.  bf16 workloads round every input to bf16.
"""
from __future__ import annotations

import dataclasses
import numpy as np

# ---------------------------------------------------------------- Philox4x32-10
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint32(0x9E3779B9)
_W1 = np.uint32(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)

# stream ids (one per tensor kind); the CUDA twin uses the same numbers
STREAM = {
    "q": 1, "k": 2, "v": 3, "g": 4, "beta": 5, "d_o": 6, "d_final": 7,
    "d_o_exp": 8, "init": 9,
    "x": 10, "d_y": 11,
    "h": 30, "w_vocab": 31, "targets": 32, "d_logp": 33,
    "group_x": 50, "group_r": 51,
    # layer weights of the hybrid group: 100 + 16 * layer + matrix id
}


def group_weight_stream(layer: int, matrix: int) -> int:
    return 100 + 16 * layer + matrix


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds; all arguments uint32 arrays (broadcast)."""
    c0 = np.asarray(c0, np.uint32).astype(np.uint64)
    c1 = np.asarray(c1, np.uint32).astype(np.uint64)
    c2 = np.asarray(c2, np.uint32).astype(np.uint64)
    c3 = np.asarray(c3, np.uint32).astype(np.uint64)
    k0 = np.asarray(k0, np.uint32)
    k1 = np.asarray(k1, np.uint32)
    with np.errstate(over="ignore"):
        for _ in range(10):
            p0 = _M0 * c0
            p1 = _M1 * c2
            hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
            hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
            k0u = k0.astype(np.uint64)
            k1u = k1.astype(np.uint64)
            c0, c1, c2, c3 = hi1 ^ c1 ^ k0u, lo1, hi0 ^ c3 ^ k1u, lo0
            k0 = (k0 + _W0).astype(np.uint32)
            k1 = (k1 + _W1).astype(np.uint32)
    return (c0.astype(np.uint32), c1.astype(np.uint32),
            c2.astype(np.uint32), c3.astype(np.uint32))


def _key(seed: int):
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.uint32(seed & 0xFFFFFFFF), np.uint32(((seed >> 32) ^ 0x5EED) & 0xFFFFFFFF)


def raw_u32(seed: int, stream: int, idx) -> tuple:
    idx = np.asarray(idx, np.uint64)
    k0, k1 = _key(seed)
    lo = (idx & _MASK).astype(np.uint32)
    hi = (idx >> np.uint64(32)).astype(np.uint32)
    return philox4x32_10(lo, hi, np.uint32(stream), np.uint32(0), k0, k1)


def normal_f64(seed: int, stream: int, idx) -> np.ndarray:
    """One standard normal per flat index (Box-Muller, 53-bit uniforms)."""
    r0, r1, r2, r3 = raw_u32(seed, stream, idx)
    a = (r0 >> np.uint32(5)).astype(np.float64) * 67108864.0 + (r1 >> np.uint32(6)).astype(np.float64)
    b = (r2 >> np.uint32(5)).astype(np.float64) * 67108864.0 + (r3 >> np.uint32(6)).astype(np.float64)
    u1 = (a + 1.0) * (1.0 / 9007199254740992.0)  # (0, 1]
    u2 = b * (1.0 / 9007199254740992.0)          # [0, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(6.283185307179586 * u2)


def uniform_int(seed: int, stream: int, idx, n: int) -> np.ndarray:
    """Integers in [0, n) for n <= 2**16: the top bits of the first output."""
    assert 0 < n <= 65536
    r0, _, _, _ = raw_u32(seed, stream, idx)
    return ((r0.astype(np.uint64) * np.uint64(n)) >> np.uint64(32)).astype(np.int32)


# ---------------------------------------------------------------- rounding
def round_f32(x) -> np.ndarray:
    return np.asarray(x, np.float64).astype(np.float32)


def round_bf16(x) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE); returned as float32 holding bf16 values."""
    f = np.ascontiguousarray(np.asarray(x, np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    u = ((u + bias) & np.uint64(0xFFFF0000)).astype(np.uint32)
    return u.view(np.float32).reshape(f.shape)


def round_to(x, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return round_f32(x)
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(dtype)


# ---------------------------------------------------------------- trees
@dataclasses.dataclass
class Tree:
    parent: np.ndarray  # int32 [n], -1 for roots, parent < child
    length: np.ndarray  # int32 [n], >= 1

    @property
    def n(self) -> int:
        return int(self.parent.shape[0])

    def node_start(self) -> np.ndarray:
        """First node-order row of every node."""
        return np.concatenate([[0], np.cumsum(self.length, dtype=np.int64)[:-1]]).astype(np.int64)

    @property
    def n_rows(self) -> int:
        return int(np.sum(self.length, dtype=np.int64))

    def children(self):
        ch = [[] for _ in range(self.n)]
        for i, p in enumerate(self.parent):
            if p >= 0:
                ch[p].append(i)
        return ch

    def leaves(self) -> np.ndarray:
        has_child = np.zeros(self.n, bool)
        for p in self.parent:
            if p >= 0:
                has_child[p] = True
        return np.nonzero(~has_child)[0].astype(np.int32)

    def path(self, leaf: int):
        out = []
        v = int(leaf)
        while v >= 0:
            out.append(v)
            v = int(self.parent[v])
        return out[::-1]

    def trajectory_rows(self, leaf: int) -> np.ndarray:
        """Node-order row index of every position of the trajectory ending at ``leaf``."""
        st = self.node_start()
        return np.concatenate([np.arange(st[v], st[v] + self.length[v]) for v in self.path(leaf)]).astype(np.int64)

    def n_expanded(self) -> int:
        return int(sum(sum(int(self.length[v]) for v in self.path(l)) for l in self.leaves()))


def fig1_tree() -> Tree:
    """The five-segment tree of the HARTS overview figure (Figure 1(a)): A(40) -> B(24), C(17); B -> D(9), E(31)."""
    return Tree(np.array([-1, 0, 0, 1, 1], np.int32), np.array([40, 24, 17, 9, 31], np.int32))


def single_fork_tree(prefix=8192, branches=16, lo=512, hi=2048, seed=1) -> Tree:
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, size=branches)
    parent = np.array([-1] + [0] * branches, np.int32)
    length = np.array([prefix] + list(lens), np.int32)
    return Tree(parent, length)


def agentic_tree(seed=2, leaves=64, max_depth=5, mu=np.log(1500.0), sigma=0.8, lo=64, hi=16384) -> Tree:
    """Random multi-turn rollout tree: fork uniformly chosen shallow leaves into 2-4 branches
    until ``leaves`` leaves exist; retry with seed+1000 until the deepest fork level is ``max_depth``."""
    s = seed
    while True:
        rng = np.random.default_rng(s)
        parent = [-1]
        depth = [0]
        is_leaf = [True]
        n_leaves = 1
        ok = True
        while n_leaves < leaves:
            cand = [i for i in range(len(parent)) if is_leaf[i] and depth[i] < max_depth]
            if not cand:
                ok = False
                break
            v = cand[int(rng.integers(0, len(cand)))]
            b = int(rng.integers(2, 5))
            b = min(b, leaves + 1 - n_leaves)
            is_leaf[v] = False
            for _ in range(b):
                parent.append(v)
                depth.append(depth[v] + 1)
                is_leaf.append(True)
            n_leaves += b - 1
        if ok and max(depth) == max_depth:
            lens = np.clip(np.round(rng.lognormal(mu, sigma, size=len(parent))), lo, hi).astype(np.int32)
            return Tree(np.array(parent, np.int32), lens)
        s += 1000


def wide_tree(seed=4, prefix=32768, fan=(8, 8, 8), mu=np.log(800.0), sigma=1.0) -> Tree:
    rng = np.random.default_rng(seed)
    parent = [-1]
    level = [0]
    for f in fan:
        nxt = []
        for v in level:
            for _ in range(f):
                parent.append(v)
                nxt.append(len(parent) - 1)
        level = nxt
    n = len(parent)
    lens = np.maximum(1, np.round(rng.lognormal(mu, sigma, size=n - 1))).astype(np.int32)
    return Tree(np.array(parent, np.int32), np.concatenate([[prefix], lens]).astype(np.int32))


@dataclasses.dataclass
class Workload:
    name: str
    tree: Tree
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str  # "f32" | "bf16"
    seed: int


def workload(cfg: str) -> Workload:
    """Named synthetic workloads (tree + KDA shapes)."""
    if cfg == "fig1":
        return Workload("fig1 tree, H=2 d=32 C=16 fp32", fig1_tree(), 2, 32, 32, 16, "f32", 0)
    if cfg == "single_fork":
        return Workload("single-fork 8192 -> 16 x U[512,2048], H=16 d=128 C=64 bf16",
                        single_fork_tree(seed=1), 16, 128, 128, 64, "bf16", 1)
    if cfg == "agentic":
        return Workload("agentic 64-leaf 5-level tree, H=16 d=128 C=64 bf16", agentic_tree(seed=2), 16, 128, 128, 64, "bf16", 2)
    if cfg == "agentic_small":
        return Workload("agentic 8-leaf tree, lognormal(ln150,0.8)", agentic_tree(seed=3, leaves=8, max_depth=3,
                        mu=np.log(150.0), lo=16, hi=1024), 16, 128, 128, 64, "bf16", 3)
    if cfg == "wide":
        return Workload("wide 32768 -> 8 -> 8 -> 8 tree, H=32 d=128 C=64 bf16", wide_tree(seed=4), 32, 128, 128, 64, "bf16", 4)
    raise KeyError(cfg)


# ---------------------------------------------------------------- KDA inputs (node order)
def kda_inputs(seed: int, rows, H: int, dk: int, dv: int, dtype: str, heads=None):
    """q, k, v, g [len(rows), H, d] and beta [len(rows), H] for the given node-order rows.

    Values are returned as float64 arrays holding exactly the rounded
    (fp32 or bf16) values that the device generator writes.  ``heads``
    (a list of head indices of the H-head tensors) returns only those heads.
    """
    rows = np.asarray(rows, np.int64)
    n = rows.shape[0]
    hs = np.arange(H) if heads is None else np.asarray(heads, np.int64)

    def flat(width):
        return (rows[:, None, None] * H + hs[None, :, None]) * width + np.arange(width)[None, None, :]

    q = round_to(normal_f64(seed, STREAM["q"], flat(dk)), dtype)
    zk = normal_f64(seed, STREAM["k"], flat(dk))
    ss = np.zeros((n, len(hs)), np.float64)
    for c in range(dk):  # fixed summation order, mirrored on the device
        ss = ss + zk[:, :, c] * zk[:, :, c]
    k = round_to(zk / np.sqrt(ss)[:, :, None], dtype)
    v = round_to(normal_f64(seed, STREAM["v"], flat(dv)), dtype)
    zg = normal_f64(seed, STREAM["g"], flat(dk))
    g = round_to(-0.1 * np.log1p(np.exp(zg)), dtype)
    zb = normal_f64(seed, STREAM["beta"], rows[:, None] * H + hs[None, :])
    beta = round_to(1.0 / (1.0 + np.exp(-zb)), dtype)
    f = np.float64
    return q.astype(f), k.astype(f), v.astype(f), g.astype(f), beta.astype(f)


def normal_tensor(seed: int, stream: int, shape, dtype: str, scale: float = 1.0, first: int = 0) -> np.ndarray:
    """A tensor of independent scaled normals, flat-indexed from ``first``."""
    n = int(np.prod(shape))
    z = normal_f64(seed, stream, np.arange(first, first + n, dtype=np.int64))
    if scale != 1.0:
        z = z * scale
    return round_to(z, dtype).astype(np.float64).reshape(shape)


def rows_normal(seed: int, stream: int, rows, width: int, dtype: str, scale: float = 1.0) -> np.ndarray:
    """[len(rows), width] normals for the given row indices of a [*, width] tensor."""
    rows = np.asarray(rows, np.int64)
    idx = rows[:, None] * width + np.arange(width)[None, :]
    z = normal_f64(seed, stream, idx)
    if scale != 1.0:
        z = z * scale
    return round_to(z, dtype).astype(np.float64)


# ---------------------------------------------------------------- hybrid layer group inputs
def group_small_tree() -> Tree:
    """Six segments (150, 70, 95, 40, 66, 33 rows): every trajectory spans several 64-row chunks
    and no fork point is chunk-aligned, so replay, ragged chunks and ragged tiles all occur."""
    return Tree(parent=np.array([-1, 0, 0, 1, 1, 2], np.int32),
                length=np.array([150, 70, 95, 40, 66, 33], np.int32))


GROUP_DIMS = {"D": 2048, "H": 16, "d_head": 128, "d_rope": 64, "d_latent": 512}


def group_weight_shapes(n_kda: int, dims=None):
    d = dims or GROUP_DIMS
    D, H = d["D"], d["H"]
    kda = [((4 * D + H, D), (D, D))] * n_kda
    mla = ((H * (d["d_head"] + d["d_rope"]) + d["d_latent"] + d["d_rope"], D), (2 * D, d["d_latent"]), (D, D))
    return {"kda": kda, "mla": mla}


def group_inputs(seed: int, tree: Tree, n_kda: int = 3, dims=None, with_r: bool = True):
    """Layer-group inputs: x [N, D] fp32 normals (node order), weights N(0, 0.02) rounded to bf16
    ({"kda": [(w_in, w_o)] * n_kda, "mla": (w_a, w_b, w_o)}, [out][in]) and the upstream
    gradient R [n_expanded, D] fp32 normals per trajectory position (trajectories in leaf order)."""
    d = dims or GROUP_DIMS
    x = rows_normal(seed, STREAM["group_x"], np.arange(tree.n_rows), d["D"], "f32")
    shapes = group_weight_shapes(n_kda, d)
    kda = [tuple(normal_tensor(seed, group_weight_stream(l, m), shp, "bf16", 0.02) for m, shp in enumerate(pair))
           for l, pair in enumerate(shapes["kda"])]
    mla = tuple(normal_tensor(seed, group_weight_stream(15, m), shp, "bf16", 0.02)
                for m, shp in enumerate(shapes["mla"]))
    R = rows_normal(seed, STREAM["group_r"], np.arange(tree.n_expanded()), d["D"], "f32") if with_r else None
    return x, {"kda": kda, "mla": mla}, R
