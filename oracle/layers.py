"""Hybrid layer group (KDA layers followed by one latent-attention layer) in fp64 -- oracle side.

HARTS Table 1 gives the models' attention layout as KDA and MLA layers in a 3:1 group and
Figure C.1 runs every layer type once per unique row of the tree; neither page gives the layer
formulas, so the plainest pre-norm residual layers are fixed here:

KDA layer (y = x + KDA(q, k, v, g, beta) W_o^T):
    xn = x / sqrt(mean(x^2) + eps)                       (RMSNorm, unit weight, eps 1e-6)
    [q | k | v | g | beta] = xn W_in^T                    (blocks of D = H d_head, then H)
    k <- k / sqrt(|k|^2 + eps) per head;  g <- -0.1 softplus(g);  beta <- sigmoid(beta)
MLA layer (y = x + o W_o^T):
    [q | c | kr] = xn W_a^T      q: H heads of (d_head no-position + d_rope rotary) dims,
                                 c: the d_latent latent, kr: the rotary key shared by all heads
    [k_nope | v] = c W_b^T
    q_rot, kr rotated by the half-split rotary map at the row's trajectory depth (base 10000)
    o = tree-masked softmax attention of q = [q_nope | q_rot], k = [k_nope | kr], v, with scale
        1/sqrt(d_head + d_rope)  (oracle.attention: causal along every trajectory)

Precision: the device keeps activations and gradients in fp32 and forms its tensor-core products
from bf16 hi/lo pairs (x = hi + lo to 2^-17 relative), so no activation is rounded to bf16 there;
the oracle is the exact fp64 function of the bf16-valued weights.

The backward is reverse-mode differentiation of this forward (torch autograd over fp64 CPU
tensors), except for KDA and attention, whose adjoints are the hand-written ones of
oracle.kda and oracle.attention.  Recomputation is a schedule, not arithmetic: the oracle keeps
everything.  TEST INFRASTRUCTURE ONLY.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import attention as oatt
from . import kda as okda


@dataclass(frozen=True)
class Dims:
    D: int = 2048
    H: int = 16
    d_head: int = 128
    d_rope: int = 64
    d_latent: int = 512
    eps: float = 1e-6
    base: float = 10000.0

    @property
    def kda_proj(self) -> int:
        return 4 * self.D + self.H

    @property
    def mla_proj(self) -> int:
        return self.H * (self.d_head + self.d_rope) + self.d_latent + self.d_rope


class _Kda(torch.autograd.Function):
    """KDA over the tree (oracle.kda token-by-token recurrence along every trajectory)."""

    @staticmethod
    def forward(ctx, q, k, v, g, beta, tree):
        ctx.tree = tree
        ctx.save_for_backward(q, k, v, g, beta)
        inputs = tuple(t.detach().numpy() for t in (q, k, v, g, beta))
        o, _ = okda.tree_forward(tree, inputs)
        return torch.from_numpy(o)

    @staticmethod
    def backward(ctx, do):
        q, k, v, g, beta = ctx.saved_tensors
        inputs = tuple(t.detach().numpy() for t in (q, k, v, g, beta))
        grads = okda.tree_backward(ctx.tree, inputs, do.detach().numpy())
        return tuple(torch.from_numpy(x) for x in grads[:5]) + (None,)


class _Attn(torch.autograd.Function):
    """Tree-masked softmax attention (oracle.attention: causal along every trajectory)."""

    @staticmethod
    def forward(ctx, q, k, v, tree, scale):
        ctx.tree, ctx.scale = tree, scale
        ctx.save_for_backward(q, k, v)
        o, _ = oatt.tree_forward(tree, q.detach().numpy(), k.detach().numpy(), v.detach().numpy(), scale)
        return torch.from_numpy(o)

    @staticmethod
    def backward(ctx, do):
        q, k, v = ctx.saved_tensors
        qn, kn, vn = (t.detach().numpy() for t in (q, k, v))
        dq, dk, dv = oatt.tree_backward(ctx.tree, qn, kn, vn, ctx.scale, do.detach().numpy())
        return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv), None, None


def rmsnorm(x: torch.Tensor, eps: float) -> torch.Tensor:
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + eps)


def rope(x: torch.Tensor, pos: torch.Tensor, base: float) -> torch.Tensor:
    """Half-split rotary map of the last axis (width 2m): pair (i, i + m) is rotated by the angle
    pos * base^(-2i / 2m).  x: [N, ..., 2m], pos: [N]."""
    m = x.shape[-1] // 2
    inv = base ** (-2.0 * torch.arange(m, dtype=torch.float64) / (2 * m))
    ang = pos.to(torch.float64)[:, None] * inv[None, :]
    shape = (x.shape[0],) + (1,) * (x.dim() - 2) + (m,)
    c, s = torch.cos(ang).reshape(shape), torch.sin(ang).reshape(shape)
    x1, x2 = x[..., :m], x[..., m:]
    return torch.cat([x1 * c - x2 * s, x1 * s + x2 * c], dim=-1)


def kda_layer(tree, x, w_in, w_o, dims: Dims, parts: dict | None = None):
    N, D, H, dh = x.shape[0], dims.D, dims.H, dims.d_head
    xn = rmsnorm(x, dims.eps)
    P = xn @ w_in.T
    q = P[:, :D].reshape(N, H, dh)
    kt = P[:, D:2 * D].reshape(N, H, dh)
    k = kt / torch.sqrt((kt * kt).sum(dim=-1, keepdim=True) + dims.eps)
    v = P[:, 2 * D:3 * D].reshape(N, H, dh)
    g = -0.1 * torch.nn.functional.softplus(P[:, 3 * D:4 * D]).reshape(N, H, dh)
    beta = torch.sigmoid(P[:, 4 * D:4 * D + H])
    o = _Kda.apply(q, k, v, g, beta, tree).reshape(N, D)
    if parts is not None:
        parts.update(xn=xn, q=q, k=k, v=v, g=g, beta=beta, o=o)
    return x + o @ w_o.T


def mla_layer(tree, pos, x, w_a, w_b, w_o, dims: Dims, parts: dict | None = None):
    N, D, H, dh, dr, dl = x.shape[0], dims.D, dims.H, dims.d_head, dims.d_rope, dims.d_latent
    xn = rmsnorm(x, dims.eps)
    P = xn @ w_a.T
    qh = P[:, :H * (dh + dr)].reshape(N, H, dh + dr)
    c = P[:, H * (dh + dr):H * (dh + dr) + dl]
    kr = rope(P[:, H * (dh + dr) + dl:], pos, dims.base)
    q = torch.cat([qh[..., :dh], rope(qh[..., dh:], pos, dims.base)], dim=-1)
    KV = c @ w_b.T
    k = torch.cat([KV[:, :D].reshape(N, H, dh), kr[:, None, :].expand(N, H, dr)], dim=-1)
    v = KV[:, D:].reshape(N, H, dh)
    o = _Attn.apply(q, k, v, tree, 1.0 / np.sqrt(dh + dr)).reshape(N, D)
    if parts is not None:
        parts.update(xn=xn, q=q, k=k, v=v, c=c, kr=kr, o=o)
    return x + o @ w_o.T


def depth_positions(tree) -> np.ndarray:
    """Trajectory position of every node-order row (its depth from the root)."""
    pos = np.zeros(tree.n_rows, np.int64)
    st = tree.node_start()
    for v in range(tree.n):
        above = sum(int(tree.length[u]) for u in tree.path(v)[:-1])
        pos[st[v]:st[v] + tree.length[v]] = above + np.arange(tree.length[v])
    return pos


def group_forward(tree, x, weights, dims: Dims = Dims()):
    """y and every layer output for node-order rows x [N, D] (fp64 numpy).

    weights: {"kda": [(w_in, w_o), ...], "mla": (w_a, w_b, w_o)} as float64 arrays.
    Returns (y, [outputs of the KDA layers]).
    """
    with torch.no_grad():
        pos = torch.from_numpy(depth_positions(tree))
        h = torch.from_numpy(np.asarray(x, np.float64))
        outs = []
        for w_in, w_o in weights["kda"]:
            h = kda_layer(tree, h, torch.from_numpy(w_in), torch.from_numpy(w_o), dims)
            outs.append(h.numpy())
        w_a, w_b, w_o = (torch.from_numpy(w) for w in weights["mla"])
        y = mla_layer(tree, pos, h, w_a, w_b, w_o, dims)
    return y.numpy(), outs


def group_backward(tree, x, weights, dy, dims: Dims = Dims()):
    """Gradients of sum <dy, y> (dy per node-order row, occurrence-summed) w.r.t. x and every
    weight: returns (y, dx, {"kda": [(dw_in, dw_o), ...], "mla": (dw_a, dw_b, dw_o)}, [outputs of
    the KDA layers])."""
    pos = torch.from_numpy(depth_positions(tree))
    xt = torch.tensor(np.asarray(x, np.float64), requires_grad=True)
    kw = [tuple(torch.tensor(w, requires_grad=True) for w in pair) for pair in weights["kda"]]
    mw = tuple(torch.tensor(w, requires_grad=True) for w in weights["mla"])
    h = xt
    outs = []
    for w_in, w_o in kw:
        h = kda_layer(tree, h, w_in, w_o, dims)
        outs.append(h.detach().numpy())
    y = mla_layer(tree, pos, h, *mw, dims)
    loss = (y * torch.from_numpy(np.asarray(dy, np.float64))).sum()
    flat = [xt] + [w for pair in kw for w in pair] + list(mw)
    grads = torch.autograd.grad(loss, flat)
    dk = [(grads[1 + 2 * i].numpy(), grads[2 + 2 * i].numpy()) for i in range(len(kw))]
    dm = tuple(g.numpy() for g in grads[1 + 2 * len(kw):])
    return y.detach().numpy(), grads[0].numpy(), {"kda": dk, "mla": dm}, outs


def occurrence_sum(tree, r_expanded) -> np.ndarray:
    """Upstream gradient per node-order row of the loss sum_j <y_{row(j)}, R_j> over expanded
    positions j (trajectories in leaf order): the sum of R over the row's occurrences."""
    out = np.zeros((tree.n_rows,) + r_expanded.shape[1:])
    j = 0
    for leaf in tree.leaves():
        rows = tree.trajectory_rows(leaf)
        np.add.at(out, rows, r_expanded[j:j + len(rows)])
        j += len(rows)
    return out
