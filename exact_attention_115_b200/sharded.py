"""Attention with the B·H heads split over the ranks of a process group.

Every (batch, head) pair is an independent problem in the forward, the
backward and the decode: the FlashAttention V1/V2 study notes (51CTO),
section "Thread Block Level 并行", give each pair its own blocks of the
grid, and nothing is reduced across pairs.  So a rank computes the heads of
its shard with the single-GPU kernels, and data crosses ranks only when the
results are gathered: one all-gather per output tensor (NCCL over
NVLink/NVSwitch on GPUs), none on the data path.

Every rank passes the same full [B, H, N, d] inputs.  The flattened B·H
axis is cut into contiguous shards of ceil(B·H / world) heads (the last
ones may be shorter or empty), so the all-gathered buffers, truncated to
B·H heads, are the outputs in order.  Outputs come back whole on every rank.
A shard is handed to the kernels as a [1, heads, N, d] view, which needs q,
k, v (and dO) whose B and H axes merge into one (any contiguous tensor); a
shard of L that does not start on a 16-byte boundary is copied.
Dropout, key padding and bias are not accepted here: their per-head
indexing (the dropout counter, kv_len by batch element, a broadcast bias)
follows the unsharded (b, h) numbering.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import backward as _fa_backward
from . import forward as _fa_forward


def shard_range(n_heads: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [start, stop) of the flattened B·H axis computed by ``rank``."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of range for world size {world}")
    per = -(-n_heads // world)
    return min(rank * per, n_heads), min((rank + 1) * per, n_heads)


def _group_info(group):
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def _heads_view(t: torch.Tensor) -> torch.Tensor:
    """[B, H, N, d] -> [B·H, N, d] without a copy."""
    B, H, N, d = t.shape
    if t.stride(0) != H * t.stride(1) or t.stride(-1) != 1:
        raise ValueError("the B and H axes must merge into one (pass a contiguous tensor)")
    return t.view(B * H, N, d) if t.is_contiguous() else t.as_strided(
        (B * H, N, d), (t.stride(1), t.stride(2), 1), t.storage_offset())


def _shard(t: torch.Tensor, start: int, stop: int) -> torch.Tensor:
    """Heads [start, stop) of t as a [1, stop − start, N, d] view."""
    return _heads_view(t)[start:stop].unsqueeze(0)


def _all_gather_heads(local: torch.Tensor, per: int, n_heads: int, group) -> torch.Tensor:
    """Concatenate every rank's [count, ...] block (zero-padded to ``per``
    rows) along dim 0 and keep the first ``n_heads`` rows.  NCCL gathers
    device tensors in place; another backend (gloo) goes through host
    memory."""
    world, _ = _group_info(group)
    if local.shape[0] < per:
        pad = local.new_zeros((per - local.shape[0], *local.shape[1:]))
        local = torch.cat([local, pad], 0)
    local = local.contiguous()
    if world == 1:
        return local[:n_heads]
    on_device = local.is_cuda and dist.get_backend(group) == "nccl"
    src = local if on_device else local.cpu()
    out = src.new_empty((world * per, *local.shape[1:]))
    dist.all_gather_into_tensor(out, src, group=group)
    if not on_device:
        out = out.to(local.device)
    return out[:n_heads]


def _check_inputs(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    if k.shape[:2] != q.shape[:2] or v.shape != k.shape:
        raise ValueError("q, k, v must share B and H, and k and v their shape")


def forward(q, k, v, causal: bool = False, scale: float | None = None, group=None):
    """O, L = attention(q, k, v) over the group: this rank runs the forward
    kernel on its heads, then O [B, H, Nq, d] and L [B, H, Nq] are
    all-gathered.  Same arguments as the single-GPU forward() otherwise."""
    _check_inputs(q, k, v)
    B, H, Nq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    world, rank = _group_info(group)
    BH = B * H
    per = -(-BH // world)
    s, e = shard_range(BH, world, rank)
    if e > s:
        O, L = _fa_forward(_shard(q, s, e), _shard(k, s, e), _shard(v, s, e), causal=causal,
                           scale=scale)
        O, L = O[0], L[0]
    else:
        O = q.new_empty((0, Nq, d))
        L = torch.empty((0, Nq), dtype=torch.float32, device=q.device)
    O = _all_gather_heads(O, per, BH, group).view(B, H, Nq, d)
    L = _all_gather_heads(L, per, BH, group).view(B, H, Nq)
    return O, L


def backward(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, group=None):
    """dQ, dK, dV over the group: this rank runs the backward kernels on its
    heads (from the full q, k, v, O, dO, L every rank holds), then the three
    gradients are all-gathered."""
    _check_inputs(q, k, v)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    world, rank = _group_info(group)
    BH = B * H
    per = -(-BH // world)
    s, e = shard_range(BH, world, rank)
    if e > s:
        L = lse.reshape(BH, Nq)[s:e].unsqueeze(0)
        if L.data_ptr() % 16:  # the kernels take 16-byte aligned pointers only
            L = L.clone()
        dq, dk, dv = _fa_backward(_shard(q, s, e), _shard(k, s, e), _shard(v, s, e),
                                  _shard(o, s, e), _shard(do, s, e), L, causal=causal,
                                  scale=scale)
        dq, dk, dv = dq[0], dk[0], dv[0]
    else:
        dq = q.new_empty((0, Nq, d))
        dk = q.new_empty((0, Nk, d))
        dv = q.new_empty((0, Nk, d))
    dq = _all_gather_heads(dq, per, BH, group).view(B, H, Nq, d)
    dk = _all_gather_heads(dk, per, BH, group).view(B, H, Nk, d)
    dv = _all_gather_heads(dv, per, BH, group).view(B, H, Nk, d)
    return dq, dk, dv


class _ShardedAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, group):
        O, L = forward(q, k, v, causal=causal, scale=scale, group=group)
        ctx.save_for_backward(q, k, v, O, L)
        ctx.args = (causal, scale, group)
        return O

    @staticmethod
    def backward(ctx, dO):
        q, k, v, O, L = ctx.saved_tensors
        causal, scale, group = ctx.args
        dq, dk, dv = backward(q, k, v, O, dO.contiguous(), L, causal=causal, scale=scale,
                              group=group)
        return dq, dk, dv, None, None, None


def attention(q, k, v, causal: bool = False, scale: float | None = None, group=None):
    """Differentiable O = attention(q, k, v) with the heads split over
    ``group`` (every rank passes the same inputs and the same upstream
    gradient, and gets the whole O and the whole gradients)."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    return _ShardedAttention.apply(q, k, v, bool(causal), float(scale), group)
