"""Ring (context-parallel) attention forward.

Page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠 FlashAttention
不够？那就加上序列并行", subsection "Ring-Attention": the devices form a ring; at every
step each one hands a chunk of K/V to its neighbour and adds the partial attention of its
own queries over the chunk it holds, so that after N-1 hand-overs every device has
attended to the whole context.  Page "ms-swift支持GPU显存碎片整理提升利用率" (its
Ring-Attention passage) adds that each transfer has a fixed size and overlaps with the
computation.

Reading taken here (the pages leave the split open): the sequence of length S = N * C is
cut into N contiguous chunks and rank r holds tokens [r*C, (r+1)*C) of q, k and v for
every batch entry -- q [B][C][Hq][D], k/v [B][C][Hkv][D].  At step s rank r holds the
K/V chunk that started on rank (r - s) mod N.  With a causal mask, chunk j < r is wholly
visible to rank r's queries (no mask), the diagonal chunk j = r takes the causal mask,
and chunks j > r are skipped.  The partials are combined by the exact log-sum-exp merge
(attn_merge), so the result is the attention over the whole sequence.

K/V chunks travel with torch.distributed point-to-point sends (NCCL on GPUs) into local
buffers; the kernels only ever read this GPU's own memory.

Backward (ring_attn_bwd, and ring_attention for autograd): each block pair's share of the
gradient is the block-pair backward with the whole rows' O and LSE (attn_bwd given the
merged o and lse).  K/V chunks circulate as in the forward; the fp32 dK/dV accumulators of
the chunk a rank holds travel with it, each rank adding its share, and return to the
chunk's owner after N hops; dQ accumulates locally.  Shares are summed in fp32 and rounded
to bf16 once.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Tuple

import torch

from . import ops

Partial = Tuple[torch.Tensor, torch.Tensor]


def ring_schedule(rank: int, world: int, causal: bool) -> List[Tuple[int, int, bool]]:
    """The partials rank `rank` computes, in step order: (step, kv_chunk, causal_mask)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    out = []
    for s in range(world):
        j = (rank - s) % world
        if causal and j > rank:
            continue
        out.append((s, j, bool(causal and j == rank)))
    return out


def _check_dense(*ts) -> None:
    for t in ts:
        if t.dim() != 4:
            raise ValueError("the Ring wrappers take dense [B][C][H][D] chunks (packed batches "
                             "are not supported)")


def _default_attend(q, k, v, causal, scale) -> Partial:
    return ops.attn_fwd(q, k, v, causal=causal, scale=scale)


def ring_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
                  scale: Optional[float] = None, group=None,
                  attend: Optional[Callable[..., Partial]] = None,
                  merge: Optional[Callable[..., Partial]] = None) -> Partial:
    """Forward of this rank's query chunk over the whole ring.  Returns (o, lse) for the
    local queries: o like q, lse [B][Hq][C].

    attend(q, k, v, causal, scale) -> (o, lse) and merge(o_parts, lse_parts) -> (o, lse)
    default to this library's attn_fwd and attn_merge; they can be replaced (the CPU tests
    put the fp64 oracle there to check the schedule and the transfers).
    """
    import torch.distributed as dist

    _check_dense(q, k, v)
    attend = attend or _default_attend
    merge = merge or ops.attn_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    plan = {s: (j, c) for s, j, c in ring_schedule(rank, world, causal)}
    if world == 1:
        return attend(q, k, v, causal, scale)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    cur_k, cur_v = k, v
    o_parts, lse_parts = [], []
    for s in range(world):
        works = []
        if s < world - 1:
            nk, nv = bufs[s % 2]
            works = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, cur_k, nxt, group),
                dist.P2POp(dist.irecv, nk, prv, group),
                dist.P2POp(dist.isend, cur_v, nxt, group),
                dist.P2POp(dist.irecv, nv, prv, group),
            ])
        if s in plan:
            o, lse = attend(q, cur_k, cur_v, plan[s][1], scale)
            o_parts.append(o)
            lse_parts.append(lse)
        for w in works:
            w.wait()
        if s < world - 1:
            cur_k, cur_v = bufs[s % 2]
    if len(o_parts) == 1:
        return o_parts[0], lse_parts[0]
    return merge(o_parts, lse_parts)


def ring_attn_fwd_single_device(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int,
                                causal: bool = True, scale: Optional[float] = None,
                                attend: Optional[Callable[..., Partial]] = None,
                                merge: Optional[Callable[..., Partial]] = None) -> Partial:
    """Every rank's share of a `world`-rank ring, run one after another on this device from
    the full tensors (q [B][S][Hq][D], k/v [B][S][Hkv][D], S divisible by `world`): the same
    partials and merges as ring_attn_fwd, without the transfers.  Returns the full (o, lse)."""
    _check_dense(q, k, v)
    attend = attend or _default_attend
    merge = merge or ops.attn_merge
    B, S = q.shape[0], q.shape[1]
    if S % world:
        raise ValueError("sequence length must be divisible by the ring size")
    C = S // world

    def chunk(t, j):
        return t[:, j * C:(j + 1) * C].contiguous()

    outs, lses = [], []
    for r in range(world):
        qr = chunk(q, r)
        parts = [attend(qr, chunk(k, j), chunk(v, j), c, scale)
                 for _, j, c in ring_schedule(r, world, causal)]
        o, lse = parts[0] if len(parts) == 1 else merge([p[0] for p in parts],
                                                         [p[1] for p in parts])
        outs.append(o)
        lses.append(lse)
    return torch.cat(outs, dim=1), torch.cat(lses, dim=2)


@dataclass
class RingHooks:
    """Compute steps of the Ring forward/backward; the defaults are this library's kernels.
    The CPU tests replace them (the fp64 oracle and plain tensor arithmetic)."""
    fwd: Callable = None       # (q, k, v, causal, scale) -> (o, lse)
    merge: Callable = None     # (o_parts, lse_parts) -> (o, lse)
    bwd: Callable = None       # (q, k, v, o, lse, do, causal, scale) -> (dq, dk, dv), block pair
    acc: Callable = None       # (acc, x, init) -> acc = (0 if init else acc) + x
    cast: Callable = None      # (acc) -> result dtype
    acc_dtype: torch.dtype = torch.float32

    def resolved(self) -> "RingHooks":
        return RingHooks(
            fwd=self.fwd or _default_attend,
            merge=self.merge or ops.attn_merge,
            bwd=self.bwd or (lambda q, k, v, o, l, do, c, s:
                             ops.attn_bwd(q, k, v, o, l, do, causal=c, scale=s)),
            acc=self.acc or (lambda a, x, init: ops.accumulate_bf16(a, x, init)),
            cast=self.cast or ops.convert_f32_bf16,
            acc_dtype=self.acc_dtype)


def ring_attn_bwd(q, k, v, o, lse, do, causal: bool = True, scale: Optional[float] = None,
                  group=None, hooks: Optional[RingHooks] = None):
    """Backward of ring_attn_fwd for this rank's chunk: o, lse are the merged forward
    results of the local queries, do the gradient of o.  Returns (dq, dk, dv) of the local
    chunk."""
    import torch.distributed as dist

    _check_dense(q, k, v, o, do)
    h = (hooks or RingHooks()).resolved()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if world == 1:
        return h.bwd(q, k, v, o, lse, do, causal, scale)
    plan = {s: (j, c) for s, j, c in ring_schedule(rank, world, causal)}
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    new_acc = lambda t: torch.empty(t.shape, dtype=h.acc_dtype, device=t.device)
    kv_bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    acc_bufs = [(new_acc(k), new_acc(v)) for _ in range(2)]
    dq_acc = new_acc(q)
    cur_k, cur_v = k, v
    cur_dk, cur_dv = new_acc(k), new_acc(v)   # this rank's own chunk; initialised at step 0
    for s in range(world):
        kv_works = []
        if s < world - 1:
            nk, nv = kv_bufs[s % 2]
            kv_works = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, cur_k, nxt, group), dist.P2POp(dist.irecv, nk, prv, group),
                dist.P2POp(dist.isend, cur_v, nxt, group), dist.P2POp(dist.irecv, nv, prv, group)])
        if s in plan:   # step 0 is always the diagonal block: it initialises the accumulators
            gq, gk, gv = h.bwd(q, cur_k, cur_v, o, lse, do, plan[s][1], scale)
            h.acc(dq_acc, gq, s == 0)
            h.acc(cur_dk, gk, s == 0)
            h.acc(cur_dv, gv, s == 0)
        ndk, ndv = acc_bufs[s % 2]
        acc_works = dist.batch_isend_irecv([
            dist.P2POp(dist.isend, cur_dk, nxt, group), dist.P2POp(dist.irecv, ndk, prv, group),
            dist.P2POp(dist.isend, cur_dv, nxt, group), dist.P2POp(dist.irecv, ndv, prv, group)])
        for w in kv_works + acc_works:
            w.wait()
        if s < world - 1:
            cur_k, cur_v = kv_bufs[s % 2]
        cur_dk, cur_dv = ndk, ndv
    # After N hops every chunk's accumulators are back with its owner.
    return h.cast(dq_acc), h.cast(cur_dk), h.cast(cur_dv)


class _RingAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, group, hooks):
        o, lse = ring_attn_fwd(q, k, v, causal, scale, group, attend=hooks.fwd, merge=hooks.merge)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale, ctx.group, ctx.hooks = causal, scale, group, hooks
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = ring_attn_bwd(q, k, v, o, lse, do.contiguous(), ctx.causal, ctx.scale,
                                   ctx.group, ctx.hooks)
        return dq, dk, dv, None, None, None, None


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
                   scale: Optional[float] = None, group=None,
                   hooks: Optional[RingHooks] = None) -> torch.Tensor:
    """Autograd-aware Ring attention of this rank's chunk (layouts as ring_attn_fwd)."""
    return _RingAttention.apply(q, k, v, causal, scale, group, (hooks or RingHooks()).resolved())


def ring_attn_bwd_single_device(q, k, v, o, lse, do, world: int, causal: bool = True,
                                scale: Optional[float] = None,
                                hooks: Optional[RingHooks] = None):
    """Every rank's share of the Ring backward, run one after another on this device from
    the full tensors (q/o/do [B][S][Hq][D], k/v [B][S][Hkv][D], lse [B][Hq][S]): the same
    block-pair backwards and fp32 accumulation as ring_attn_bwd, without the transfers.
    Returns the full (dq, dk, dv)."""
    _check_dense(q, k, v, o, do)
    h = (hooks or RingHooks()).resolved()
    S = q.shape[1]
    if S % world:
        raise ValueError("sequence length must be divisible by the ring size")
    C = S // world

    def chunk(t, j):
        return t[:, j * C:(j + 1) * C].contiguous()

    new_acc = lambda t: torch.empty(t.shape, dtype=h.acc_dtype, device=t.device)
    dk_acc = [new_acc(chunk(k, j)) for j in range(world)]
    dv_acc = [new_acc(chunk(v, j)) for j in range(world)]
    kv_started = [False] * world          # has chunk j's accumulator received a share yet
    dq_out = []
    for r in range(world):
        qr, orr, dor = chunk(q, r), chunk(o, r), chunk(do, r)
        lr = lse[:, :, r * C:(r + 1) * C].contiguous()
        dq_acc = new_acc(qr)
        for s, j, c in ring_schedule(r, world, causal):
            gq, gk, gv = h.bwd(qr, chunk(k, j), chunk(v, j), orr, lr, dor, c, scale)
            h.acc(dq_acc, gq, s == 0)          # step 0 is every rank's first share
            h.acc(dk_acc[j], gk, not kv_started[j])
            h.acc(dv_acc[j], gv, not kv_started[j])
            kv_started[j] = True
        dq_out.append(h.cast(dq_acc))
    return (torch.cat(dq_out, dim=1), torch.cat([h.cast(a) for a in dk_acc], dim=1),
            torch.cat([h.cast(a) for a in dv_acc], dim=1))
