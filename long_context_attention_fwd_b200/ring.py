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
"""
from __future__ import annotations

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
