"""Ulysses sequence parallelism: forward and backward.

Page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠 FlashAttention
不够？那就加上序列并行", Ulysses subsection: the input is split along the sequence
across N devices, an all-to-all exchange gives every device the keys and values of the
whole sequence, every device computes attention for its own queries against all of
them, and a second all-to-all puts the output back in sequence order.  Page
"ms-swift长文本训练秘诀：Ulysses并行技术解析", section 1, adds that the model weights are
not split, only the input sequence.

Reading taken here (the pages give three different accounts of what is exchanged): the
standard head-parallel form.  Rank r starts with tokens [r*C, (r+1)*C) of q, k, v for
every head; the first all-to-all trades sequence chunks for head groups, so rank p holds
the whole sequence for query heads [p*Hq/N, (p+1)*Hq/N) and the key/value heads they
read; attention then runs unchanged on that head group; the second all-to-all trades
back.  Both Hq and Hkv must be divisible by N (no key/value head replication).  The
backward sends dO the same way as q and returns dq, dk, dv the same way as o.

Packed batches work the same way: the token stream [T][H][D] of all sequences is cut
into N equal slices, rank r holding tokens [r*T/N, (r+1)*T/N) whatever sequences they
belong to.  The exchange gives every rank the whole stream for its heads, so the
attention runs with the batch's global cu_seqlens, unchanged.

The all-to-alls are torch.distributed collectives (NCCL on GPUs); the layout changes
around them and the attention itself run in libattn.so.  Nothing reads another GPU's
memory directly.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional

import torch

from . import ops


@dataclass
class Hooks:
    """The compute and layout steps; the defaults are this library's kernels.  The CPU
    tests replace them (the fp64 oracle and a plain tensor transpose) to check the
    exchanges on gloo without a GPU."""
    fwd: Callable = None        # (q, k, v, causal, scale[, cu_seqlens]) -> (o, lse)
    bwd: Callable = None        # (q, k, v, o, lse, do, causal, scale[, cu_seqlens]) -> grads
    transpose: Callable = None  # (x, n_outer, n_inner) -> x as [n_inner][n_outer][block]

    def resolved(self) -> "Hooks":
        return Hooks(
            fwd=self.fwd or (lambda q, k, v, c, s, cu=None:
                             ops.attn_fwd(q, k, v, causal=c, scale=s, cu_seqlens=cu)),
            bwd=self.bwd or (lambda q, k, v, o, l, do, c, s, cu=None:
                             ops.attn_bwd(q, k, v, o, l, do, causal=c, scale=s, cu_seqlens=cu)),
            transpose=self.transpose or ops.transpose_blocks)


def check_dense(*ts) -> None:
    for t in ts:
        if t.dim() != 4:
            raise ValueError("dense Ulysses inputs are [B][C][H][D] chunks")


def check_packed(*ts) -> None:
    for t in ts:
        if t.dim() != 3:
            raise ValueError("packed Ulysses inputs are [Tc][H][D] slices of the token stream")


def _as_batch(x: torch.Tensor) -> torch.Tensor:
    """A packed slice [Tc][H][D] seen as a one-sequence dense batch [1][Tc][H][D]."""
    return x.view(1, *x.shape) if x.dim() == 3 else x


def _call(fn, args, cu):
    return fn(*args) if cu is None else fn(*args, cu)


def check_split(Hq: int, Hkv: int, N: int) -> None:
    if Hq % N or Hkv % N:
        raise ValueError(f"Ulysses needs Hq ({Hq}) and Hkv ({Hkv}) divisible by the number "
                         f"of ranks ({N})")


# Layout steps.  A send buffer is [N][B][C][h][D]: chunk p goes to rank p.  The buffer an
# all-to-all returns has the same shape, chunk p coming from rank p.
def seq_to_send(x: torch.Tensor, N: int, tr) -> torch.Tensor:
    """[B][C][H][D] (this rank's tokens, all heads) -> send buffer of head groups."""
    B, C, H, D = x.shape
    return tr(x, B * C, N).view(N, B, C, H // N, D)


def recv_to_full(r: torch.Tensor, tr) -> torch.Tensor:
    """Received sequence chunks [N][B][C][h][D] -> [B][N*C][h][D] (whole sequence)."""
    N, B, C, h, D = r.shape
    if B == 1:
        return r.view(1, N * C, h, D)
    return tr(r, N, B).view(B, N * C, h, D)


def full_to_send(y: torch.Tensor, N: int, tr) -> torch.Tensor:
    """[B][S][h][D] (whole sequence, this rank's heads) -> send buffer of sequence chunks."""
    B, S, h, D = y.shape
    C = S // N
    if B == 1:
        return y.view(N, 1, C, h, D)
    return tr(y, B, N).view(N, B, C, h, D)


def recv_to_seq(r: torch.Tensor, tr) -> torch.Tensor:
    """Received head groups [N][B][C][h][D] -> [B][C][N*h][D] (this rank's tokens)."""
    N, B, C, h, D = r.shape
    return tr(r, N, B * C).view(B, C, N * h, D)


def _all_to_all(x: torch.Tensor, group) -> torch.Tensor:
    import torch.distributed as dist
    out = torch.empty_like(x)
    dist.all_to_all_single(out, x.contiguous(), group=group)
    return out


class _UlyssesAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, group, hooks, cu_seqlens):
        import torch.distributed as dist
        N = dist.get_world_size(group)
        packed = cu_seqlens is not None
        (check_packed if packed else check_dense)(q, k, v)
        check_split(q.shape[-2], k.shape[-2], N)
        tr = hooks.transpose

        def to_heads(x):   # -> the whole sequence (stream) of this rank's heads
            f = recv_to_full(_all_to_all(seq_to_send(_as_batch(x), N, tr), group), tr)
            return f.view(f.shape[1:]) if packed else f

        def to_seq(y, shape):   # -> this rank's chunk (slice), all heads, in `shape`
            return recv_to_seq(_all_to_all(full_to_send(_as_batch(y), N, tr), group),
                               tr).view(shape)

        qf, kf, vf = to_heads(q), to_heads(k), to_heads(v)
        o_loc, lse_loc = _call(hooks.fwd, (qf, kf, vf, causal, scale), cu_seqlens)
        o = to_seq(o_loc, q.shape)
        ctx.save_for_backward(qf, kf, vf, o_loc, lse_loc)
        ctx.causal, ctx.scale, ctx.group, ctx.hooks, ctx.N = causal, scale, group, hooks, N
        ctx.cu, ctx.to_heads, ctx.to_seq = cu_seqlens, to_heads, to_seq
        ctx.shapes = (q.shape, k.shape, v.shape)
        return o

    @staticmethod
    def backward(ctx, do):
        qf, kf, vf, o_loc, lse_loc = ctx.saved_tensors
        dof = ctx.to_heads(do.contiguous())
        grads = _call(ctx.hooks.bwd, (qf, kf, vf, o_loc, lse_loc, dof, ctx.causal, ctx.scale),
                      ctx.cu)
        dq, dk, dv = (ctx.to_seq(g, t) for g, t in zip(grads, ctx.shapes))
        return dq, dk, dv, None, None, None, None, None


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
                      scale: Optional[float] = None, group=None,
                      hooks: Optional[Hooks] = None,
                      cu_seqlens: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Attention of this rank's sequence chunk over the whole sequence, autograd-aware.
    Dense: q [B][C][Hq][D], k/v [B][C][Hkv][D], the chunks of all ranks in rank order
    forming the sequence; returns o [B][C][Hq][D].  Packed (cu_seqlens given): q
    [Tc][Hq][D], k/v [Tc][Hkv][D] are this rank's slice of the token stream and
    cu_seqlens the whole batch's offsets (the same on every rank); returns o [Tc][Hq][D]."""
    import torch.distributed as dist
    if hooks is None and dist.get_world_size(group) == 1:
        return ops.attention(q, k, v, causal=causal, scale=scale, cu_seqlens=cu_seqlens)
    return _UlyssesAttention.apply(q, k, v, causal, scale, group, (hooks or Hooks()).resolved(),
                                   cu_seqlens)


def _emulated_all_to_all(sends: List[torch.Tensor]) -> List[torch.Tensor]:
    N = len(sends)
    return [torch.stack([sends[r][p] for r in range(N)]) for p in range(N)]


def ulysses_attention_single_device(q, k, v, world: int, causal: bool = True,
                                    scale: Optional[float] = None, do=None,
                                    hooks: Optional[Hooks] = None,
                                    cu_seqlens: Optional[torch.Tensor] = None):
    """Every rank of a `world`-rank Ulysses group, run one after another on this device
    from the full tensors (dense q [B][S][Hq][D], k/v [B][S][Hkv][D]; packed q [T][Hq][D],
    k/v [T][Hkv][D] with cu_seqlens): the same layout steps and per-head-group attention
    as ulysses_attention, with the all-to-alls done as plain copies.  Returns o, or
    (o, dq, dk, dv) when `do` is given."""
    packed = cu_seqlens is not None
    (check_packed if packed else check_dense)(q, k, v)
    hooks = (hooks or Hooks()).resolved()
    tr = hooks.transpose
    q4, k4, v4 = _as_batch(q), _as_batch(k), _as_batch(v)
    S = q4.shape[1]
    check_split(q4.shape[2], k4.shape[2], world)
    if S % world:
        raise ValueError("sequence length (packed: token count) must be divisible by the "
                         "number of ranks")
    C = S // world

    def chunks(t):
        return [t[:, r * C:(r + 1) * C].contiguous() for r in range(world)]

    def to_heads(t):
        sends = [seq_to_send(x, world, tr) for x in chunks(_as_batch(t))]
        full = [recv_to_full(r, tr) for r in _emulated_all_to_all(sends)]
        return [f.view(f.shape[1:]) for f in full] if packed else full

    def to_seq(ys, like):
        sends = [full_to_send(_as_batch(y), world, tr) for y in ys]
        out = torch.cat([recv_to_seq(r, tr) for r in _emulated_all_to_all(sends)], dim=1)
        return out.view(like.shape)

    qf, kf, vf = to_heads(q), to_heads(k), to_heads(v)
    outs = [_call(hooks.fwd, (qf[p], kf[p], vf[p], causal, scale), cu_seqlens)
            for p in range(world)]
    o = to_seq([x[0] for x in outs], q)
    if do is None:
        return o
    dof = to_heads(do)
    grads = [_call(hooks.bwd, (qf[p], kf[p], vf[p], outs[p][0], outs[p][1], dof[p], causal,
                               scale), cu_seqlens)
             for p in range(world)]
    return (o,) + tuple(to_seq([g[i] for g in grads], t) for i, t in enumerate((q, k, v)))
