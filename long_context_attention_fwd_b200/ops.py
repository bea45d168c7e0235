"""PyTorch-facing wrappers over the C ABI (torch supplies device memory and streams).

    o, lse = attn_fwd(q, k, v, causal=True)                   # q [B,S,Hq,D], k/v [B,S,Hkv,D]
    o, lse = attn_fwd(q, k, v, cu_seqlens=cu)                  # packed: q [T,Hq,D], cu int32 [n+1]
    dq, dk, dv = attn_bwd(q, k, v, o, lse, do, causal=True)
    o = attention(q, k, v, causal=True)                        # autograd-aware
    o, lse = attn_merge([o1, o2], [lse1, lse2])                # exact merge of key-chunk partials
    o, lse = attn_decode(q, k_cache, v_cache, cache_len)       # one new token per sequence
    o, lse = attn_fwd_fp8(q8, k8, v8, qd, kd, vd)              # e4m3 inputs + descale factors

All arithmetic runs in libattn.so; these functions only check shapes, allocate
outputs with torch and pass raw pointers and the current CUDA stream.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import torch

from . import capi

MERGE_MAX_PARTS = 16  # ATTN_MERGE_MAX_PARTS of the C ABI


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _dims(q: torch.Tensor, k: torch.Tensor, cu_seqlens: Optional[torch.Tensor],
          v: Optional[torch.Tensor] = None):
    _same_device(q.device, k, v, cu_seqlens)
    if v is not None and v.shape != k.shape:
        raise ValueError("v must have k's shape")
    if cu_seqlens is None:
        if q.dim() != 4 or k.dim() != 4:
            raise ValueError("dense inputs must be [B, S, H, D]")
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
        if k.shape[0] != B or k.shape[1] != S or k.shape[3] != D:
            raise ValueError("k/v shape does not match q")
    else:
        if q.dim() != 3 or k.dim() != 3:
            raise ValueError("packed inputs must be [T, H, D]")
        S, Hq, D = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda \
                or not cu_seqlens.is_contiguous() or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a contiguous 1-D int32 CUDA tensor")
        if k.shape[0] != S or k.shape[2] != D:
            raise ValueError("k/v shape does not match q")
    return B, S, Hq, Hkv, D


def _same_device(device, *ts) -> None:
    for t in ts:
        if t is not None and t.device != device:
            raise ValueError(f"all tensors must be on {device} (one is on {t.device})")


def _check_tensor(t: Optional[torch.Tensor], name: str, shape, dtype, device) -> None:
    """A caller-supplied output, or an input whose size the kernel takes from another
    tensor, must be exactly what the kernel writes or reads: a smaller one would send
    the kernel past its end."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != device \
            or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape "
                         f"{tuple(shape)} on {device}")


def _workspace_bytes(ws: torch.Tensor, device) -> int:
    if not ws.is_cuda or ws.device != device or not ws.is_contiguous():
        raise ValueError(f"workspace must be a contiguous tensor on {device}")
    return ws.numel() * ws.element_size()


def _lse_shape(B: int, S: int, Hq: int, packed: bool):
    return (Hq, S) if packed else (B, Hq, S)


def _check_inputs(*ts: torch.Tensor) -> None:
    for t in ts:
        if not t.is_cuda:
            raise ValueError("libattn needs CUDA tensors (there is no CPU path)")
        if t.dtype != torch.bfloat16:
            raise ValueError("tensors must be bfloat16")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
             scale: Optional[float] = None, cu_seqlens: Optional[torch.Tensor] = None,
             out: Optional[torch.Tensor] = None,
             lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Fused forward: returns (o, lse); lse is fp32 [B,Hq,S] (dense) or [Hq,T] (packed)."""
    _check_inputs(q, k, v)
    B, S, Hq, Hkv, D = _dims(q, k, cu_seqlens, v)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    shape = _lse_shape(B, S, Hq, cu_seqlens is not None)
    _check_tensor(out, "out", q.shape, torch.bfloat16, q.device)
    _check_tensor(lse, "lse", shape, torch.float32, q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(shape, dtype=torch.float32, device=q.device)
    st = capi.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                       B, Hq, Hkv, S, D, causal, scale,
                       cu_seqlens.data_ptr() if cu_seqlens is not None else None,
                       _stream(q.device))
    capi.check(st, "attn_fwd")
    return out, lse


def attn_bwd_workspace_size(q: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None) -> int:
    if cu_seqlens is None:
        B, S, Hq, D = q.shape
        return capi.attn_bwd_workspace_size(B, Hq, S, D, None)
    S, Hq, D = q.shape
    return capi.attn_bwd_workspace_size(cu_seqlens.numel() - 1, Hq, S, D, 1)


def attn_bwd(q, k, v, o, lse, dout, causal: bool = True, scale: Optional[float] = None,
             cu_seqlens: Optional[torch.Tensor] = None, dq=None, dk=None, dv=None,
             workspace: Optional[torch.Tensor] = None):
    """Fused backward: returns (dq, dk, dv)."""
    _check_inputs(q, k, v, o, dout)
    B, S, Hq, Hkv, D = _dims(q, k, cu_seqlens, v)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dev = q.device
    _check_tensor(o, "o", q.shape, torch.bfloat16, dev)
    _check_tensor(dout, "dout", q.shape, torch.bfloat16, dev)
    _check_tensor(lse, "lse", _lse_shape(B, S, Hq, cu_seqlens is not None), torch.float32, dev)
    _check_tensor(dq, "dq", q.shape, torch.bfloat16, dev)
    _check_tensor(dk, "dk", k.shape, torch.bfloat16, dev)
    _check_tensor(dv, "dv", v.shape, torch.bfloat16, dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = attn_bwd_workspace_size(q, cu_seqlens)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = _workspace_bytes(workspace, dev)
    st = capi.attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                       B, Hq, Hkv, S, D, causal, scale,
                       cu_seqlens.data_ptr() if cu_seqlens is not None else None,
                       workspace.data_ptr(), ws_bytes, _stream(q.device))
    capi.check(st, "attn_bwd")
    return dq, dk, dv


class _FusedAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, cu_seqlens):
        o, lse = attn_fwd(q, k, v, causal=causal, scale=scale, cu_seqlens=cu_seqlens)
        ctx.save_for_backward(q, k, v, o, lse, cu_seqlens)
        ctx.causal, ctx.scale = causal, scale
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, cu = ctx.saved_tensors
        dq, dk, dv = attn_bwd(q, k, v, o, lse, do.contiguous(), causal=ctx.causal,
                              scale=ctx.scale, cu_seqlens=cu)
        return dq, dk, dv, None, None, None


def attention(q, k, v, causal: bool = True, scale: Optional[float] = None,
              cu_seqlens: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Autograd-aware fused attention (forward and backward both in libattn.so)."""
    return _FusedAttention.apply(q, k, v, causal, scale, cu_seqlens)


def attn_merge(o_parts: Sequence[torch.Tensor], lse_parts: Sequence[torch.Tensor],
               out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact merge of partial attention results over disjoint key sets (Ring attention).

    o_parts: bf16 [B,S,H,D] (or packed [T,H,D]); lse_parts: fp32 [B,H,S] (or [H,T]) -- the
    outputs of attn_fwd for each key chunk.  Returns (o, lse) over the union of the chunks.
    `out`/`lse` may be o_parts[0]/lse_parts[0] for an in-place merge.  More than
    ATTN_MERGE_MAX_PARTS partials are merged in groups, then the groups are merged.
    """
    if len(o_parts) == 0 or len(o_parts) != len(lse_parts):
        raise ValueError("need the same positive number of o and lse partials")
    _check_inputs(*o_parts)
    o0, l0 = o_parts[0], lse_parts[0]
    if o0.dim() == 4:
        B, S, H, D = o0.shape
        lse_shape = (B, H, S)
    elif o0.dim() == 3:
        S, H, D = o0.shape
        B = 1
        lse_shape = (H, S)
    else:
        raise ValueError("o partials must be [B,S,H,D] or [T,H,D]")
    for o_p, l_p in zip(o_parts, lse_parts):
        if o_p.shape != o0.shape or o_p.device != o0.device:
            raise ValueError("o partials differ in shape or device")
        if tuple(l_p.shape) != lse_shape or l_p.dtype != torch.float32 or not l_p.is_contiguous() \
                or l_p.device != o0.device:
            raise ValueError(f"lse partials must be contiguous fp32 {lse_shape} on {o0.device}")
    if len(o_parts) > MERGE_MAX_PARTS:
        groups = [attn_merge(o_parts[i:i + MERGE_MAX_PARTS], lse_parts[i:i + MERGE_MAX_PARTS])
                  for i in range(0, len(o_parts), MERGE_MAX_PARTS)]
        return attn_merge([g[0] for g in groups], [g[1] for g in groups], out, lse)
    _check_tensor(out, "out", o0.shape, torch.bfloat16, o0.device)
    _check_tensor(lse, "lse", lse_shape, torch.float32, o0.device)
    out = torch.empty_like(o0) if out is None else out
    lse = torch.empty_like(l0) if lse is None else lse
    st = capi.attn_merge([t.data_ptr() for t in o_parts], [t.data_ptr() for t in lse_parts],
                         out.data_ptr(), lse.data_ptr(), B, H, S, D, _stream(o0.device))
    capi.check(st, "attn_merge")
    return out, lse


def transpose_blocks(x: torch.Tensor, n_outer: int, n_inner: int,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x seen as [n_outer][n_inner][block] -> [n_inner][n_outer][block] (a copy in
    libattn.so; the block is x.numel() / (n_outer * n_inner) elements).  Returns a tensor
    of x's dtype and shape [n_inner, n_outer, block] unless `out` is given."""
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("transpose_blocks needs a contiguous CUDA tensor (there is no CPU path)")
    n = x.numel()
    if n_outer < 1 or n_inner < 1 or n % (n_outer * n_inner):
        raise ValueError("x does not split into n_outer * n_inner equal blocks")
    blk = n // (n_outer * n_inner)
    if out is None:
        out = torch.empty((n_inner, n_outer, blk), dtype=x.dtype, device=x.device)
    elif out.numel() != n or not out.is_contiguous() or out.dtype != x.dtype \
            or out.device != x.device:
        raise ValueError("out must be contiguous, of x's dtype and size, on x's device")
    st = capi.attn_transpose_blocks(x.data_ptr(), out.data_ptr(), n_outer, n_inner,
                                    blk * x.element_size(), _stream(x.device))
    capi.check(st, "attn_transpose_blocks")
    return out


def attn_decode_workspace_size(q: torch.Tensor, k_cache: torch.Tensor) -> int:
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    return capi.attn_decode_workspace_size(B, Hq, Hkv, Lmax, D)


def attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                cache_len: torch.Tensor, scale: Optional[float] = None,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Decode attention: q [B,Hq,D] against k/v cache [B,Lmax,Hkv,D] with cache_len int32
    [B] (on the GPU).  Returns (o [B,Hq,D] bf16, lse [B,Hq] fp32)."""
    _check_inputs(q, k_cache, v_cache)
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q must be [B,Hq,D] and the caches [B,Lmax,Hkv,D]")
    B, Hq, D = q.shape
    Bk, Lmax, Hkv, Dk = k_cache.shape
    if Bk != B or Dk != D:
        raise ValueError("cache shape does not match q")
    if cache_len.dtype != torch.int32 or not cache_len.is_cuda or cache_len.numel() != B \
            or not cache_len.is_contiguous():
        raise ValueError("cache_len must be a contiguous int32 CUDA tensor of B entries")
    _same_device(q.device, k_cache, v_cache, cache_len)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _check_tensor(out, "out", q.shape, torch.bfloat16, q.device)
    _check_tensor(lse, "lse", (B, Hq), torch.float32, q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    need = capi.attn_decode_workspace_size(B, Hq, Hkv, Lmax, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace_bytes(workspace, q.device)
    st = capi.attn_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                          cache_len.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lmax,
                          D, scale, workspace.data_ptr(), ws_bytes, _stream(q.device))
    capi.check(st, "attn_decode")
    return out, lse


def _check_e4m3(*ts: torch.Tensor) -> None:
    for t in ts:
        if not t.is_cuda:
            raise ValueError("libattn needs CUDA tensors (there is no CPU path)")
        if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
            raise ValueError("fp8 tensors must be float8_e4m3fn (or their bytes as uint8)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def attn_fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_descale: float,
                 k_descale: float, v_descale: float, causal: bool = True,
                 scale: Optional[float] = None, cu_seqlens: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """e4m3 forward: attention of (q_descale q, k_descale k, v_descale v), D = 128.
    Returns (o bf16, lse fp32) in attn_fwd's layouts."""
    _check_e4m3(q, k, v)
    B, S, Hq, Hkv, D = _dims(q, k, cu_seqlens, v)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    shape = _lse_shape(B, S, Hq, cu_seqlens is not None)
    _check_tensor(out, "out", q.shape, torch.bfloat16, q.device)
    _check_tensor(lse, "lse", shape, torch.float32, q.device)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(shape, dtype=torch.float32, device=q.device)
    st = capi.attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                           B, Hq, Hkv, S, D, causal, scale, q_descale, k_descale, v_descale,
                           cu_seqlens.data_ptr() if cu_seqlens is not None else None,
                           _stream(q.device))
    capi.check(st, "attn_fwd_fp8")
    return out, lse


def accumulate_bf16(acc: torch.Tensor, x: torch.Tensor, init: bool = False) -> torch.Tensor:
    """acc (fp32) = (0 if init else acc) + x (bf16), element-wise in libattn.so."""
    if not (acc.is_cuda and x.is_cuda and acc.is_contiguous() and x.is_contiguous()):
        raise ValueError("accumulate_bf16 needs contiguous CUDA tensors (there is no CPU path)")
    if acc.dtype != torch.float32 or x.dtype != torch.bfloat16 or acc.numel() != x.numel() \
            or acc.device != x.device:
        raise ValueError("acc must be fp32 and x bf16 of the same size, on one device")
    capi.check(capi.attn_accumulate_bf16(acc.data_ptr(), x.data_ptr(), x.numel(), init,
                                         _stream(x.device)), "attn_accumulate_bf16")
    return acc


def convert_f32_bf16(x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bf16 copy of an fp32 tensor (round to nearest even) in libattn.so."""
    if not (x.is_cuda and x.is_contiguous() and x.dtype == torch.float32):
        raise ValueError("convert_f32_bf16 needs a contiguous fp32 CUDA tensor")
    _check_tensor(out, "out", x.shape, torch.bfloat16, x.device)
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device) if out is None else out
    capi.check(capi.attn_convert_f32_bf16(out.data_ptr(), x.data_ptr(), x.numel(),
                                          _stream(x.device)), "attn_convert_f32_bf16")
    return out
