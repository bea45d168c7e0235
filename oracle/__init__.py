"""fp64 CPU oracle for exact scaled-dot-product attention (forward and backward).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline / reference arm may import this package; the product library never
does, and it shares no code with the CUDA path.

The arithmetic lives in ``attn_oracle.c`` (plain loops, OpenMP over rows); this
module only compiles it with gcc on first use and marshals numpy arrays.  Every
function takes fp64 arrays; bf16 inputs are widened exactly with
``inputs.bf16_bits_to_f64`` before the call.

Parity status per function (pins live in tests/test_oracle_pins.py):
  fwd, fwd_rows, bwd, bwd_dq_rows, bwd_dkdv_range -- pinned by closed forms,
  invariants, finite differences and hand-derived golden values;
  merge_partials -- pinned by "merging chunk partials equals attention over all keys"
  and its special cases;
  bwd_given -- pinned by summing its block-pair gradients over a ring split and comparing
  with PyTorch's fp64 autograd of the whole attention;
  decode -- pinned by PyTorch's fp64 attention routine, closed forms (V = ones, identical
  keys, one cached key, an empty cache) and grouped-query = repeated multi-head.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "_attn_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile the oracle shared object (gcc, -O3, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp,
               _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def use_library(path: Optional[str]) -> None:
    """Points the bindings at another build of attn_oracle.c (the mutation tests
    load deliberately broken copies); None restores the default library."""
    global _lib, _LIB_OVERRIDE
    with _lock:
        _LIB_OVERRIDE = path
        _lib = None


_LIB_OVERRIDE: Optional[str] = None


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE is None:
                build()
            lib = ctypes.CDLL(_LIB_OVERRIDE or _LIB)
            common = [ctypes.c_int] * 6 + [ctypes.c_double, _I32]
            lib.oracle_attn_fwd.argtypes = [_D, _D, _D, _D, _D] + common
            lib.oracle_attn_fwd_rows.argtypes = [_D, _D, _D] + common + [
                ctypes.c_int, _I32, _I32, _I32, _D, _D]
            lib.oracle_attn_bwd.argtypes = [_D] * 7 + common
            lib.oracle_attn_bwd_dq_rows.argtypes = [_D] * 4 + common + [
                ctypes.c_int, _I32, _I32, _I32, _D, _D, _D]
            lib.oracle_attn_bwd_dkdv_range.argtypes = [_D] * 4 + common + [
                ctypes.c_int] * 4 + [_D, _D]
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_attn_bwd_given.argtypes = [_D, _D, _D, _D, _D, _D, _D, _D, _D, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_double]
            lib.oracle_attn_decode.argtypes = [_D, _D, _D, _I32, _D, _D, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_double]
            lib.oracle_merge_partials.argtypes = [ctypes.c_int, ctypes.POINTER(_D),
                                                  ctypes.POINTER(_D), _D, _D, ctypes.c_int64,
                                                  ctypes.c_int]
            _lib = lib
    return _lib


def _dp(a: np.ndarray):
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_D)


def _ip(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.dtype == np.int32 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_I32)


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _dims(q, k, B, S, cu):
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    if cu is None:
        assert T == B * S
    else:
        cu = np.ascontiguousarray(cu, dtype=np.int32)
        if cu.ndim != 1 or cu.size < 1 or int(cu[-1]) != T:
            raise ValueError("cu_seqlens must be 1-D and end at the token count")
        B = cu.size - 1
        S = T
    return B, Hq, Hkv, S, D, cu


def num_threads() -> int:
    return _load().oracle_num_threads()


def fwd(q, k, v, causal: bool, scale: float, B: int = 1, S: Optional[int] = None,
        cu_seqlens=None):
    """Full forward.  q [T,Hq,D], k/v [T,Hkv,D] -> (o [T,Hq,D], lse).
    lse is [B,Hq,S] (dense) or [Hq,T] (packed)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if S is None:
        S = q.shape[0] // max(B, 1)
    B, Hq, Hkv, S, D, cu = _dims(q, k, B, S, cu_seqlens)
    o = np.zeros_like(q)
    lse = np.zeros((Hq, S) if cu is not None else (B, Hq, S), dtype=np.float64)
    rc = _load().oracle_attn_fwd(_dp(q), _dp(k), _dp(v), _dp(o), _dp(lse), B, Hq, Hkv, S, D,
                                 int(causal), float(scale), _ip(cu))
    if rc:
        raise ValueError(f"oracle_attn_fwd failed ({rc})")
    return o, lse


def fwd_rows(q, k, v, causal: bool, scale: float, rows, B: int = 1, S: Optional[int] = None,
             cu_seqlens=None):
    """Forward for selected rows; ``rows`` is an (n,3) int array of (b, h, i).
    Returns (o_rows [n,D], lse_rows [n])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if S is None:
        S = q.shape[0] // max(B, 1)
    B, Hq, Hkv, S, D, cu = _dims(q, k, B, S, cu_seqlens)
    rows = np.asarray(rows, dtype=np.int32).reshape(-1, 3)
    rb, rh, ri = (np.ascontiguousarray(rows[:, c]) for c in range(3))
    n = rows.shape[0]
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = _load().oracle_attn_fwd_rows(_dp(q), _dp(k), _dp(v), B, Hq, Hkv, S, D, int(causal),
                                      float(scale), _ip(cu), n, _ip(rb), _ip(rh), _ip(ri),
                                      _dp(o), _dp(lse))
    if rc:
        raise ValueError(f"oracle_attn_fwd_rows failed ({rc})")
    return o, lse


def bwd(q, k, v, do, causal: bool, scale: float, B: int = 1, S: Optional[int] = None,
        cu_seqlens=None):
    """Full backward -> (dq [T,Hq,D], dk [T,Hkv,D], dv [T,Hkv,D])."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    if S is None:
        S = q.shape[0] // max(B, 1)
    B, Hq, Hkv, S, D, cu = _dims(q, k, B, S, cu_seqlens)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rc = _load().oracle_attn_bwd(_dp(q), _dp(k), _dp(v), _dp(do), _dp(dq), _dp(dk), _dp(dv),
                                 B, Hq, Hkv, S, D, int(causal), float(scale), _ip(cu))
    if rc:
        raise ValueError(f"oracle_attn_bwd failed ({rc})")
    return dq, dk, dv


def bwd_dq_rows(q, k, v, do, causal: bool, scale: float, rows, B: int = 1,
                S: Optional[int] = None, cu_seqlens=None):
    """dQ for selected rows (b, h, i) -> (dq_rows [n,D], lse_rows [n], delta_rows [n])."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    if S is None:
        S = q.shape[0] // max(B, 1)
    B, Hq, Hkv, S, D, cu = _dims(q, k, B, S, cu_seqlens)
    rows = np.asarray(rows, dtype=np.int32).reshape(-1, 3)
    rb, rh, ri = (np.ascontiguousarray(rows[:, c]) for c in range(3))
    n = rows.shape[0]
    dq = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    delta = np.zeros(n, dtype=np.float64)
    rc = _load().oracle_attn_bwd_dq_rows(_dp(q), _dp(k), _dp(v), _dp(do), B, Hq, Hkv, S, D,
                                         int(causal), float(scale), _ip(cu), n, _ip(rb), _ip(rh),
                                         _ip(ri), _dp(dq), _dp(lse), _dp(delta))
    if rc:
        raise ValueError(f"oracle_attn_bwd_dq_rows failed ({rc})")
    return dq, lse, delta


def bwd_dkdv_range(q, k, v, do, causal: bool, scale: float, b: int, g: int, j0: int, j1: int,
                   B: int = 1, S: Optional[int] = None, cu_seqlens=None):
    """dK, dV of keys j0..j1-1 of kv head g in sequence b -> (dk [j1-j0,D], dv [j1-j0,D])."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    if S is None:
        S = q.shape[0] // max(B, 1)
    B, Hq, Hkv, S, D, cu = _dims(q, k, B, S, cu_seqlens)
    dk = np.zeros((max(j1 - j0, 0), D), dtype=np.float64)
    dv = np.zeros_like(dk)
    rc = _load().oracle_attn_bwd_dkdv_range(_dp(q), _dp(k), _dp(v), _dp(do), B, Hq, Hkv, S, D,
                                            int(causal), float(scale), _ip(cu), b, g, j0, j1,
                                            _dp(dk), _dp(dv))
    if rc:
        raise ValueError(f"oracle_attn_bwd_dkdv_range failed ({rc})")
    return dk, dv


def merge_partials(o_parts, lse_parts):
    """Exact merge of partial attention results over disjoint key subsets.
    o_parts: list of [R, D] arrays, lse_parts: list of [R] arrays -> (o [R, D], lse [R])."""
    o_parts = [_f64(x) for x in o_parts]
    lse_parts = [_f64(x) for x in lse_parts]
    n = len(o_parts)
    R, D = o_parts[0].shape
    for a, l in zip(o_parts, lse_parts):
        if a.shape != (R, D) or l.shape != (R,):
            raise ValueError("partials must share shapes")
    optrs = (_D * n)(*[_dp(a) for a in o_parts])
    lptrs = (_D * n)(*[_dp(l) for l in lse_parts])
    o = np.zeros((R, D), dtype=np.float64)
    lse = np.zeros(R, dtype=np.float64)
    rc = _load().oracle_merge_partials(n, optrs, lptrs, _dp(o), _dp(lse), R, D)
    if rc:
        raise ValueError(f"oracle_merge_partials failed ({rc})")
    return o, lse


def decode(q, k_cache, v_cache, cache_len, scale: float):
    """Decode attention: q [B,Hq,D], k/v cache [B,Lmax,Hkv,D], cache_len [B] ->
    (o [B,Hq,D], lse [B,Hq])."""
    q, k_cache, v_cache = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    if k_cache.shape != (B, Lmax, Hkv, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shapes must be [B, Lmax, Hkv, D]")
    cl = np.ascontiguousarray(cache_len, dtype=np.int32)
    if cl.shape != (B,):
        raise ValueError("cache_len must have B entries")
    o = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    rc = _load().oracle_attn_decode(_dp(q), _dp(k_cache), _dp(v_cache), _ip(cl), _dp(o), _dp(lse),
                                    B, Hq, Hkv, Lmax, D, float(scale))
    if rc:
        raise ValueError(f"oracle_attn_decode failed ({rc})")
    return o, lse


def bwd_given(q, k, v, o, lse, do, causal: bool, scale: float, B: int, S: int):
    """Block-pair backward with the whole problem's O [B*S,Hq,D] and LSE [B,Hq,S] given
    -> (dq, dk, dv); dense layouts as in bwd."""
    q, k, v, o, lse, do = (_f64(x) for x in (q, k, v, o, lse, do))
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    if T != B * S or lse.shape != (B, Hq, S) or o.shape != q.shape or do.shape != q.shape:
        raise ValueError("shapes do not match")
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    rc = _load().oracle_attn_bwd_given(_dp(q), _dp(k), _dp(v), _dp(o), _dp(lse), _dp(do), _dp(dq),
                                       _dp(dk), _dp(dv), B, Hq, Hkv, S, D, int(causal),
                                       float(scale))
    if rc:
        raise ValueError(f"oracle_attn_bwd_given failed ({rc})")
    return dq, dk, dv
