"""ctypes binding of libattn.so: the C entry points under the same names.

Argument marshalling only -- every step of the attention runs in the library's
CUDA kernels.  Loading fails loudly when the library has not been built; there
is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "attn.h")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_MISALIGNED = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5
ATTN_BWD_NOALLOC_MAX_BYTES = 64 << 20  # the header's define of the same name


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == ATTN_ERR_CUDA:
            try:
                detail = " [" + lib().attn_last_error().decode() + "]"
            except Exception:
                pass
        super().__init__(f"{where}: {strerror(status)} (status {status}){detail}")


_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_fp = ctypes.c_void_p  # float* passed as raw address
_sz = ctypes.c_size_t

_SIGNATURES = {
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _fp, _i, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp]),
    "attn_fwd_fp8": (_i, [_vp, _vp, _vp, _vp, _fp, _i, _i, _i, _i, _i, _i, ctypes.c_float,
                          ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp]),
    "attn_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _vp]),
    "attn_bwd": (_i, [_vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                      ctypes.c_float, _vp, _vp, _sz, _vp]),
    "attn_strerror": (ctypes.c_char_p, [_i]),
    "attn_device_status": (_i, [_vp, ctypes.POINTER(ctypes.c_uint)]),
    "attn_set_wait_timeout_ns": (None, [ctypes.c_ulonglong]),
    "attn_check_cu_seqlens": (_i, [ctypes.POINTER(ctypes.c_int32), _i, _i]),
    "attn_selftest_wait_timeout": (_i, [ctypes.c_ulonglong, _vp]),
    "attn_selftest_umma": (_i, [_i, _i, _vp, _vp, _fp, _vp, _fp, _vp]),
    "attn_selftest_umma_fp8": (_i, [_i, _vp, _vp, _fp, _fp, _fp, _vp]),
    "attn_version": (_i, []),
    "attn_last_error": (ctypes.c_char_p, []),
    "attn_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "attn_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _fp, _i, _i, _i, _i, _i, ctypes.c_float, _vp,
                         _sz, _vp]),
    "attn_accumulate_bf16": (_i, [_fp, _vp, ctypes.c_longlong, _i, _vp]),
    "attn_convert_f32_bf16": (_i, [_vp, _fp, ctypes.c_longlong, _vp]),
    "attn_transpose_blocks": (_i, [_vp, _vp, ctypes.c_longlong, ctypes.c_longlong,
                                   ctypes.c_longlong, _vp]),
    "attn_merge": (_i, [_vp, _vp, _i, _vp, _fp, _i, _i, _i, _i, _vp]),
    "attn_selftest_exp2": (_i, [_fp, _fp, ctypes.c_longlong, _vp]),
    "attn_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                              ctypes.c_float, _vp, _vp]),
}


def declared_symbols() -> list:
    """Names of the functions include/attn.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def lib():
    """The loaded library (built on first use if nvcc is available)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                try:
                    from . import build as _build
                    _build.build()
                except Exception as e:  # pragma: no cover - depends on the toolchain
                    raise ImportError(
                        f"libattn.so is not built and building it failed: {e}. "
                        "Run `python -m long_context_attention_fwd_b200.build`.") from e
            l = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(l, name)
                fn.restype = res
                fn.argtypes = args
            _lib = l
    return _lib


def strerror(status: int) -> str:
    try:
        return lib().attn_strerror(int(status)).decode()
    except Exception:
        return f"status {status}"


def check(status: int, where: str) -> None:
    if status != ATTN_OK:
        raise AttnError(status, where)


# Raw entry points under the C names (addresses as Python ints, stream as an int).
def attn_fwd(q, k, v, o, lse, B, Hq, Hkv, S, D, causal, scale, cu_seqlens, stream) -> int:
    return lib().attn_fwd(q, k, v, o, lse, B, Hq, Hkv, S, D, int(causal), float(scale),
                          cu_seqlens, stream)


def attn_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, S, D, causal, scale, q_descale, k_descale,
                 v_descale, cu_seqlens, stream) -> int:
    return lib().attn_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, S, D, int(causal), float(scale),
                              float(q_descale), float(k_descale), float(v_descale), cu_seqlens,
                              stream)


def attn_bwd_workspace_size(B, Hq, S, D, cu_seqlens) -> int:
    return lib().attn_bwd_workspace_size(B, Hq, S, D, cu_seqlens)


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, causal, scale, cu_seqlens,
             workspace, workspace_bytes, stream) -> int:
    return lib().attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, int(causal),
                          float(scale), cu_seqlens, workspace, workspace_bytes, stream)


def attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, causal, scale,
                     cu_seqlens, stream) -> int:
    return lib().attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, int(causal),
                                  float(scale), cu_seqlens, stream)


def attn_merge(o_parts, lse_parts, o, lse, B, H, S, D, stream) -> int:
    """o_parts / lse_parts: sequences of device addresses (marshalled into host arrays)."""
    n = len(o_parts)
    if n != len(lse_parts):
        return ATTN_ERR_INVALID_ARG
    oa = (ctypes.c_void_p * max(n, 1))(*o_parts)
    la = (ctypes.c_void_p * max(n, 1))(*lse_parts)
    return lib().attn_merge(ctypes.cast(oa, _vp), ctypes.cast(la, _vp), n, o, lse, B, H, S, D,
                            stream)


def attn_decode_workspace_size(B, Hq, Hkv, Lmax, D) -> int:
    return lib().attn_decode_workspace_size(B, Hq, Hkv, Lmax, D)


def attn_decode(q, k_cache, v_cache, cache_len, o, lse, B, Hq, Hkv, Lmax, D, scale, workspace,
                workspace_bytes, stream) -> int:
    return lib().attn_decode(q, k_cache, v_cache, cache_len, o, lse, B, Hq, Hkv, Lmax, D,
                             float(scale), workspace, workspace_bytes, stream)


def attn_accumulate_bf16(acc, x, n, init, stream) -> int:
    return lib().attn_accumulate_bf16(acc, x, int(n), int(init), stream)


def attn_convert_f32_bf16(out, inp, n, stream) -> int:
    return lib().attn_convert_f32_bf16(out, inp, int(n), stream)


def attn_transpose_blocks(inp, out, n_outer, n_inner, block_bytes, stream) -> int:
    return lib().attn_transpose_blocks(inp, out, int(n_outer), int(n_inner), int(block_bytes),
                                       stream)


def attn_device_status(stream=None):
    site = ctypes.c_uint(0)
    st = lib().attn_device_status(stream, ctypes.byref(site))
    return st, site.value


def attn_set_wait_timeout_ns(ns: int) -> None:
    lib().attn_set_wait_timeout_ns(int(ns))


def attn_check_cu_seqlens(cu_host, B: int, S: int) -> int:
    import numpy as np
    a = np.ascontiguousarray(cu_host, dtype=np.int32)
    if a.size != B + 1:
        return ATTN_ERR_INVALID_ARG
    return lib().attn_check_cu_seqlens(a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), B, S)


def attn_selftest_wait_timeout(ns: int, stream=None) -> int:
    return lib().attn_selftest_wait_timeout(int(ns), stream)


def attn_selftest_umma(mode, D, a, b, p, at, c, stream=None) -> int:
    return lib().attn_selftest_umma(mode, D, a, b, p, at, c, stream)


def attn_selftest_umma_fp8(mode, a, b, pin, pq, c, stream=None) -> int:
    return lib().attn_selftest_umma_fp8(mode, a, b, pin, pq, c, stream)


def attn_selftest_exp2(x, y, n, stream=None) -> int:
    return lib().attn_selftest_exp2(x, y, int(n), stream)


def attn_version() -> int:
    return lib().attn_version()


def attn_last_error() -> str:
    return lib().attn_last_error().decode()
