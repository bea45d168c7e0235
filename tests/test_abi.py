"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/attn.h declares, and validates arguments before launching."""
import ctypes

import numpy as np
import pytest

from long_context_attention_fwd_b200 import capi


def test_exports_every_declared_symbol():
    lib = capi.lib()
    names = capi.declared_symbols()
    assert {"attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attn_strerror"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        assert n in capi._SIGNATURES, n


def test_version_and_strerror():
    assert capi.attn_version() >= 100
    for s in range(6):
        assert capi.strerror(s)
    assert capi.strerror(0) == "ok"


A = 0x10000  # fake, 16-byte aligned addresses: validation fails before any CUDA call


@pytest.mark.parametrize("args,want", [
    ((0, 2, 2, 128, 64), capi.ATTN_ERR_INVALID_ARG),     # B = 0
    ((1, 0, 2, 128, 64), capi.ATTN_ERR_INVALID_ARG),     # Hq = 0
    ((1, 3, 2, 128, 64), capi.ATTN_ERR_INVALID_ARG),     # Hq % Hkv
    ((1, 2, 2, 0, 64), capi.ATTN_ERR_INVALID_ARG),       # S = 0
    ((1, 2, 2, 128, 96), capi.ATTN_ERR_UNSUPPORTED),     # D
    ((1, 2, 2, 128, 256), capi.ATTN_ERR_UNSUPPORTED),
])
def test_fwd_validation(args, want):
    B, Hq, Hkv, S, D = args
    assert capi.attn_fwd(A, A, A, A, A, B, Hq, Hkv, S, D, 1, 0.125, None, None) == want


def test_fwd_scale_and_pointers():
    assert capi.attn_fwd(A, A, A, A, A, 1, 2, 2, 128, 64, 1, float("nan"), None, None) == 1
    assert capi.attn_fwd(A, A, A, A, A, 1, 2, 2, 128, 64, 1, float("inf"), None, None) == 1
    assert capi.attn_fwd(None, A, A, A, A, 1, 2, 2, 128, 64, 1, 0.1, None, None) == 1
    assert capi.attn_fwd(A + 8, A, A, A, A, 1, 2, 2, 128, 64, 1, 0.1, None, None) == 3
    assert capi.attn_fwd(A, A, A, A, A + 2, 1, 2, 2, 128, 64, 1, 0.1, None, None) == 3
    assert capi.attn_fwd(A, A, A, A, A, 1, 2, 2, 128, 64, 1, 0.1, A + 2, None) == 3


def test_bwd_validation_and_workspace():
    ws = capi.attn_bwd_workspace_size(1, 28, 32768, 128, None)
    T, Hq, D = 32768, 28, 128
    ntile = T // 128 + 1
    assert ws >= T * Hq * D * 4 + 2 * Hq * ntile * 128 * 4
    assert capi.attn_bwd_workspace_size(0, 28, 32768, 128, None) == 0
    assert capi.attn_bwd_workspace_size(1, 28, 32768, 96, None) == 0
    # packed: S is the total token count, so the workspace does not scale with B
    # (only one padding tile per sequence and head is added)
    assert capi.attn_bwd_workspace_size(8, 28, 32768, 128, 1) < 1.05 * ws
    args = [A] * 9 + [1, 2, 2, 128, 64, 1, 0.1, None]
    need = capi.attn_bwd_workspace_size(1, 2, 128, 64, None)
    assert capi.attn_bwd(*args, A, need - 1, None) == capi.ATTN_ERR_INVALID_ARG
    assert capi.attn_bwd(*args, A + 16, need, None) == capi.ATTN_ERR_MISALIGNED
    assert capi.attn_bwd(*args, None, need, None) == capi.ATTN_ERR_INVALID_ARG


def test_check_cu_seqlens_host():
    assert capi.attn_check_cu_seqlens([0, 3, 3, 10], 3, 10) == 0
    assert capi.attn_check_cu_seqlens([0, 3, 2, 10], 3, 10) == 1
    assert capi.attn_check_cu_seqlens([1, 3, 3, 10], 3, 10) == 1
    assert capi.attn_check_cu_seqlens([0, 3, 3, 9], 3, 10) == 1
    assert capi.attn_check_cu_seqlens([0, 3, 10], 3, 10) == 1


def test_ops_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    from long_context_attention_fwd_b200 import ops
    q = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.attn_fwd(q, q, q)


def test_merge_validation():
    m = capi.attn_merge
    assert m([], [], A, A, 1, 2, 8, 64, None) == capi.ATTN_ERR_INVALID_ARG          # no partials
    assert m([A] * 17, [A] * 17, A, A, 1, 2, 8, 64, None) == capi.ATTN_ERR_INVALID_ARG
    assert m([A, A], [A], A, A, 1, 2, 8, 64, None) == capi.ATTN_ERR_INVALID_ARG     # counts differ
    assert m([A, None], [A, A], A, A, 1, 2, 8, 64, None) == capi.ATTN_ERR_INVALID_ARG
    assert m([A, A], [A, A], None, A, 1, 2, 8, 64, None) == capi.ATTN_ERR_INVALID_ARG
    assert m([A, A], [A, A], A, A, 0, 2, 8, 64, None) == capi.ATTN_ERR_INVALID_ARG  # B = 0
    assert m([A, A], [A, A], A, A, 1, 2, 8, 96, None) == capi.ATTN_ERR_UNSUPPORTED  # D
    assert m([A, A], [A, A], A, A, 1 << 16, 1 << 8, 1 << 8, 64, None) == capi.ATTN_ERR_INVALID_ARG
    assert m([A, A + 8], [A, A], A, A, 1, 2, 8, 64, None) == capi.ATTN_ERR_MISALIGNED
    assert m([A, A], [A, A + 2], A, A, 1, 2, 8, 64, None) == capi.ATTN_ERR_MISALIGNED
    assert m([A, A], [A, A], A + 8, A, 1, 2, 8, 64, None) == capi.ATTN_ERR_MISALIGNED


def test_transpose_blocks_validation():
    t = capi.attn_transpose_blocks
    assert t(None, A, 2, 2, 16, None) == capi.ATTN_ERR_INVALID_ARG
    assert t(A, A + (1 << 20), 0, 2, 16, None) == capi.ATTN_ERR_INVALID_ARG      # n_outer = 0
    assert t(A, A + (1 << 20), 2, 2, 8, None) == capi.ATTN_ERR_INVALID_ARG       # < 16 bytes
    assert t(A, A + (1 << 20), 2, 2, 24, None) == capi.ATTN_ERR_MISALIGNED       # not 16k bytes
    assert t(A + 8, A + (1 << 20), 2, 2, 16, None) == capi.ATTN_ERR_MISALIGNED
    assert t(A, A + 32, 2, 2, 16, None) == capi.ATTN_ERR_INVALID_ARG             # overlap
    assert t(A, A + (1 << 40), 1 << 20, 1 << 8, 1 << 10, None) == capi.ATTN_ERR_INVALID_ARG


def test_decode_validation_and_workspace():
    ws = capi.attn_decode_workspace_size(16, 28, 4, 32768, 128)
    assert ws > 0
    assert capi.attn_decode_workspace_size(0, 28, 4, 32768, 128) == 0
    assert capi.attn_decode_workspace_size(1, 28, 3, 1024, 128) == 0      # Hq % Hkv
    assert capi.attn_decode_workspace_size(1, 256, 1, 1024, 128) == 0     # Hq/Hkv > 128
    assert capi.attn_decode_workspace_size(1, 28, 4, 1024, 96) == 0
    d = capi.attn_decode
    need = capi.attn_decode_workspace_size(2, 8, 2, 512, 64)
    args = (A, A, A, A, A, A, 2, 8, 2, 512, 64, 0.125)
    assert d(*args, A, need - 1, None) == capi.ATTN_ERR_INVALID_ARG
    assert d(*args, None, need, None) == capi.ATTN_ERR_INVALID_ARG
    assert d(*args, A + 16, need, None) == capi.ATTN_ERR_MISALIGNED      # workspace 256-aligned
    assert d(A + 8, *args[1:], A, need, None) == capi.ATTN_ERR_MISALIGNED
    assert d(A, A, A, A + 2, A, A, 2, 8, 2, 512, 64, 0.125, A, need, None) == capi.ATTN_ERR_MISALIGNED
    assert d(A, A, A, A, A, A, 2, 8, 2, 512, 96, 0.125, A, need, None) == capi.ATTN_ERR_UNSUPPORTED
    assert d(A, A, A, A, A, A, 2, 8, 2, 512, 64, float("nan"), A, need, None) == capi.ATTN_ERR_INVALID_ARG


def test_fwd_fp8_validation():
    f = capi.attn_fwd_fp8
    ok = (A, A, A, A, A, 1, 8, 2, 256, 128, 1, 0.125, 0.01, 0.02, 0.03, None, None)
    assert f(*ok[:9], 64, *ok[10:]) == capi.ATTN_ERR_UNSUPPORTED               # D must be 128
    assert f(*ok[:12], float("nan"), *ok[13:]) == capi.ATTN_ERR_INVALID_ARG      # q descale
    assert f(*ok[:14], float("inf"), *ok[15:]) == capi.ATTN_ERR_INVALID_ARG      # v descale
    assert f(*ok[:12], 1e30, 1e30, *ok[14:]) == capi.ATTN_ERR_INVALID_ARG        # scale product
    assert f(None, *ok[1:]) == capi.ATTN_ERR_INVALID_ARG
    assert f(A + 8, *ok[1:]) == capi.ATTN_ERR_MISALIGNED
    assert f(*ok[:5], 1, 6, 4, 256, 128, *ok[10:]) == capi.ATTN_ERR_INVALID_ARG  # Hq % Hkv


def test_selftest_fp8_validation():
    t = capi.attn_selftest_umma_fp8
    assert t(2, A, A, A, A, A, None) == capi.ATTN_ERR_INVALID_ARG
    assert t(3, None, A, None, None, A, None) == capi.ATTN_ERR_INVALID_ARG       # mode 3 needs a
    assert t(4, None, A, None, A, A, None) == capi.ATTN_ERR_INVALID_ARG          # mode 4 needs pin
    assert t(3, A, A + 8, None, None, A, None) == capi.ATTN_ERR_MISALIGNED
