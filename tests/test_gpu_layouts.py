"""Tensor-core operand layouts, one tile each, through attn_selftest_umma.

Each mode is one of the MMA shapes the attention kernels issue (K-major x K-major
for S = QK^T, TMEM A x MN-major B for O += PV, MN-major A written by threads for
dQ = dS K); a descriptor or TMEM-layout error shows up here as a plain matrix
mismatch against torch's fp32 matmul.
"""
import pytest

from long_context_attention_fwd_b200 import capi

torch = pytest.importorskip("torch")


def _run(mode, D, a=None, b=None, p=None, at=None):
    ncol = 128 if mode == 0 else D
    c = torch.full((128, ncol), float("nan"), dtype=torch.float32, device="cuda")
    ptr = lambda t: t.data_ptr() if t is not None else None
    st = capi.attn_selftest_umma(mode, D, ptr(a), ptr(b), ptr(p), ptr(at), c.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    capi.check(st, "attn_selftest_umma")
    torch.cuda.synchronize()
    st, site = capi.attn_device_status(None)
    assert st == capi.ATTN_OK, (st, hex(site))
    return c


@pytest.mark.gpu
@pytest.mark.parametrize("D", [64, 128])
def test_kmajor_ss(D):
    g = torch.Generator(device="cuda").manual_seed(1)
    a = torch.randn(128, D, device="cuda", generator=g).bfloat16()
    b = torch.randn(128, D, device="cuda", generator=g).bfloat16()
    c = _run(0, D, a=a, b=b)
    ref = a.float() @ b.float().T
    torch.testing.assert_close(c, ref, rtol=1e-4, atol=1e-3)


@pytest.mark.gpu
@pytest.mark.parametrize("D", [64, 128])
def test_tmem_a_mn_major_b(D):
    g = torch.Generator(device="cuda").manual_seed(2)
    p = torch.rand(128, 128, device="cuda", generator=g)
    b = torch.randn(128, D, device="cuda", generator=g).bfloat16()
    c = _run(1, D, b=b, p=p)
    ref = p.bfloat16().float() @ b.float()
    torch.testing.assert_close(c, ref, rtol=1e-4, atol=1e-3)


@pytest.mark.gpu
@pytest.mark.parametrize("D", [64, 128])
def test_mn_major_a_from_threads(D):
    g = torch.Generator(device="cuda").manual_seed(3)
    at = torch.randn(128, 128, device="cuda", generator=g).bfloat16()
    b = torch.randn(128, D, device="cuda", generator=g).bfloat16()
    c = _run(2, D, b=b, at=at)
    ref = at.float().T @ b.float()
    torch.testing.assert_close(c, ref, rtol=1e-4, atol=1e-3)
