"""Tensor-core operand layouts, one tile each, through attn_selftest_umma.

Each mode is one of the MMA shapes the attention kernels issue (K-major x K-major
for S = QK^T, TMEM A x MN-major B for O += PV, MN-major A written by threads for
dQ = dS K); a descriptor or TMEM-layout error shows up here as a plain matrix
mismatch against torch's fp32 matmul.  The e4m3 modes (kind::f8f6f4) are checked
against exact products of the same e4m3 values in fp64.
"""
import numpy as np
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


def _fp8_run(mode, a_bytes, b_bytes, p=None):
    torch = pytest.importorskip("torch")
    dev = "cuda"
    b = torch.from_numpy(np.ascontiguousarray(b_bytes)).to(dev)
    a = torch.from_numpy(np.ascontiguousarray(a_bytes)).to(dev) if a_bytes is not None else None
    pin = torch.from_numpy(np.ascontiguousarray(p, dtype=np.float32)).to(dev) if p is not None else None
    pq = torch.full((128, 128), float("nan"), device=dev)
    c = torch.full((128, 128), float("nan"), device=dev)
    st = capi.attn_selftest_umma_fp8(mode, a.data_ptr() if a is not None else None, b.data_ptr(),
                                     pin.data_ptr() if pin is not None else None, pq.data_ptr(),
                                     c.data_ptr(), None)
    assert st == 0
    torch.cuda.synchronize()
    st, site = capi.attn_device_status(None)
    assert st == 0, hex(site)
    return c.cpu().numpy().astype(np.float64), pq.cpu().numpy().astype(np.float64)


@pytest.mark.gpu
def test_fp8_kmajor_ss():
    import e4m3
    rng = np.random.default_rng(7)
    a, b = e4m3.random_bytes(rng, (128, 128)), e4m3.random_bytes(rng, (128, 128))
    c, _ = _fp8_run(3, a, b)
    ref = e4m3.decode(a) @ e4m3.decode(b).T
    assert np.abs(c - ref).max() <= 1e-5 * np.abs(ref).max()


@pytest.mark.gpu
def test_fp8_tmem_a_mn_major_b():
    import e4m3
    rng = np.random.default_rng(8)
    v = e4m3.random_bytes(rng, (128, 128))
    p = (10.0 ** rng.uniform(-7, 0, size=(128, 128))).astype(np.float32)  # subnormal range too
    c, pq = _fp8_run(4, None, v, p)
    want_q = e4m3.quantize(256.0 * p.astype(np.float64))
    np.testing.assert_array_equal(pq, want_q)                 # packing and rounding of 256 P
    ref = want_q @ e4m3.decode(v)
    assert np.abs(c - ref).max() <= 1e-5 * np.abs(ref).max()
