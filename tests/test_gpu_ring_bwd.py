"""Ring-Attention backward on the GPU: the fp32 accumulation kernels bit for bit against
torch, and every rank of an N-rank ring run on one GPU (attn_bwd on each block pair with
the merged O and LSE, shares summed by attn_accumulate_bf16, rounded once by
attn_convert_f32_bf16) against the single-kernel backward and the fp64 oracle.

Expected differences: each block pair's share is rounded to bf16 before it is summed, so
the ring's gradients differ from the single-kernel ones by about one bf16 rounding
(relative L2 ~1e-3, bound 4e-3); against the oracle the bar is the gradient bar, 1e-2."""
import numpy as np
import pytest

import oracle
from helpers import TOL_GRAD, bits_of, f64, make_case, oracle_args, rel_l2, torch_bf16
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")


@pytest.mark.gpu
@pytest.mark.parametrize("n", [8, 8 * 1000 + 8, 3 * 28 * 128 * 64])
def test_accumulate_and_convert_bit_exact(n):
    from long_context_attention_fwd_b200 import ops
    g = torch.Generator(device="cuda").manual_seed(n)
    x = torch.randn(n, device="cuda", generator=g).bfloat16()
    a0 = torch.randn(n, device="cuda", generator=g)
    acc = a0.clone()
    ops.accumulate_bf16(acc, x)
    assert torch.equal(acc, a0 + x.float())
    ops.accumulate_bf16(acc, x, init=True)
    assert torch.equal(acc, x.float())
    y = torch.randn(n, device="cuda", generator=g) * 3
    assert torch.equal(ops.convert_f32_bf16(y).view(torch.int16), y.bfloat16().view(torch.int16))


def _ring_grads(w, world):
    from long_context_attention_fwd_b200 import ops, ring
    x = I.make_inputs(w)
    shp_q, shp_k = (w.B, w.S, w.Hq, w.D), (w.B, w.S, w.Hkv, w.D)
    q, k, v, do = (torch_bf16(x[n]).view(s) for n, s in
                   (("q", shp_q), ("k", shp_k), ("v", shp_k), ("do", shp_q)))
    o, lse = ops.attn_fwd(q, k, v, causal=w.causal, scale=w.softmax_scale)
    rq, rk, rv = ring.ring_attn_bwd_single_device(q, k, v, o, lse, do, world, w.causal,
                                                  w.softmax_scale)
    fq, fk, fv = ops.attn_bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.softmax_scale)
    torch.cuda.synchronize()
    from long_context_attention_fwd_b200 import capi
    st, site = capi.attn_device_status(None)
    assert st == 0, hex(site)
    return x, (rq, rk, rv), (fq, fk, fv)


def _rel(a, b):
    a, b = a.float(), b.float()
    return float((a - b).norm() / b.norm())


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("dims,causal", [((1, 8, 2, 512, 128), True), ((2, 4, 4, 384, 64), False)])
def test_ring_backward_small_equals_oracle(world, dims, causal):
    B, Hq, Hkv, S, D = dims
    w = make_case(B, Hq, Hkv, S, D, causal=causal, seed=70 + S + world)
    x, ring_g, full_g = _ring_grads(w, world)
    for a, b in zip(ring_g, full_g):
        assert _rel(a, b) <= 4e-3
    q, k, v, do, kw = oracle_args(w, x)
    ref = oracle.bwd(q, k, v, do, causal, w.softmax_scale, **kw)
    T = w.tokens
    for got, want, H in zip(ring_g, ref, (Hq, Hkv, Hkv)):
        assert rel_l2(f64(bits_of(got)).reshape(T, H, D), want) <= TOL_GRAD


@pytest.mark.gpu
def test_ring_backward_8k_equals_single_kernel():
    w = I.workload(1)   # 8K causal, 28/4 heads, D = 128
    _, ring_g, full_g = _ring_grads(w, 4)
    for a, b in zip(ring_g, full_g):
        assert _rel(a, b) <= 4e-3
