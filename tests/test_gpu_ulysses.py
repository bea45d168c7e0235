"""Ulysses sequence parallelism on the GPU: the relayout kernel (attn_transpose_blocks)
against a plain tensor permutation, bit for bit, and every rank of an N-rank Ulysses group
run on one GPU (relayout kernels around emulated all-to-alls, attention on each head
group) against the single-kernel attention over all heads and against the fp64 oracle.

Splitting the heads changes neither the per-head forward nor the order in which the
backward sums a key/value head's group, so o, lse-derived outputs, dk and dv must match
the unsplit kernels bit for bit; dq is summed with fp32 atomics, so it is compared with a
tolerance."""
import numpy as np
import pytest

import oracle
from helpers import (TOL_GRAD, TOL_LSE, bits_of, f64, make_case, o_error_report, oracle_args,
                     rel_l2, torch_bf16)
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")


@pytest.mark.gpu
@pytest.mark.parametrize("n_outer,n_inner,block_elems", [
    (1, 1, 8), (3, 5, 8), (37, 4, 896), (4, 37, 128), (8192, 4, 128), (4, 8192, 896),
    (2, 3, 7 * 8192 * 128), (1000, 7, 24)])
def test_transpose_blocks_bit_exact(n_outer, n_inner, block_elems):
    from long_context_attention_fwd_b200 import ops
    g = torch.Generator(device="cuda").manual_seed(n_outer * 31 + n_inner)
    x = torch.randint(-32768, 32767, (n_outer, n_inner, block_elems), dtype=torch.int16,
                      device="cuda", generator=g)
    y = ops.transpose_blocks(x, n_outer, n_inner)
    torch.cuda.synchronize()
    assert torch.equal(y, x.transpose(0, 1).contiguous())


def _ulysses_case(w, world):
    from long_context_attention_fwd_b200 import ops
    from long_context_attention_fwd_b200 import ulysses as U
    x = I.make_inputs(w)
    shp_q, shp_k = (w.B, w.S, w.Hq, w.D), (w.B, w.S, w.Hkv, w.D)
    q, k, v, do = (torch_bf16(x[n]).view(s) for n, s in
                   (("q", shp_q), ("k", shp_k), ("v", shp_k), ("do", shp_q)))
    o, dq, dk, dv = U.ulysses_attention_single_device(q, k, v, world, w.causal,
                                                      w.softmax_scale, do=do)
    of, lf = ops.attn_fwd(q, k, v, causal=w.causal, scale=w.softmax_scale)
    dqf, dkf, dvf = ops.attn_bwd(q, k, v, of, lf, do, causal=w.causal, scale=w.softmax_scale)
    torch.cuda.synchronize()
    return x, (o, dq, dk, dv), (of, dqf, dkf, dvf)


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("dims,causal", [((2, 8, 4, 512, 64), True), ((1, 8, 4, 384, 128), False),
                                         ((1, 4, 4, 640, 128), True)])
def test_ulysses_small_equals_oracle(world, dims, causal):
    B, Hq, Hkv, S, D = dims
    w = make_case(B, Hq, Hkv, S, D, causal=causal, seed=50 + S + world)
    x, (o, dq, dk, dv), (of, dqf, dkf, dvf) = _ulysses_case(w, world)
    assert _same_bits(o, of) and _same_bits(dk, dkf) and _same_bits(dv, dvf)
    q, k, v, d_o, kw = oracle_args(w, x)
    o_r, _ = oracle.fwd(q, k, v, causal, w.softmax_scale, **kw)
    oa_r, _ = oracle.fwd(q, k, np.abs(v), causal, w.softmax_scale, **kw)
    g_r = oracle.bwd(q, k, v, d_o, causal, w.softmax_scale, **kw)
    T = w.tokens
    rep = o_error_report(f64(bits_of(o)).reshape(T, Hq, D), o_r, oa_r)
    assert rep["n_over_model"] == 0 and rep["max_abs"] <= 1e-2, rep
    for got, ref, H in ((dq, g_r[0], Hq), (dk, g_r[1], Hkv), (dv, g_r[2], Hkv)):
        assert rel_l2(f64(bits_of(got)).reshape(T, H, D), ref) <= TOL_GRAD


@pytest.mark.gpu
@pytest.mark.parametrize("idx,world", [(1, 2), (1, 4), (2, 4)], ids=["S8K_N2", "S8K_N4",
                                                                       "S32K_N4"])
def test_ulysses_full_size_matches_unsplit_kernels(idx, world):
    w = I.workload(idx)
    x, (o, dq, dk, dv), (of, dqf, dkf, dvf) = _ulysses_case(w, world)
    assert _same_bits(o, of)
    assert _same_bits(dk, dkf) and _same_bits(dv, dvf)
    # dq: same arithmetic, different fp32 atomic order.  Where a sum cancels, the order
    # moves the result by the rounding of its terms, not of the result, so the bound is on
    # the tensor's scale: relative L2 within a bf16 rounding, max difference within one
    # bf16 step of the largest element.
    a, b = dq.float(), dqf.float()
    assert float((a - b).norm() / b.norm()) <= 2.0 ** -8
    assert float((a - b).abs().max()) <= 2.0 ** -7 * float(b.abs().max())
    # sampled rows against the oracle
    q, k, v, _, kw = oracle_args(w, x)
    rng = np.random.default_rng(idx * 7 + world)
    rows = np.array([(0, int(rng.integers(w.Hq)), int(rng.integers(w.S))) for _ in range(12)],
                    dtype=np.int32)
    o_r, l_r = oracle.fwd_rows(q, k, v, w.causal, w.softmax_scale, rows, **kw)
    oa_r, _ = oracle.fwd_rows(q, k, np.abs(v), w.causal, w.softmax_scale, rows, **kw)
    og = f64(bits_of(o)).reshape(w.S, w.Hq, w.D)[rows[:, 2], rows[:, 1]]
    rep = o_error_report(og, o_r, oa_r)
    assert rep["n_over_model"] == 0 and rep["max_abs"] <= 1e-2, rep


@pytest.mark.gpu
@pytest.mark.parametrize("lens,world", [([300, 1, 0, 211, 128], 2), (None, 4)],
                         ids=["packed_small_N2", "packed32K_N4"])
def test_ulysses_packed_matches_unsplit_kernels(lens, world):
    """Packed batches: every rank holds a slice of the token stream that cuts sequences
    mid-way; after the exchange each head group runs the packed kernels with the batch's
    global cu_seqlens, so o, dk and dv equal the unsplit packed kernels bit for bit."""
    from long_context_attention_fwd_b200 import ops
    from long_context_attention_fwd_b200 import ulysses as U
    w = I.workload(3) if lens is None else make_case(0, 4, 2, 0, 128, True, lens=lens, seed=61)
    x = I.make_inputs(w)
    T = w.tokens
    q, k, v, do = (torch_bf16(x[n]).view(T, h, w.D) for n, h in
                   (("q", w.Hq), ("k", w.Hkv), ("v", w.Hkv), ("do", w.Hq)))
    cu = torch.from_numpy(x["cu_seqlens"]).cuda()
    o, dq, dk, dv = U.ulysses_attention_single_device(q, k, v, world, w.causal, w.softmax_scale,
                                                      do=do, cu_seqlens=cu)
    of, lf = ops.attn_fwd(q, k, v, causal=w.causal, scale=w.softmax_scale, cu_seqlens=cu)
    dqf, dkf, dvf = ops.attn_bwd(q, k, v, of, lf, do, causal=w.causal, scale=w.softmax_scale,
                                 cu_seqlens=cu)
    torch.cuda.synchronize()
    assert _same_bits(o, of)
    assert _same_bits(dk, dkf) and _same_bits(dv, dvf)
    a, b = dq.float(), dqf.float()
    assert float((a - b).norm() / b.norm()) <= 2.0 ** -8
    if lens is not None:   # small: the whole result against the oracle
        qn, kn, vn, don, kw = oracle_args(w, x)
        o_r, _ = oracle.fwd(qn, kn, vn, True, w.softmax_scale, **kw)
        oa_r, _ = oracle.fwd(qn, kn, np.abs(vn), True, w.softmax_scale, **kw)
        rep = o_error_report(f64(bits_of(o)).reshape(T, w.Hq, w.D), o_r, oa_r)
        assert rep["n_over_model"] == 0 and rep["max_abs"] <= 1e-2, rep
        g_r = oracle.bwd(qn, kn, vn, don, True, w.softmax_scale, **kw)
        for got, ref, H in ((dq, g_r[0], w.Hq), (dk, g_r[1], w.Hkv), (dv, g_r[2], w.Hkv)):
            assert rel_l2(f64(bits_of(got)).reshape(T, H, w.D), ref) <= TOL_GRAD
