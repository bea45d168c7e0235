"""FP8 (e4m3) forward (attn_fwd_fp8) on the GPU against the fp64 oracle on the dequantized
inputs (descale * e4m3 value, exact in fp64).

Tolerance (derived from the arithmetic; the bf16 bound of 1e-2 does not apply to 8-bit
inputs): the scores are exact products of e4m3 values summed in fp32, and the output is
O_i = sum_j w_j v_j / sum_j w_j with w_j = e4m3(256 p_j) / 256 the weights the PV MMA uses.
Rounding to e4m3 changes each weight by at most 2^-4 p_j (normal range) or 2^-17.5 in
absolute terms (subnormal range, p below about 2^-14.5 relative to the running maximum,
which lags the true maximum by at most 2^0.5).  So per output element
    |O_gpu - O_ref| <= sum_j |dw_j| |v_jd - O_id| / ((1 - 2^-4) sum_j p_j)
                       + half a bf16 ulp of O + 1e-5 (P|V|)_i,
computed here in fp64 for every checked row from that row's own scores.  The LSE comes
from the unquantised probabilities and keeps the 1e-3 bar.
"""
import numpy as np
import pytest

import e4m3
import oracle
from helpers import TOL_LSE, bf16_ulp, bits_of, f64, make_case
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")


def _fp8_inputs(w):
    x = I.make_inputs(w, with_do=False)
    out = {}
    for n in ("q", "k", "v"):
        b, d = e4m3.quantize_tensor(f64(x[n]))
        out[n] = (b, d, d * e4m3.decode(b))
    return x, out


def _run(w, out):
    from long_context_attention_fwd_b200 import ops
    dense = w.varlen is None
    T = w.tokens
    shp = lambda H: (w.B, w.S, H, w.D) if dense else (T, H, w.D)
    t = lambda n, H: torch.from_numpy(np.ascontiguousarray(out[n][0])).cuda().view(
        torch.float8_e4m3fn).view(shp(H))
    cu = None if dense else torch.from_numpy(I.cu_seqlens_from(w.varlen)).cuda()
    o, lse = ops.attn_fwd_fp8(t("q", w.Hq), t("k", w.Hkv), t("v", w.Hkv), out["q"][1], out["k"][1],
                              out["v"][1], causal=w.causal, scale=w.softmax_scale, cu_seqlens=cu)
    torch.cuda.synchronize()
    from long_context_attention_fwd_b200 import capi
    st, site = capi.attn_device_status(None)
    assert st == 0, hex(site)
    return f64(bits_of(o)).reshape(T, w.Hq, w.D), lse.double().cpu().numpy()


def _row_bound(qrow, K, V, o_ref, scale):
    s = scale * (K @ qrow)
    p = np.exp(s - s.max())
    dw = np.maximum(2.0 ** -4 * p, 2.0 ** -17.5)
    num = dw @ np.abs(V - o_ref[None, :])
    psum = p.sum()
    return (num / ((1 - 2.0 ** -4) * psum) + 0.5 * bf16_ulp(o_ref)
            + 1e-5 * (p @ np.abs(V)) / psum + 1e-7)


def _check_rows(w, out, o_g, lse_g, rows, o_r, l_r):
    """rows: (b, h, i) triples; o_r / l_r: the oracle's values for them."""
    q, k, v = (out[n][2].reshape(w.tokens, -1, w.D) for n in ("q", "k", "v"))
    cu = I.cu_seqlens_from(w.seq_lengths())
    G = w.Hq // w.Hkv
    worst = 0.0
    for (b, h, i), orow, lrow in zip(rows, o_r, l_r):
        t0 = int(cu[b])
        n = i + 1 if w.causal else w.seq_lengths()[b]
        K = k[t0:t0 + n, h // G]
        V = v[t0:t0 + n, h // G]
        bound = _row_bound(q[t0 + i, h], K, V, orow, w.softmax_scale)
        err = np.abs(o_g[t0 + i, h] - orow)
        assert (err <= bound).all(), (b, h, i, float((err - bound).max()))
        worst = max(worst, float((err / bound).max()))
        lg = lse_g[h, t0 + i] if w.varlen is not None else lse_g[b, h, i]
        assert abs(lg - lrow) <= TOL_LSE
    return worst


CASES = [
    make_case(1, 8, 2, 512, 128, causal=True, seed=91),
    make_case(2, 4, 4, 300, 128, causal=False, seed=92),
    make_case(0, 8, 2, 0, 128, causal=True, lens=[130, 1, 257, 64], seed=93),
    make_case(1, 4, 1, 384, 128, causal=True, seed=94, qkv_mult=2.0),   # peakier rows
]


@pytest.mark.gpu
@pytest.mark.parametrize("w", CASES, ids=["gqa4_S512_causal", "mha_B2_S300_full", "varlen_ragged",
                                          "mqa_peaky"])
def test_fp8_small_every_row(w):
    x, out = _fp8_inputs(w)
    o_g, lse_g = _run(w, out)
    kw = {"cu_seqlens": I.cu_seqlens_from(w.varlen)} if w.varlen is not None else {"B": w.B, "S": w.S}
    q, k, v = (out[n][2].reshape(w.tokens, -1, w.D) for n in ("q", "k", "v"))
    o_r, l_r = oracle.fwd(q, k, v, w.causal, w.softmax_scale, **kw)
    rows, orr, lrr = [], [], []
    cu = I.cu_seqlens_from(w.seq_lengths())
    for b, L in enumerate(w.seq_lengths()):
        for h in range(w.Hq):
            for i in range(L):
                rows.append((b, h, i))
                orr.append(o_r[cu[b] + i, h])
                lrr.append(l_r[h, cu[b] + i] if w.varlen is not None else l_r[b, h, i])
    _check_rows(w, out, o_g, lse_g, rows, orr, lrr)
    # overall: every weight is within 2^-4 of its own value, so the whole output is too
    # (about 2.4% relative L2 is typical: e4m3 keeps 3 mantissa bits of each probability)
    rel = np.linalg.norm(o_g - o_r) / np.linalg.norm(o_r)
    assert rel <= 2.0 ** -4, rel


@pytest.mark.gpu
def test_fp8_full_size_sampled_rows():
    w = I.workload(2)   # 32K causal, 28/4 heads, D = 128
    x, out = _fp8_inputs(w)
    o_g, lse_g = _run(w, out)
    rng = np.random.default_rng(11)
    rows = [(0, int(rng.integers(w.Hq)), int(i)) for i in
            list(rng.integers(0, w.S, size=20)) + [0, 1, 127, 128, 255, 256, w.S - 1]]
    q, k, v = (out[n][2].reshape(w.tokens, -1, w.D) for n in ("q", "k", "v"))
    o_r, l_r = oracle.fwd_rows(q, k, v, w.causal, w.softmax_scale, np.array(rows, np.int32),
                               B=1, S=w.S)
    _check_rows(w, out, o_g, lse_g, rows, o_r, l_r)
