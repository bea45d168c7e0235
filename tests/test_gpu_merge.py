"""The exact merge of partial attention results (attn_merge) and the Ring forward built
on it, on the GPU, against the fp64 oracle.

  * attn_merge on seeded partials (bf16 o, fp32 lse spread over a wide range, some -inf
    partials, rows whose partials are all -inf), D 64 and 128, 1 to 20 partials, row
    counts that leave a ragged last group; bound: half a bf16 ulp of the exact result
    plus the fp32 rounding of the weighted sum;
  * in-place use (out = o_parts[0], lse = lse_parts[0]) and determinism;
  * the Ring forward of every rank of an N-rank ring, run on one GPU from attn_fwd
    partials (unmasked off-diagonal chunks, causal diagonal chunk) and attn_merge, against
    the oracle's attention over the whole sequence: small cases element by element,
    the 8K and 32K grouped-query workloads on sampled rows.
"""
import numpy as np
import pytest

import oracle
from helpers import (TOL_LSE, bf16_ulp, bits_of, f64, o_error_report, oracle_args, torch_bf16)
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")


def _partials(n, B, S, H, D, seed, ninf_frac=0.05, dead_rows=3):
    """n seeded partials: o bf16 [B,S,H,D], lse fp32 [B,H,S] (some entries -inf)."""
    key = lambda sub: I.stream_key(seed, sub)
    R = B * S * H
    o_bits = [I.to_bf16_bits(I.normal(key(10 + p), R * D) * 1.5) for p in range(n)]
    lse = []
    for p in range(n):
        l = (I.normal(key(40 + p), R) * 4.0 + 2.0).astype(np.float32)
        u = I.uniform(key(70 + p), R)
        l[u < ninf_frac] = -np.inf
        lse.append(l.reshape(B, H, S))
    for r in range(min(dead_rows, S)):          # rows (b=0, h=0, i=r): nothing visible
        for p in range(n):
            lse[p][0, 0, r] = -np.inf
    return o_bits, lse


def _oracle_merge(o_bits, lse, B, S, H, D):
    po = [f64(b).reshape(B * S * H, D) for b in o_bits]                           # (b, i, h)
    pl = [l.astype(np.float64).transpose(0, 2, 1).reshape(-1) for l in lse]
    o, l = oracle.merge_partials(po, pl)
    return o, l.reshape(B, S, H).transpose(0, 2, 1)


def _gpu_parts(o_bits, lse, B, S, H, D):
    o_t = [torch_bf16(b).view(B, S, H, D) for b in o_bits]
    l_t = [torch.from_numpy(l).cuda() for l in lse]
    return o_t, l_t


def _check_merge(o_g, lse_g, o_bits, lse, B, S, H, D):
    o_ref, l_ref = _oracle_merge(o_bits, lse, B, S, H, D)
    og = f64(bits_of(o_g)).reshape(B * S * H, D)
    # weights of the exact merge, for the bound on the fp32 weighted sum
    pl = np.stack([l.astype(np.float64).transpose(0, 2, 1).reshape(-1) for l in lse])
    with np.errstate(invalid="ignore"):
        w = np.exp(pl - l_ref.transpose(0, 2, 1).reshape(-1))
    w = np.nan_to_num(w)
    sum_abs = sum(w[p][:, None] * np.abs(f64(o_bits[p]).reshape(-1, D)) for p in range(len(o_bits)))
    bound = 0.5 * bf16_ulp(o_ref) + 4e-6 * sum_abs + 1e-30
    err = np.abs(og - o_ref)
    assert (err <= bound).all(), float((err - bound).max())
    lg = lse_g.double().cpu().numpy()
    dead = np.isneginf(l_ref)
    assert (np.isneginf(lg) == dead).all()
    assert (og.reshape(B, S, H, D)[dead.transpose(0, 2, 1)] == 0).all()
    fin = ~dead
    assert (np.abs(lg[fin] - l_ref[fin]) <= 4e-6 * np.maximum(1.0, np.abs(l_ref[fin]))).all()


@pytest.mark.gpu
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 16])
@pytest.mark.parametrize("shape", [(1, 37, 3), (2, 129, 4)])
def test_merge_matches_oracle(D, n, shape):
    from long_context_attention_fwd_b200 import ops
    B, S, H = shape
    o_bits, lse = _partials(n, B, S, H, D, seed=D * 100 + n)
    o_t, l_t = _gpu_parts(o_bits, lse, B, S, H, D)
    o_g, lse_g = ops.attn_merge(o_t, l_t)
    torch.cuda.synchronize()
    _check_merge(o_g, lse_g, o_bits, lse, B, S, H, D)
    if n == 1:   # a single partial passes through unchanged
        fin = np.isfinite(lse[0])
        assert (bits_of(o_g).reshape(B, S, H, D)[fin.transpose(0, 2, 1)] ==
                o_bits[0].reshape(B, S, H, D)[fin.transpose(0, 2, 1)]).all()
        assert (lse_g.cpu().numpy()[fin] == lse[0][fin]).all()


@pytest.mark.gpu
def test_merge_more_than_max_parts_and_packed_layout():
    from long_context_attention_fwd_b200 import ops
    n, T, H, D = 20, 301, 2, 128
    o_bits, lse = _partials(n, 1, T, H, D, seed=77, dead_rows=0)
    o_t = [torch_bf16(b).view(T, H, D) for b in o_bits]
    l_t = [torch.from_numpy(l.reshape(H, T)).cuda() for l in lse]
    o_g, lse_g = ops.attn_merge(o_t, l_t)
    torch.cuda.synchronize()
    o_ref, l_ref = _oracle_merge(o_bits, lse, 1, T, H, D)
    og = f64(bits_of(o_g)).reshape(-1, D)
    # two levels of merging: each group's result is rounded to bf16 once more
    assert np.abs(og - o_ref).max() <= 2.0 ** -7 * np.abs(o_ref).max()
    assert np.abs(lse_g.double().cpu().numpy() - l_ref[0]).max() <= 1e-5 * np.abs(l_ref).max()


@pytest.mark.gpu
def test_merge_in_place_and_deterministic():
    from long_context_attention_fwd_b200 import ops
    B, S, H, D = 1, 1000, 7, 128
    o_bits, lse = _partials(3, B, S, H, D, seed=5)
    o_t, l_t = _gpu_parts(o_bits, lse, B, S, H, D)
    a = ops.attn_merge(o_t, l_t)
    b = ops.attn_merge(o_t, l_t)
    ops.attn_merge(o_t, l_t, out=o_t[0], lse=l_t[0])
    torch.cuda.synchronize()
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[0].view(torch.int16), o_t[0].view(torch.int16))
    assert torch.equal(a[1], b[1]) and torch.equal(a[1], l_t[0])


def _ring_case(w, world):
    from long_context_attention_fwd_b200 import ring
    x = I.make_inputs(w)
    q = torch_bf16(x["q"]).view(w.B, w.S, w.Hq, w.D)
    k = torch_bf16(x["k"]).view(w.B, w.S, w.Hkv, w.D)
    v = torch_bf16(x["v"]).view(w.B, w.S, w.Hkv, w.D)
    o, lse = ring.ring_attn_fwd_single_device(q, k, v, world, w.causal, w.softmax_scale)
    torch.cuda.synchronize()
    return x, o, lse


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dims", [(2, 4, 2, 320, 64), (1, 4, 1, 512, 128)])
def test_ring_forward_small_equals_oracle(world, causal, dims):
    from helpers import make_case
    B, Hq, Hkv, S, D = dims
    w = make_case(B, Hq, Hkv, S, D, causal=causal, seed=31 + S + world)
    x, o, lse = _ring_case(w, world)
    q, k, v, _, kw = oracle_args(w, x)
    o_ref, l_ref = oracle.fwd(q, k, v, causal, w.softmax_scale, **kw)
    oa_ref, _ = oracle.fwd(q, k, np.abs(v), causal, w.softmax_scale, **kw)
    og = f64(bits_of(o)).reshape(o_ref.shape)
    rep = o_error_report(og, o_ref, oa_ref)
    assert rep["n_over_model"] == 0 and rep["max_abs"] <= 1e-2, rep
    assert np.abs(lse.double().cpu().numpy() - l_ref).max() <= TOL_LSE


@pytest.mark.gpu
@pytest.mark.parametrize("idx,world", [(1, 4), (2, 4), (2, 8)], ids=["S8K_ring4", "S32K_ring4",
                                                                       "S32K_ring8"])
def test_ring_forward_full_size_sampled(idx, world):
    from long_context_attention_fwd_b200 import ops
    w = I.workload(idx)
    x, o, lse = _ring_case(w, world)
    q, k, v, _, kw = oracle_args(w, x)
    rng = np.random.default_rng(idx * 10 + world)
    C = w.S // world
    rows = []
    for r in range(world):          # each rank's first / last rows and a few inside
        for i in (r * C, r * C + 1, r * C + C // 2, (r + 1) * C - 1):
            rows.append((0, int(rng.integers(w.Hq)), i))
    for _ in range(16):
        rows.append((0, int(rng.integers(w.Hq)), int(rng.integers(w.S))))
    rows = np.array(rows, dtype=np.int32)
    o_r, l_r = oracle.fwd_rows(q, k, v, w.causal, w.softmax_scale, rows, **kw)
    oa_r, _ = oracle.fwd_rows(q, k, np.abs(v), w.causal, w.softmax_scale, rows, **kw)
    og = f64(bits_of(o)).reshape(w.S, w.Hq, w.D)[rows[:, 2], rows[:, 1]]
    rep = o_error_report(og, o_r, oa_r)
    assert rep["n_over_model"] == 0 and rep["max_abs"] <= 1e-2, rep
    lg = lse.double().cpu().numpy()[0][rows[:, 1], rows[:, 2]]
    assert np.abs(lg - l_r).max() <= TOL_LSE
    # against the single-kernel forward over the whole sequence, every element
    qf = torch_bf16(x["q"]).view(w.B, w.S, w.Hq, w.D)
    kf = torch_bf16(x["k"]).view(w.B, w.S, w.Hkv, w.D)
    vf = torch_bf16(x["v"]).view(w.B, w.S, w.Hkv, w.D)
    of, lf = ops.attn_fwd(qf, kf, vf, causal=w.causal, scale=w.softmax_scale)
    torch.cuda.synchronize()
    assert (o.float() - of.float()).abs().max().item() <= 1e-2
    assert (lse - lf).abs().max().item() <= 1e-4
