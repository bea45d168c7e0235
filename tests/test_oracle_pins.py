"""Pins for the fp64 oracle: every check here compares it with something other
than itself -- hand-derived golden values, closed forms, invariants, finite
differences, and PyTorch's own fp64 attention routine on the CPU.

Each test is chosen so that a plausible slip in the oracle (a dropped scale, a
wrong sign, a transposed operand, a wrong head-group map, a causal off-by-one,
a mix-up of packed sequence offsets) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from long_context_attention_fwd_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, mult=1.0):
    return I.normal(I.stream_key(seed, 99), int(np.prod(shape))).reshape(shape) * mult


# ---------------------------------------------------------------- golden values
@pytest.mark.parametrize("fname", ["hand_s2_d1_causal.json", "hand_s2_d1_full.json"])
def test_golden_hand_derived(fname):
    g = json.load(open(os.path.join(GOLDEN, fname)))
    p = g["problem"]
    shp = (p["S"], 1, p["D"])
    q = np.array(p["q"], dtype=np.float64).reshape(shp)
    k = np.array(p["k"], dtype=np.float64).reshape(shp)
    v = np.array(p["v"], dtype=np.float64).reshape(shp)
    do = np.array(p["dO"], dtype=np.float64).reshape(shp)
    o, lse = oracle.fwd(q, k, v, p["causal"], p["scale"], B=1, S=p["S"])
    dq, dk, dv = oracle.bwd(q, k, v, do, p["causal"], p["scale"], B=1, S=p["S"])
    e = g["expected"]
    np.testing.assert_allclose(o.ravel(), e["o"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse.ravel(), e["lse"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dq.ravel(), e["dq"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk.ravel(), e["dk"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv.ravel(), e["dv"], rtol=0, atol=1e-13)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("gqa", [(2, 2), (4, 2), (6, 1)])
def test_v_ones_gives_ones(causal, gqa):
    Hq, Hkv = gqa
    S, D = 37, 8
    q = rnd((S, Hq, D), 1)
    k = rnd((S, Hkv, D), 2)
    v = np.ones((S, Hkv, D))
    o, _ = oracle.fwd(q, k, v, causal, 0.7, B=1, S=S)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_identity_values_expose_softmax_rows(causal):
    # v_j = e_j (S <= D) turns O_i into the probability row P_i.
    S, D, H = 9, 12, 2
    q = rnd((S, H, D), 3)
    k = rnd((S, H, D), 4)
    v = np.zeros((S, H, D))
    for j in range(S):
        v[j, :, j] = 1.0
    scale = 0.9
    o, lse = oracle.fwd(q, k, v, causal, scale, B=1, S=S)
    P = o[:, :, :S]  # [i, h, j]
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (P >= 0).all()
    np.testing.assert_array_equal(o[:, :, S:], 0.0)
    for i in range(S):
        for h in range(H):
            n = i + 1 if causal else S
            if causal:
                np.testing.assert_array_equal(P[i, h, n:], 0.0)
            # ratios of probabilities are exponentials of score differences
            s = scale * (k[:n, h, :] @ q[i, h, :])
            np.testing.assert_allclose(np.log(P[i, h, :n] / P[i, h, 0]), s - s[0], atol=1e-10)
            # lse is the log of the normaliser: P_ij = exp(s_ij - lse_i)
            np.testing.assert_allclose(P[i, h, :n], np.exp(s - lse[0, h, i]), rtol=1e-12)


def test_identical_keys_causal_prefix_mean():
    S, H, D = 40, 3, 8
    q = rnd((S, H, D), 5)
    kk = rnd((1, H, D), 6)
    k = np.repeat(kk, S, axis=0)
    v = rnd((S, H, D), 7)
    scale = 0.37
    o, lse = oracle.fwd(q, k, v, True, scale, B=1, S=S)
    for i in range(S):
        np.testing.assert_allclose(o[i], v[: i + 1].mean(0), rtol=0, atol=1e-12)
        for h in range(H):
            want = scale * float(q[i, h] @ kk[0, h]) + math.log(i + 1)
            assert abs(lse[0, h, i] - want) < 1e-12
    # gradients: a uniform softmax has dQ = 0, and dK sums to zero over keys
    do = rnd((S, H, D), 8)
    dq, dk, dv = oracle.bwd(q, k, v, do, True, scale, B=1, S=S)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk.sum(0), 0.0, atol=1e-11)
    # dV_j = sum_{i>=j} dO_i / (i+1)
    for j in range(S):
        want = sum(do[i] / (i + 1) for i in range(j, S))
        np.testing.assert_allclose(dv[j], want, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_scale_zero_is_mean(causal):
    S, H, D = 23, 2, 4
    q = rnd((S, H, D), 9)
    k = rnd((S, H, D), 10)
    v = rnd((S, H, D), 11)
    o, lse = oracle.fwd(q, k, v, causal, 0.0, B=1, S=S)
    for i in range(S):
        n = i + 1 if causal else S
        np.testing.assert_allclose(o[i], v[:n].mean(0), atol=1e-12)
        np.testing.assert_allclose(lse[0, :, i], math.log(n), atol=1e-12)


def test_single_token():
    Hq, Hkv, D = 4, 2, 8
    q = rnd((1, Hq, D), 12)
    k = rnd((1, Hkv, D), 13)
    v = rnd((1, Hkv, D), 14)
    do = rnd((1, Hq, D), 15)
    scale = 0.5
    o, lse = oracle.fwd(q, k, v, True, scale, B=1, S=1)
    dq, dk, dv = oracle.bwd(q, k, v, do, True, scale, B=1, S=1)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        np.testing.assert_allclose(o[0, h], v[0, g], atol=1e-14)
        assert abs(lse[0, h, 0] - scale * float(q[0, h] @ k[0, g])) < 1e-13
    np.testing.assert_allclose(dq, 0.0, atol=1e-14)
    np.testing.assert_allclose(dk, 0.0, atol=1e-14)
    for g in range(Hkv):
        np.testing.assert_allclose(dv[0, g], do[0, 2 * g] + do[0, 2 * g + 1], atol=1e-14)


# ---------------------------------------------------------------- structure
@pytest.mark.parametrize("causal", [True, False])
def test_gqa_equals_mha_with_repeated_kv(causal):
    S, Hq, Hkv, D = 19, 6, 2, 8
    G = Hq // Hkv
    q, k, v, do = rnd((S, Hq, D), 16), rnd((S, Hkv, D), 17), rnd((S, Hkv, D), 18), rnd((S, Hq, D), 19)
    kr, vr = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)  # head h reads kv head h // G
    o1, l1 = oracle.fwd(q, k, v, causal, 0.3, B=1, S=S)
    o2, l2 = oracle.fwd(q, kr, vr, causal, 0.3, B=1, S=S)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)
    dq1, dk1, dv1 = oracle.bwd(q, k, v, do, causal, 0.3, B=1, S=S)
    dq2, dk2, dv2 = oracle.bwd(q, kr, vr, do, causal, 0.3, B=1, S=S)
    np.testing.assert_allclose(dq1, dq2, atol=1e-12)
    np.testing.assert_allclose(dk1, dk2.reshape(S, Hkv, G, D).sum(2), atol=1e-12)
    np.testing.assert_allclose(dv1, dv2.reshape(S, Hkv, G, D).sum(2), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_packed_equals_separate(causal):
    lens = [5, 0, 13, 1, 9]
    Hq, Hkv, D = 4, 2, 8
    T = sum(lens)
    q, k, v, do = rnd((T, Hq, D), 20), rnd((T, Hkv, D), 21), rnd((T, Hkv, D), 22), rnd((T, Hq, D), 23)
    cu = I.cu_seqlens_from(lens)
    o, lse = oracle.fwd(q, k, v, causal, 0.4, cu_seqlens=cu)
    dq, dk, dv = oracle.bwd(q, k, v, do, causal, 0.4, cu_seqlens=cu)
    for s, L in enumerate(lens):
        a, b = cu[s], cu[s + 1]
        if L == 0:
            continue
        o1, l1 = oracle.fwd(q[a:b], k[a:b], v[a:b], causal, 0.4, B=1, S=L)
        g1 = oracle.bwd(q[a:b], k[a:b], v[a:b], do[a:b], causal, 0.4, B=1, S=L)
        assert np.array_equal(o[a:b], o1)
        assert np.array_equal(lse[:, a:b], l1[0])
        assert np.array_equal(dq[a:b], g1[0])
        assert np.array_equal(dk[a:b], g1[1])
        assert np.array_equal(dv[a:b], g1[2])


def test_batch_equals_separate():
    B, S, H, D = 3, 11, 2, 4
    q, k, v = rnd((B * S, H, D), 24), rnd((B * S, H, D), 25), rnd((B * S, H, D), 26)
    o, lse = oracle.fwd(q, k, v, True, 0.5, B=B, S=S)
    for b in range(B):
        sl = slice(b * S, (b + 1) * S)
        o1, l1 = oracle.fwd(q[sl], k[sl], v[sl], True, 0.5, B=1, S=S)
        assert np.array_equal(o[sl], o1)
        assert np.array_equal(lse[b], l1[0])


def test_noncausal_key_permutation_invariance():
    S, H, D = 17, 2, 8
    q, k, v = rnd((S, H, D), 27), rnd((S, H, D), 28), rnd((S, H, D), 29)
    perm = np.random.default_rng(0).permutation(S)
    o1, l1 = oracle.fwd(q, k, v, False, 0.6, B=1, S=S)
    o2, l2 = oracle.fwd(q, k[perm], v[perm], False, 0.6, B=1, S=S)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_causal_row_ignores_future_keys():
    # Changing keys/values after position i leaves rows <= i untouched.
    S, H, D = 16, 2, 4
    q, k, v = rnd((S, H, D), 30), rnd((S, H, D), 31), rnd((S, H, D), 32)
    o1, l1 = oracle.fwd(q, k, v, True, 0.5, B=1, S=S)
    k2, v2 = k.copy(), v.copy()
    k2[9:] += 3.0
    v2[9:] -= 2.0
    o2, l2 = oracle.fwd(q, k2, v2, True, 0.5, B=1, S=S)
    assert np.array_equal(o1[:9], o2[:9])
    assert not np.allclose(o1[9:], o2[9:])


# ---------------------------------------------------------------- gradients
@pytest.mark.parametrize("causal", [True, False])
def test_finite_differences(causal):
    S, Hq, Hkv, D = 7, 4, 2, 3
    scale = 0.8
    q, k, v, do = rnd((S, Hq, D), 33), rnd((S, Hkv, D), 34), rnd((S, Hkv, D), 35), rnd((S, Hq, D), 36)

    def loss(q_, k_, v_):
        o, _ = oracle.fwd(q_, k_, v_, causal, scale, B=1, S=S)
        return float((o * do).sum())

    dq, dk, dv = oracle.bwd(q, k, v, do, causal, scale, B=1, S=S)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (loss(args_p["q"], args_p["k"], args_p["v"])
                       - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
        rel = np.linalg.norm(fd - g) / np.linalg.norm(g)
        assert rel < 1e-6, (name, rel)


# ---------------------------------------------------------------- library routine
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("gqa", [(4, 4), (6, 2)])
def test_matches_torch_sdpa_fp64(causal, gqa):
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    S, D = 33, 16
    Hq, Hkv = gqa
    scale = 0.21
    q, k, v, do = rnd((S, Hq, D), 37), rnd((S, Hkv, D), 38), rnd((S, Hkv, D), 39), rnd((S, Hq, D), 40)
    tq = torch.tensor(q).permute(1, 0, 2)[None].requires_grad_(True)
    tk = torch.tensor(k).permute(1, 0, 2)[None].requires_grad_(True)
    tv = torch.tensor(v).permute(1, 0, 2)[None].requires_grad_(True)
    to = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale,
                                        enable_gqa=Hq != Hkv)
    to.backward(torch.tensor(do).permute(1, 0, 2)[None])
    o, lse = oracle.fwd(q, k, v, causal, scale, B=1, S=S)
    dq, dk, dv = oracle.bwd(q, k, v, do, causal, scale, B=1, S=S)
    np.testing.assert_allclose(o, to[0].permute(1, 0, 2).detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad[0].permute(1, 0, 2).numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad[0].permute(1, 0, 2).numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad[0].permute(1, 0, 2).numpy(), atol=1e-11)
    # logsumexp against torch's own reduction of the masked score matrix
    s = torch.einsum("qhd,khd->hqk", torch.tensor(q),
                     torch.tensor(np.repeat(k, Hq // Hkv, axis=1))) * scale
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(S, S, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse[0], torch.logsumexp(s, -1).numpy(), atol=1e-12)


# ---------------------------------------------------------------- brute force
def _brute_force_long_double(q, k, v, causal, scale, B, S):
    """The definition written out element by element in extended precision
    (np.longdouble), with no maximum subtracted before exponentiating:
    O_i = sum_j exp(s_ij) v_j / sum_j exp(s_ij), LSE_i = ln sum_j exp(s_ij), over the keys
    j the mask lets row i see, s_ij = scale * q_i . k_j, query head h reading kv head
    h // (Hq / Hkv)."""
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    ld = np.longdouble
    o = np.zeros((T, Hq, D), dtype=ld)
    lse = np.zeros((B, Hq, S), dtype=ld)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(S):
                ti = b * S + i
                den = ld(0)
                num = np.zeros(D, dtype=ld)
                for j in range(S if not causal else i + 1):
                    tj = b * S + j
                    s = ld(scale) * sum(ld(q[ti, h, d]) * ld(k[tj, g, d]) for d in range(D))
                    e = np.exp(s)
                    den += e
                    num += e * v[tj, g].astype(ld)
                o[ti, h] = num / den
                lse[b, h, i] = np.log(den)
    return o, lse


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("shape", [(1, 4, 4, 32, 8), (2, 6, 2, 13, 3)],
                         ids=["B1_mha4_S32_D8", "B2_gqa6x2_S13_D3"])
def test_brute_force_long_double(causal, shape):
    B, Hq, Hkv, S, D = shape
    scale = 0.37
    q, k, v = rnd((B * S, Hq, D), 51), rnd((B * S, Hkv, D), 52), rnd((B * S, Hkv, D), 53)
    o, lse = oracle.fwd(q, k, v, causal, scale, B=B, S=S)
    o_bf, lse_bf = _brute_force_long_double(q, k, v, causal, scale, B, S)
    assert np.abs(o - o_bf.astype(np.float64)).max() <= 1e-12
    assert np.abs(lse - lse_bf.astype(np.float64)).max() <= 1e-12


# ---------------------------------------------------------------- row APIs
def test_row_apis_agree_with_full():
    lens = [70, 3, 45]
    Hq, Hkv, D = 4, 2, 8
    T = sum(lens)
    cu = I.cu_seqlens_from(lens)
    q, k, v, do = rnd((T, Hq, D), 41), rnd((T, Hkv, D), 42), rnd((T, Hkv, D), 43), rnd((T, Hq, D), 44)
    o, lse = oracle.fwd(q, k, v, True, 0.3, cu_seqlens=cu)
    dq, dk, dv = oracle.bwd(q, k, v, do, True, 0.3, cu_seqlens=cu)
    rows = [(0, 1, 69), (1, 3, 2), (2, 0, 0), (2, 2, 44), (0, 0, 0)]
    orow, lrow = oracle.fwd_rows(q, k, v, True, 0.3, rows, cu_seqlens=cu)
    dqr, lr2, _ = oracle.bwd_dq_rows(q, k, v, do, True, 0.3, rows, cu_seqlens=cu)
    for n, (b, h, i) in enumerate(rows):
        t = cu[b] + i
        assert np.array_equal(orow[n], o[t, h])
        assert lrow[n] == lse[h, t] == lr2[n]
        np.testing.assert_allclose(dqr[n], dq[t, h], atol=1e-13)
    dk2, dv2 = oracle.bwd_dkdv_range(q, k, v, do, True, 0.3, b=2, g=1, j0=30, j1=45, cu_seqlens=cu)
    np.testing.assert_allclose(dk2, dk[cu[2] + 30: cu[2] + 45, 1], atol=1e-13)
    np.testing.assert_allclose(dv2, dv[cu[2] + 30: cu[2] + 45, 1], atol=1e-13)


def test_rejects_bad_arguments():
    q = np.zeros((4, 3, 2))
    k = np.zeros((4, 2, 2))
    with pytest.raises(ValueError):
        oracle.fwd(q, k, k, True, 1.0, B=1, S=4)  # Hq % Hkv != 0
    with pytest.raises(ValueError):
        oracle.fwd(np.zeros((4, 2, 2)), k, k, True, 1.0, cu_seqlens=np.array([0, 3, 2], np.int32))


# ---------------------------------------------------------------- partial merge
def _chunk_partials(q, k, v, bounds, scale):
    """Non-causal attention of every query over each key chunk: the partials a ring of
    devices holding those chunks would produce."""
    S, H, D = q.shape
    parts_o, parts_l = [], []
    for a, b in bounds:
        o = np.zeros((S, H, D))
        lse = np.zeros((H, S))
        for h in range(H):
            s_ = scale * q[:, h, :] @ k[a:b, h, :].T          # [S, L]
            m = s_.max(1, keepdims=True)
            e = np.exp(s_ - m)
            o[:, h, :] = (e / e.sum(1, keepdims=True)) @ v[a:b, h, :]
            lse[h] = (m[:, 0] + np.log(e.sum(1)))
        parts_o.append(o.reshape(S * H, D))
        parts_l.append(lse.T.reshape(S * H))
    return parts_o, parts_l


def test_merge_of_key_chunks_equals_full_attention():
    S, H, D = 40, 2, 8
    q, k, v = rnd((S, H, D), 60), rnd((S, H, D), 61), rnd((S, H, D), 62)
    po, pl = _chunk_partials(q, k, v, [(0, 7), (7, 25), (25, 40)], 0.4)
    o, lse = oracle.merge_partials(po, pl)
    of, lf = oracle.fwd(q, k, v, False, 0.4, B=1, S=S)          # oracle over all keys
    np.testing.assert_allclose(o.reshape(S, H, D), of, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(S, H).T, lf[0], atol=1e-12)


def test_merge_special_cases():
    r = np.random.default_rng(3)
    o1 = r.standard_normal((5, 4))
    l1 = r.standard_normal(5)
    o, l = oracle.merge_partials([o1], [l1])                   # one partial: identity
    np.testing.assert_allclose(o, o1, atol=1e-15)
    np.testing.assert_allclose(l, l1, atol=1e-15)
    ninf = np.full(5, -np.inf)
    o, l = oracle.merge_partials([o1, 7 * o1], [l1, ninf])      # -inf partial: ignored
    np.testing.assert_allclose(o, o1, atol=1e-15)
    o, l = oracle.merge_partials([o1, o1], [ninf, ninf])        # nothing visible
    assert (o == 0).all() and np.isneginf(l).all()
    o, l = oracle.merge_partials([o1, 3 * o1], [l1, l1])        # equal weights: mean
    np.testing.assert_allclose(o, 2 * o1, atol=1e-14)
    np.testing.assert_allclose(l, l1 + np.log(2), atol=1e-14)


# ---------------------------------------------------------------- decode over a cache
def _decode_problem(B, Hq, Hkv, Lmax, D, seed):
    q = rnd((B, Hq, D), seed)
    k = rnd((B, Lmax, Hkv, D), seed + 1)
    v = rnd((B, Lmax, Hkv, D), seed + 2)
    return q, k, v


def test_decode_matches_torch_sdpa():
    torch = pytest.importorskip("torch")
    B, Hq, Hkv, Lmax, D = 3, 6, 2, 23, 8
    q, k, v = _decode_problem(B, Hq, Hkv, Lmax, D, 70)
    lens = np.array([23, 1, 9], dtype=np.int32)
    o, lse = oracle.decode(q, k, v, lens, 0.45)
    G = Hq // Hkv
    for b in range(B):
        L = lens[b]
        for h in range(Hq):
            qt = torch.from_numpy(q[b, h]).view(1, 1, 1, D)
            kt = torch.from_numpy(k[b, :L, h // G]).view(1, 1, L, D)
            vt = torch.from_numpy(v[b, :L, h // G]).view(1, 1, L, D)
            ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=0.45)
            np.testing.assert_allclose(o[b, h], ref.view(D).numpy(), atol=1e-13)
            want = torch.logsumexp(0.45 * (kt.view(L, D) @ qt.view(D)), 0).item()
            assert abs(lse[b, h] - want) < 1e-12


def test_decode_closed_forms():
    B, Hq, Hkv, Lmax, D = 4, 4, 2, 17, 4
    q, k, v = _decode_problem(B, Hq, Hkv, Lmax, D, 80)
    lens = np.array([17, 5, 1, 0], dtype=np.int32)
    o, _ = oracle.decode(q, k, np.ones_like(v), lens, 0.3)          # V = ones
    np.testing.assert_allclose(o[:3], 1.0, atol=1e-13)
    assert (o[3] == 0).all()
    kk = np.repeat(k[:, :1], Lmax, axis=1)                              # identical keys
    o, lse = oracle.decode(q, kk, v, lens, 0.3)
    for b in range(3):
        L = lens[b]
        for h in range(Hq):
            g = h // 2
            np.testing.assert_allclose(o[b, h], v[b, :L, g].mean(0), atol=1e-13)
            assert abs(lse[b, h] - (0.3 * q[b, h] @ kk[b, 0, g] + math.log(L))) < 1e-12
    o, lse = oracle.decode(q, k, v, lens, 0.3)                          # one key, no key
    for h in range(Hq):
        np.testing.assert_allclose(o[2, h], v[2, 0, h // 2], atol=1e-14)
        assert abs(lse[2, h] - 0.3 * q[2, h] @ k[2, 0, h // 2]) < 1e-13
    assert (o[3] == 0).all() and np.isneginf(lse[3]).all()


def test_decode_gqa_and_ignores_entries_past_the_length():
    B, Hq, Hkv, Lmax, D = 2, 6, 2, 11, 4
    q, k, v = _decode_problem(B, Hq, Hkv, Lmax, D, 90)
    lens = np.array([7, 11], dtype=np.int32)
    o1, l1 = oracle.decode(q, k, v, lens, 0.5)
    o2, l2 = oracle.decode(q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), lens, 0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)
    k2, v2 = k.copy(), v.copy()
    k2[0, 7:], v2[0, 7:] = 1e30, np.nan
    o3, l3 = oracle.decode(q, k2, v2, lens, 0.5)
    assert np.array_equal(o1, o3) and np.array_equal(l1, l3)


# ---------------------------------------------------------------- e4m3 helper used by the fp8 tests
def test_e4m3_helper_against_the_format():
    import e4m3
    # every finite code decodes to a value that quantises back to itself
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = e4m3.decode(codes)
    np.testing.assert_array_equal(e4m3.quantize(vals), vals)
    assert e4m3.decode(np.array([0x7E], np.uint8))[0] == 448.0          # largest finite
    assert e4m3.decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9      # smallest subnormal
    assert e4m3.decode(np.array([0x08], np.uint8))[0] == 2.0 ** -6      # smallest normal
    assert np.isnan(e4m3.decode(np.array([0x7F], np.uint8))[0])
    # ties go to the even mantissa; saturation at 448
    assert e4m3.quantize(1.0 + 1.0 / 16) == 1.0           # halfway 1.0 / 1.125 -> even (1.0)
    assert e4m3.quantize(1.0 + 3.0 / 16) == 1.25          # halfway 1.125 / 1.25 -> even (1.25)
    assert e4m3.quantize(1000.0) == 448.0 and e4m3.quantize(-1000.0) == -448.0
    assert e4m3.quantize(2.0 ** -10) == 0.0               # halfway 0 / 2^-9 -> even (0)
    # encoding is the inverse of decoding on every finite code (except -0 -> +0)
    enc = e4m3.encode(vals)
    assert all(a == b or (a == 0x80 and b == 0) for a, b in zip(codes, enc))


# ---------------------------------------------------------------- block-pair backward (Ring)
def test_bwd_given_block_pairs_sum_to_torch_autograd():
    torch = pytest.importorskip("torch")
    C, Hq, Hkv, D, scale = 9, 4, 2, 4, 0.6
    S = 2 * C
    q, k, v, do = rnd((S, Hq, D), 101), rnd((S, Hkv, D), 102), rnd((S, Hkv, D), 103), rnd((S, Hq, D), 104)
    o, lse = oracle.fwd(q, k, v, True, scale, B=1, S=S)          # statistics of the whole rows
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    for r in range(2):                                           # query block r
        qs = slice(r * C, (r + 1) * C)
        for j in range(r + 1):                                   # key blocks it sees
            ks = slice(j * C, (j + 1) * C)
            gq, gk, gv = oracle.bwd_given(q[qs], k[ks], v[ks], o[qs], lse[:, :, qs], do[qs],
                                          j == r, scale, B=1, S=C)
            dq[qs] += gq; dk[ks] += gk; dv[ks] += gv
    G = Hq // Hkv
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    kk = tk.repeat_interleave(G, dim=1); vv = tv.repeat_interleave(G, dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(
        tq.permute(1, 0, 2)[None], kk.permute(1, 0, 2)[None], vv.permute(1, 0, 2)[None],
        is_causal=True, scale=scale)[0].permute(1, 0, 2)
    out.backward(torch.tensor(do))
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)
