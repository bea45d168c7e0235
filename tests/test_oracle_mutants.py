"""Mutation tests for the oracle's pins: each mutant is a copy of oracle/attn_oracle.c
with one plausible mistake planted in it (on the CPU, in a temporary build).  The pin
suite below -- the same kinds of checks as test_oracle_pins.py -- must pass on the real
oracle and fail on every mutant, which shows the pins can tell a correct oracle from
a subtly wrong one."""
import json
import math
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from long_context_attention_fwd_b200 import inputs as I

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "attn_oracle.c")

MUTANTS = {
    "dropped_scale": ("s[j] = p->scale * acc;", "s[j] = acc;"),
    "gqa_map_modulo": ("const int g = h / (p->Hq / p->Hkv);\n    const int D = p->D;\n    const int n = visible(p, L, i);\n    const double *qi",
                       "const int g = h % p->Hkv;\n    const int D = p->D;\n    const int n = visible(p, L, i);\n    const double *qi"),
    "causal_off_by_one": ("return p->causal ? i + 1 : L;", "return p->causal ? (i > 0 ? i : 1) : L;"),
    "dk_missing_scale": ("for (int d = 0; d < D; ++d) dk_row[d] *= p->scale;", ""),
    "ds_sign_flipped": ("const double ds = pij * (dp - delta_g[(int64_t)hh * L + i]);",
                        "const double ds = pij * (delta_g[(int64_t)hh * L + i] - dp);"),
    "dv_wrong_operand": ("dv_row[d] += pij * doi[d];", "dv_row[d] += pij * qi[d];"),
    "lse_without_max": ("*lse_out = m + log(sum);", "*lse_out = log(sum);"),
    "merge_weight_unnormalised": ("const double w = exp(lse_parts[p][r] - L);",
                                  "const double w = exp(lse_parts[p][r] - m);"),
    "merge_lse_without_max": ("const double L = m + log(sum);", "const double L = log(sum);"),
    "decode_drops_last_key": ("const int L = cache_len[b];", "const int L = cache_len[b] > 1 ? cache_len[b] - 1 : cache_len[b];"),
    "bwd_given_ignores_lse": ("const double p = exp(scale * s - L);", "const double p = exp(scale * s);"),
    "decode_gqa_map_modulo": ("const int b = (int)(r / Hq), h = (int)(r % Hq), g = h / G;",
                              "const int b = (int)(r / Hq), h = (int)(r % Hq), g = h % Hkv;"),
}


def _rnd(shape, seed):
    return I.normal(I.stream_key(seed, 77), int(np.prod(shape))).reshape(shape)


def _pin_suite() -> list:
    """Names of the pins that fail on the currently loaded oracle build."""
    failed = []
    # hand-derived golden values (forward and every gradient)
    for fname in ("hand_s2_d1_causal.json", "hand_s2_d1_full.json"):
        g = json.load(open(os.path.join(HERE, "golden", fname)))
        p = g["problem"]
        shp = (p["S"], 1, p["D"])
        q, k, v, do = (np.array(p[n], dtype=np.float64).reshape(shp) for n in ("q", "k", "v", "dO"))
        try:
            o, lse = oracle.fwd(q, k, v, p["causal"], p["scale"], B=1, S=p["S"])
            dq, dk, dv = oracle.bwd(q, k, v, do, p["causal"], p["scale"], B=1, S=p["S"])
            e = g["expected"]
            for got, want in ((o, e["o"]), (lse, e["lse"]), (dq, e["dq"]), (dk, e["dk"]), (dv, e["dv"])):
                if not np.allclose(got.ravel(), want, rtol=0, atol=1e-12):
                    failed.append("golden:" + fname)
                    break
        except ValueError:
            failed.append("golden:" + fname)
    # GQA equals MHA with repeated K/V
    S, Hq, Hkv, D = 9, 4, 2, 4
    q, k, v, do = _rnd((S, Hq, D), 1), _rnd((S, Hkv, D), 2), _rnd((S, Hkv, D), 3), _rnd((S, Hq, D), 4)
    o1, _ = oracle.fwd(q, k, v, True, 0.5, B=1, S=S)
    o2, _ = oracle.fwd(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1), True, 0.5, B=1, S=S)
    if not np.allclose(o1, o2, atol=1e-12):
        failed.append("gqa")
    # identical keys: causal prefix mean and LSE = s + ln(i+1)
    kk = np.repeat(_rnd((1, Hq, D), 5), S, axis=0)
    o, lse = oracle.fwd(q, kk, kk, True, 0.5, B=1, S=S)
    vv = kk
    for i in range(S):
        if not np.allclose(o[i], vv[: i + 1].mean(0), atol=1e-12):
            failed.append("prefix_mean")
            break
    for i in range(S):
        if abs(lse[0, 0, i] - (0.5 * float(q[i, 0] @ kk[0, 0]) + math.log(i + 1))) > 1e-12:
            failed.append("lse_closed_form")
            break
    # merging the partials over key chunks gives the attention over all keys (partials
    # computed here with numpy, non-causal, one chunk at a time)
    S3, H3, D3 = 12, 2, 4
    q, k, v = _rnd((S3, H3, D3), 11), _rnd((S3, H3, D3), 12), _rnd((S3, H3, D3), 13)
    po, pl = [], []
    for a, b in ((0, 5), (5, 12)):
        s_ = 0.6 * np.einsum("ihd,jhd->hij", q, k[a:b])
        mx = s_.max(-1, keepdims=True)
        e = np.exp(s_ - mx)
        po.append(np.einsum("hij,jhd->ihd", e / e.sum(-1, keepdims=True), v[a:b]).reshape(-1, D3))
        pl.append((mx[..., 0] + np.log(e.sum(-1))).T.reshape(-1))
    om, lm = oracle.merge_partials(po, pl)
    of, lf = oracle.fwd(q, k, v, False, 0.6, B=1, S=S3)
    if not (np.allclose(om.reshape(of.shape), of, atol=1e-12)
            and np.allclose(lm.reshape(S3, H3).T, lf[0], atol=1e-12)):
        failed.append("merge_equals_full")
    # decode: one query over a cache equals the oracle's causal attention for the last
    # row of a sequence whose last query is that token (computed here directly in numpy)
    Lc, Hq4, Hkv4, D4 = 9, 4, 2, 4
    qd, kc, vc = _rnd((1, Hq4, D4), 21), _rnd((1, Lc, Hkv4, D4), 22), _rnd((1, Lc, Hkv4, D4), 23)
    od, ld = oracle.decode(qd, kc, vc, np.array([Lc], dtype=np.int32), 0.8)
    ok = True
    for h in range(Hq4):
        g = h // (Hq4 // Hkv4)
        s_ = 0.8 * kc[0, :, g] @ qd[0, h]
        e = np.exp(s_ - s_.max())
        ok &= np.allclose(od[0, h], (e / e.sum()) @ vc[0, :, g], atol=1e-12)
        ok &= abs(ld[0, h] - (s_.max() + np.log(e.sum()))) < 1e-12
    if not ok:
        failed.append("decode_direct")
    # block-pair backward with the whole rows' statistics: the two-block causal split sums
    # to PyTorch's fp64 autograd of the whole attention
    try:
        import torch
        C, Hq5, Hkv5, D5, sc = 5, 2, 1, 3, 0.7
        S5 = 2 * C
        q5, k5, v5, do5 = _rnd((S5, Hq5, D5), 31), _rnd((S5, Hkv5, D5), 32), _rnd((S5, Hkv5, D5), 33), _rnd((S5, Hq5, D5), 34)
        o5, l5 = oracle.fwd(q5, k5, v5, True, sc, B=1, S=S5)
        g = [np.zeros_like(q5), np.zeros_like(k5), np.zeros_like(v5)]
        for r in range(2):
            qs = slice(r * C, (r + 1) * C)
            for j in range(r + 1):
                ks = slice(j * C, (j + 1) * C)
                a, b_, c_ = oracle.bwd_given(q5[qs], k5[ks], v5[ks], o5[qs], l5[:, :, qs], do5[qs], j == r, sc, B=1, S=C)
                g[0][qs] += a; g[1][ks] += b_; g[2][ks] += c_
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q5, k5, v5))
        out = torch.nn.functional.scaled_dot_product_attention(
            tq.permute(1, 0, 2)[None], tk.repeat_interleave(2, 1).permute(1, 0, 2)[None],
            tv.repeat_interleave(2, 1).permute(1, 0, 2)[None], is_causal=True, scale=sc)[0].permute(1, 0, 2)
        out.backward(torch.tensor(do5))
        if not all(np.allclose(a, b_.grad.numpy(), atol=1e-10) for a, b_ in zip(g, (tq, tk, tv))):
            failed.append("bwd_given_sum")
    except ValueError:
        failed.append("bwd_given_sum")
    # finite differences of L = sum(dO * O)
    S2 = 5
    q, k, v, do = _rnd((S2, 2, 3), 6), _rnd((S2, 1, 3), 7), _rnd((S2, 1, 3), 8), _rnd((S2, 2, 3), 9)
    dq, dk, dv = oracle.bwd(q, k, v, do, True, 0.7, B=1, S=S2)
    h = 1e-6
    for name, x, gr in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            args = {"q": q, "k": k, "v": v}
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args[name] = xp
            lp = float((oracle.fwd(args["q"], args["k"], args["v"], True, 0.7, B=1, S=S2)[0] * do).sum())
            args[name] = xm
            lm = float((oracle.fwd(args["q"], args["k"], args["v"], True, 0.7, B=1, S=S2)[0] * do).sum())
            fd[idx] = (lp - lm) / (2 * h)
        if not np.linalg.norm(fd - gr) <= 1e-6 * max(np.linalg.norm(gr), 1e-30):
            failed.append("fd:" + name)
    return failed


def _build_mutant(tmp: str, name: str) -> str:
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site of {name} not found"
    src = src.replace(old, new, 1)
    c = os.path.join(tmp, f"{name}.c")
    so = os.path.join(tmp, f"{name}.so")
    open(c, "w").write(src)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", so, c, "-lm"], check=True)
    return so


def test_real_oracle_passes_the_suite():
    oracle.use_library(None)
    assert _pin_suite() == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_is_caught(name):
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(tmp, name)
        try:
            oracle.use_library(so)
            with np.errstate(all="ignore"):
                failed = _pin_suite()
        finally:
            oracle.use_library(None)
    assert failed, f"mutant {name} passed every pin"
