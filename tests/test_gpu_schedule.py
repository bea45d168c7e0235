"""The backward's CTA orders, checked against the fp64 oracle.

The backward enumerates (sequence, kv head, 128-key tile) work items in one of two
orders.  Dense batches whose kv group has at least as many tiles as the GPU has SMs
take the group-major order, with the batch's sequences innermost inside a group; all
other problems keep the kv head innermost.  These cases are sized to land on each
side of that threshold, with ragged sequence ends (S not a multiple of 128), several
sequences and several kv groups, so a wrong mapping from block index to work item
(a missed or repeated tile, a wrong sequence start) would show up as wrong dK/dV/dQ
rows.  Whole (sequence, kv head) slices are compared, every element.
"""
import numpy as np
import pytest

import oracle
from helpers import TOL_GRAD, TOL_LSE, DeviceRun, make_case, o_error_report, rel_l2
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")

# (name, case, whether the group-major order applies on a 148-SM B200)
CASES = [
    # 7 sequences of 2999 tokens: (7 * 2999) >> 7 = 164, + 7 = 171 tiles a group >= 148.
    ("gqa4x2_B7_S2999_D64_causal", make_case(7, 4, 2, 2999, 64, True, seed=31), True),
    ("gqa4x2_B7_S2999_D64_full", make_case(7, 4, 2, 2999, 64, False, seed=32), True),
    # 3 sequences of 1000 tokens: 23 + 3 = 26 tiles a group < 148: kv head innermost.
    ("gqa6x3_B3_S1000_D128_causal", make_case(3, 6, 3, 1000, 128, True, seed=33), False),
]


def _slice(t, b, S, heads):
    return np.ascontiguousarray(t[b * S:(b + 1) * S, heads])


@pytest.mark.gpu
@pytest.mark.parametrize("name,w,group_major", CASES, ids=[c[0] for c in CASES])
def test_backward_orders(name, w, group_major):
    G = w.Hq // w.Hkv
    ntile = (w.B * w.S >> 7) + w.B
    assert (ntile >= 148) == group_major, "case no longer lands on its side of the threshold"
    run = DeviceRun(w)
    g = run.np_out()
    q, k, v, do = (I.bf16_bits_to_f64(run.x[n]) for n in ("q", "k", "v", "do"))
    # first, middle and last sequence; first and last kv head
    for b, gh in ((0, 0), (w.B // 2, w.Hkv - 1), (w.B - 1, w.Hkv - 1)):
        hq = list(range(gh * G, (gh + 1) * G))
        qs, ds = _slice(q, b, w.S, hq), _slice(do, b, w.S, hq)
        ks, vs = _slice(k, b, w.S, [gh]), _slice(v, b, w.S, [gh])
        o_r, lse_r = oracle.fwd(qs, ks, vs, w.causal, w.softmax_scale, B=1, S=w.S)
        oa_r, _ = oracle.fwd(qs, ks, np.abs(vs), w.causal, w.softmax_scale, B=1, S=w.S)
        dq_r, dk_r, dv_r = oracle.bwd(qs, ks, vs, ds, w.causal, w.softmax_scale, B=1, S=w.S)
        rows = slice(b * w.S, (b + 1) * w.S)
        rep = o_error_report(g["o"][rows][:, hq], o_r, oa_r)
        assert rep["max_abs"] <= 1e-2 and rep["n_over_model"] == 0, (b, gh, rep)
        assert float(np.abs(g["lse"][b, hq] - lse_r[0]).max()) <= TOL_LSE
        assert rel_l2(g["dq"][rows][:, hq], dq_r) <= TOL_GRAD, (b, gh)
        assert rel_l2(g["dk"][rows][:, [gh]], dk_r) <= TOL_GRAD, (b, gh)
        assert rel_l2(g["dv"][rows][:, [gh]], dv_r) <= TOL_GRAD, (b, gh)
    # every key row of every (sequence, kv head) was written: no NaN left from the
    # poisoned outputs, and dV sums to the group's dO over the sequence
    for t in ("dq", "dk", "dv"):
        assert np.isfinite(g[t]).all(), t
    for b in range(w.B):
        rows = slice(b * w.S, (b + 1) * w.S)
        want = do[rows].reshape(w.S, w.Hkv, G, w.D).sum((0, 2))
        assert rel_l2(g["dv"][rows].sum(0), want) <= 1e-2, b
