"""Full-size workloads (8K and 32K causal GQA, packed 32K, MHA D=64 with outliers) in
the launch configuration the bench times, checked against the fp64 oracle on
sampled outputs it can compute one by one, plus properties that hold at any size:

  * O and LSE of sampled query rows (first/last rows, tile edges, random rows);
  * dQ of the same sampled query rows;
  * multi-head workloads: dQ, dK, dV over two whole (sequence, head) slices;
    grouped-query workloads: dK, dV of the FIRST 256 keys of the first and last kv
    head (of the longest sequence when packed) -- every query row after them sees
    those keys, so these are the longest reductions the kernel makes (at 32K, 7 heads x
    256 query tiles accumulate into one key tile) -- and of the last keys of sampled
    (sequence, kv head) pairs;
  * over ALL keys of every (sequence, kv head): sum_j dV_j equals the sum of dO over
    the group's heads and rows (each probability row sums to one), and sum_j dK_j is
    zero (each row of dS sums to zero) -- both up to bf16 rounding of P and dS.

The Qwen2.5-7B-shaped 8K workload is also compared whole: every element of O and LSE,
and dQ, dK, dV by relative L2 over the whole tensors (the stated metric), against the
oracle's full forward and backward.
"""
import numpy as np
import pytest

import oracle
from helpers import (TOL_GRAD, TOL_LSE, TOL_O, DeviceRun, o_error_report, oracle_args, record,
                     rel_l2, row_dispersion)
from long_context_attention_fwd_b200 import inputs as I

torch = pytest.importorskip("torch")


def _sample_rows(w, rng, n_random=24):
    lens = w.seq_lengths()
    rows = []
    for _ in range(n_random):
        b = int(rng.integers(len(lens)))
        while lens[b] == 0:
            b = int(rng.integers(len(lens)))
        rows.append((b, int(rng.integers(w.Hq)), int(rng.integers(lens[b]))))
    for b, L in enumerate(lens[:3]):
        for i in (0, 1, 127, 128, 255, 256, L // 2, L - 129, L - 128, L - 1):
            if 0 <= i < L:
                rows.append((b, int(rng.integers(w.Hq)), int(i)))
    return np.array(rows, dtype=np.int32)


@pytest.mark.gpu
@pytest.mark.parametrize("idx", [1, 2, 3, 4], ids=["S8K", "S32K", "varlen32K", "mha_D64_outliers"])
def test_full_size_sampled(idx):
    w = I.workload(idx)
    run = DeviceRun(w, poison=False)
    g = run.np_out()
    q, k, v, do, kw = oracle_args(w, run.x)
    rng = np.random.default_rng(100 + idx)
    cu = I.cu_seqlens_from(w.seq_lengths())
    lens = w.seq_lengths()

    # ---- forward rows
    rows = _sample_rows(w, rng)
    o_r, lse_r = oracle.fwd_rows(q, k, v, w.causal, w.softmax_scale, rows, **kw)
    oa_r, _ = oracle.fwd_rows(q, k, np.abs(v), w.causal, w.softmax_scale, rows, **kw)
    t = cu[rows[:, 0]] + rows[:, 2]
    o_g = g["o"][t, rows[:, 1]]
    if w.varlen is None:
        lse_g = g["lse"][rows[:, 0], rows[:, 1], rows[:, 2]]
    else:
        lse_g = g["lse"][rows[:, 1], t]
    disp = row_dispersion(q, k, v, o_r, lambda r: tuple(int(x) for x in rows[r]), w.causal,
                          w.softmax_scale, cu)
    rep = o_error_report(o_g, o_r, oa_r, nkeys=max(lens), disp=disp)
    lse_err = float(np.abs(lse_g - lse_r).max())
    figures = record(f"full_size/{w.name}", o_rows=len(rows), o_max_abs=rep["max_abs"],
                     o_n_over_1e_2=rep["n_over_strict"], o_n_over_bound=rep["n_over_model"],
                     o_over=rep["over"], lse_max_abs=lse_err)
    # every element above the stated 1e-2 must lie within its derived rounding bound
    assert rep["n_over_model"] == 0, rep
    if w.outlier_p == 0:
        assert rep["max_abs"] <= TOL_O, rep
    assert lse_err <= TOL_LSE

    # ---- dQ of every sampled row
    dq_r, _, _ = oracle.bwd_dq_rows(q, k, v, do, w.causal, w.softmax_scale, rows, **kw)
    figures["dq_rows_rel_l2"] = rel_l2(g["dq"][t, rows[:, 1]], dq_r)
    assert figures["dq_rows_rel_l2"] <= TOL_GRAD

    G = w.Hq // w.Hkv
    if G == 1:
        # ---- multi-head: whole (sequence, head) slices are independent problems the
        # oracle can afford outright, so the gradient bar is checked over full slices
        # (the stated metric is relative L2 over whole tensors; a handful of keys is a
        # biased sample when one key dominates their norm).
        for b, h in ((0, 0), (len(lens) - 1, w.Hq - 1)):
            L, a = lens[b], cu[b]
            sl = slice(a, a + L)
            qs, ks, vs, ds = (np.ascontiguousarray(t[sl, h:h + 1]) for t in (q, k, v, do))
            dq_r, dk_r, dv_r = oracle.bwd(qs, ks, vs, ds, w.causal, w.softmax_scale, B=1, S=L)
            for n_, ref in (("dq", dq_r), ("dk", dk_r), ("dv", dv_r)):
                e = rel_l2(g[n_][sl, h], ref[:, 0])
                figures[f"slice_b{b}_h{h}_{n_}_rel_l2"] = e
                assert e <= TOL_GRAD, (b, h, n_, e)
    else:
        # ---- grouped-query: dK, dV of the first 256 keys (the longest accumulations)
        # of the first and last kv head, in the longest sequence
        bl = int(np.argmax(lens))
        for gh in (0, w.Hkv - 1):
            j1 = min(256, lens[bl])
            dk_r, dv_r = oracle.bwd_dkdv_range(q, k, v, do, w.causal, w.softmax_scale, bl, gh, 0, j1,
                                               **kw)
            a = cu[bl]
            ek = rel_l2(g["dk"][a:a + j1, gh], dk_r)
            ev = rel_l2(g["dv"][a:a + j1, gh], dv_r)
            figures[f"first_keys_kv{gh}_dk_rel_l2"] = ek
            figures[f"first_keys_kv{gh}_dv_rel_l2"] = ev
            assert ek <= TOL_GRAD and ev <= TOL_GRAD, (gh, ek, ev)
        # ---- and of the last keys of a few (sequence, kv head) pairs
        for b, gh in ((len(lens) - 1, w.Hkv - 1), (0, 0)):
            L = lens[b]
            if L == 0:
                continue
            j0 = max(0, L - 160)
            dk_r, dv_r = oracle.bwd_dkdv_range(q, k, v, do, w.causal, w.softmax_scale, b, gh, j0, L,
                                               **kw)
            a = cu[b]
            assert rel_l2(g["dk"][a + j0:a + L, gh], dk_r) <= TOL_GRAD
            assert rel_l2(g["dv"][a + j0:a + L, gh], dv_r) <= TOL_GRAD

    # ---- properties over all keys
    for b, L in enumerate(lens):
        if L == 0:
            continue
        a = cu[b]
        sum_dv = g["dv"][a:a + L].sum(0)                              # [Hkv, D]
        want = g_do = do[a:a + L].reshape(L, w.Hkv, G, w.D).sum((0, 2))  # exact inputs
        assert rel_l2(sum_dv, want) <= 1e-2
        sum_dk = g["dk"][a:a + L].sum(0)
        scale_ref = np.abs(g["dk"][a:a + L]).sum(0)
        assert float(np.abs(sum_dk).max()) <= 2e-2 * float(scale_ref.max()), "sum_j dK_j != 0"
        del g_do


@pytest.mark.gpu
def test_whole_tensors_8k():
    """The 8K workload against the oracle's full forward and backward: O element by
    element, LSE, and dQ, dK, dV by relative L2 over the whole tensors."""
    w = I.workload(1)
    run = DeviceRun(w, poison=True)
    g = run.np_out()
    q, k, v, do, kw = oracle_args(w, run.x)
    o_r, lse_r = oracle.fwd(q, k, v, w.causal, w.softmax_scale, **kw)
    rep = o_error_report(g["o"], o_r, nkeys=w.S)
    lse_err = float(np.abs(g["lse"] - lse_r).max())
    dq_r, dk_r, dv_r = oracle.bwd(q, k, v, do, w.causal, w.softmax_scale, **kw)
    grads = {"dq": rel_l2(g["dq"], dq_r), "dk": rel_l2(g["dk"], dk_r), "dv": rel_l2(g["dv"], dv_r)}
    record(f"whole/{w.name}", o_max_abs=rep["max_abs"], o_n_over_1e_2=rep["n_over_strict"],
           o_elements=rep["n"], lse_max_abs=lse_err, **{f"{n}_rel_l2": e for n, e in grads.items()})
    assert np.isfinite(g["o"]).all() and np.isfinite(g["lse"]).all()
    assert rep["max_abs"] <= TOL_O, rep
    assert lse_err <= TOL_LSE
    for n, e in grads.items():
        assert np.isfinite(g[n]).all(), n
        assert e <= TOL_GRAD, (n, e)
