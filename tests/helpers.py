"""Shared helpers for the tests: input conversion, running the CUDA path through
the C ABI, running the oracle, and the parity metrics with their tolerances."""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

from long_context_attention_fwd_b200 import inputs as I

# Tolerances of the parity bar: bf16 output max |err| <= 1e-2 against the fp64
# oracle, LSE max |err| <= 1e-3, gradients relative L2 <= 1e-2 per tensor.
TOL_O = 1e-2
TOL_LSE = 1e-3
TOL_GRAD = 1e-2


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


# Error model of the bf16 forward output, derived from the kernel's arithmetic.
#
# The kernel forms w_j = bf16(p_j) from the fp32 probabilities p_j of a row (relative
# to its running maximum) and returns O = bf16(O'), O' = sum_j w_j v_j / sum_j w_j: the
# PV product and the normaliser use the same rounded weights.  Write w_j = p_j (1 + e_j)
# with p_j the exact weights.  From sum_j w_j (v_j - O') = 0 it follows exactly that
#     O' - O_ref = sum_j P_j e_j (v_j - O'),      P_j = p_j / sum_k p_k,
# so |O' - O_ref| <= u_w * sum_j P_j |v_j - O_ref| / (1 - u_w), where u_w bounds |e_j|
# and the sum is the row's dispersion about its output ("disp"):
#   * U_BF16 = 2^-8, bf16's unit roundoff: an 8-bit significand has spacing 2^-7 on
#     [1, 2), and rounding to nearest errs by at most half of it;
#   * ETA = 2^-13 covers the 1 / (1 - u_w) factor (2^-16) and the fp32 part of e_j: the
#     scores' tensor-core accumulation over D and ex2.approx, below 2^-15 in relative
#     terms at these inputs' score magnitudes (scale * sum_d |q_d k_d| < 64).
# The final bf16 rounding adds half an ulp of the stored value (round to nearest:
# |bf16(x) - x| <= ulp(bf16(x)) / 2).  fp32 accumulation adds, relative to
# (P|V|)_i = sum_j P_j |v_j|: the PV accumulator (one fp32 rounding per 16-key MMA step,
# truncation allowed: 2^-23 each), the normaliser (at most one rounding per 16 keys after
# the pairwise register sums) and the lazy rescales (one per 128-key tile at most); with
# both numerator and denominator counted, gamma(L) = 2 (L/16 + L/16 + L/128 + 64) 2^-23
# for rows of at most L visible keys.
U_BF16 = 2.0 ** -8
ETA = 2.0 ** -13


def fp32_gamma(nkeys: int) -> float:
    return 2.0 * (nkeys / 16 + nkeys / 16 + nkeys / 128 + 64) * 2.0 ** -23


def o_error_report(o_gpu: np.ndarray, o_ref: np.ndarray, o_absv: Optional[np.ndarray] = None,
                   nkeys: int = 65536, disp=None, max_details: int = 16) -> dict:
    """Errors of a bf16 attention output against the fp64 oracle.

    max_abs        max |O_gpu - O_ref| (the stated bar is 1e-2)
    n_over_strict  elements above 1e-2
    n_over_model   elements above both 1e-2 and their derived bound
                   ulp(O_gpu)/2 + (U_BF16 + ETA) * disp_i + fp32_gamma(nkeys) * (P|V|)_i
    over           details of the elements above 1e-2: flat index, error, |O_ref|,
                   (P|V|)_i, disp_i and the bound
    o_absv = the oracle's attention output with |V| in place of V, i.e. (P|V|)_i.
    disp   = callable(flat indices) -> the rows' dispersions sum_j P_j |v_j - O_ref| at
             those elements (from the oracle); without it the upper bound
             (P|V|)_i + |O_ref,i| is used.  Only elements above 1e-2 need it.
    nkeys  = an upper bound on the keys any row sees.
    """
    o_gpu = o_gpu.astype(np.float64)
    err = np.abs(o_gpu - o_ref)
    if o_absv is None:
        o_absv = np.abs(o_ref)
    flat = np.flatnonzero(err.ravel() > TOL_O)
    details = []
    n_model = 0
    if flat.size:
        e = err.ravel()[flat]
        oref = np.abs(o_ref.ravel()[flat])
        pv = np.abs(o_absv.ravel()[flat])
        d = np.asarray(disp(flat), dtype=np.float64) if disp is not None else pv + oref
        bound = (0.5 * bf16_ulp(o_gpu.ravel()[flat]) + (U_BF16 + ETA) * d
                 + fp32_gamma(nkeys) * pv)
        n_model = int((e > bound).sum())
        for i in range(min(flat.size, max_details)):
            details.append({"index": int(flat[i]), "err": float(e[i]), "abs_o_ref": float(oref[i]),
                            "PabsV": float(pv[i]), "disp": float(d[i]), "bound": float(bound[i])})
    return {"max_abs": float(err.max()) if err.size else 0.0,
            "n_over_strict": int(flat.size), "n_over_model": n_model, "n": int(err.size),
            "over": details}


def row_dispersion(q, k, v, o_ref_rows, row_of, causal, scale, cu):
    """disp callable for o_error_report over an array of output rows.

    o_ref_rows: [n, D] oracle rows; row_of(r) -> (b, h, i) names output row r (sequence,
    query head, position).  For element (r, d) it returns sum_j P_rj |v_jd - O_ref[r, d]|
    over the keys row r sees, from the oracle's forward on the row's own sequence and kv
    head with |V - O_ref[r]| in place of V."""
    import oracle
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    D = q.shape[2]

    def disp(flat):
        out = np.empty(len(flat))
        cache = {}
        for n, f in enumerate(flat):
            r, d = divmod(int(f), D)
            if r not in cache:
                b, h, i = row_of(r)
                a, L = int(cu[b]), int(cu[b + 1] - cu[b])
                g = h // G
                qs = np.ascontiguousarray(q[a:a + L, h:h + 1])
                ks = np.ascontiguousarray(k[a:a + L, g:g + 1])
                vs = np.ascontiguousarray(np.abs(v[a:a + L, g:g + 1] - o_ref_rows[r]))
                o1, _ = oracle.fwd_rows(qs, ks, vs, causal, scale,
                                        np.array([[0, 0, i]], dtype=np.int32), B=1, S=L)
                cache[r] = o1[0]
            out[n] = cache[r][d]
        return out
    return disp


# Parity figures recorded by the GPU tests; the terminal summary prints them (conftest).
PARITY_LOG: list = []


def record(label: str, **metrics) -> dict:
    """Logs figures under `label`; returns the logged dict, so that a test can add
    figures as it goes and the ones it reached still print when an assertion fails."""
    PARITY_LOG.append((label, metrics))
    return metrics


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def torch_bf16(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bits_of(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(bits: np.ndarray) -> np.ndarray:
    return I.bf16_bits_to_f64(bits)


def make_case(B, Hq, Hkv, S, D, causal=True, lens=None, seed=1234, qkv_mult=0.5, do_mult=1.0,
              outlier_p=0.0, outlier_mult=1.0, scale=None):
    w = I.Workload(name="case", B=B if lens is None else 0, Hq=Hq, Hkv=Hkv,
                   S=S if lens is None else sum(lens), D=D, causal=causal, qkv_mult=qkv_mult,
                   do_mult=do_mult, outlier_p=outlier_p, outlier_mult=outlier_mult, varlen=lens,
                   seed=seed, scale=scale)
    return w


class DeviceRun:
    """Runs attn_fwd / attn_bwd of the library on a workload's seeded inputs."""

    def __init__(self, w: I.Workload, device="cuda", poison=True):
        import torch
        from long_context_attention_fwd_b200 import ops
        self.w = w
        x = I.make_inputs(w)
        self.x = x
        T = w.tokens
        dense = w.varlen is None
        shp_q = (w.B, w.S, w.Hq, w.D) if dense else (T, w.Hq, w.D)
        shp_k = (w.B, w.S, w.Hkv, w.D) if dense else (T, w.Hkv, w.D)
        self.q = torch_bf16(x["q"], device).view(shp_q)
        self.k = torch_bf16(x["k"], device).view(shp_k)
        self.v = torch_bf16(x["v"], device).view(shp_k)
        self.do = torch_bf16(x["do"], device).view(shp_q)
        self.cu = None if dense else torch.from_numpy(x["cu_seqlens"]).to(device)
        o = torch.empty_like(self.q)
        lse = torch.empty((w.Hq, T) if not dense else (w.B, w.Hq, w.S), dtype=torch.float32,
                          device=device)
        if poison:
            o.view(torch.int16).fill_(0x7FC0)  # bf16 NaN
            lse.fill_(float("nan"))
        self.o, self.lse = ops.attn_fwd(self.q, self.k, self.v, causal=w.causal,
                                        scale=w.softmax_scale, cu_seqlens=self.cu, out=o, lse=lse)
        dq, dk, dv = (torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v))
        if poison:
            for t in (dq, dk, dv):
                t.view(torch.int16).fill_(0x7FC0)
        self.dq, self.dk, self.dv = ops.attn_bwd(self.q, self.k, self.v, self.o, self.lse, self.do,
                                                 causal=w.causal, scale=w.softmax_scale,
                                                 cu_seqlens=self.cu, dq=dq, dk=dk, dv=dv)
        torch.cuda.synchronize()
        from long_context_attention_fwd_b200 import capi
        st, site = capi.attn_device_status(None)   # no device wait may have run out
        assert st == capi.ATTN_OK, (capi.strerror(st), hex(site))

    def np_out(self):
        """GPU results as fp64 numpy in the oracle's layouts ([T,H,D], lse [B,Hq,S] or [Hq,T])."""
        w = self.w
        T = w.tokens
        cv = lambda t, H: f64(bits_of(t)).reshape(T, H, w.D)
        return {"o": cv(self.o, w.Hq), "lse": self.lse.double().cpu().numpy(),
                "dq": cv(self.dq, w.Hq), "dk": cv(self.dk, w.Hkv), "dv": cv(self.dv, w.Hkv)}


def oracle_args(w: I.Workload, x: dict):
    kw = {"cu_seqlens": x["cu_seqlens"]} if w.varlen is not None else {"B": w.B, "S": w.S}
    return f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), kw


def flops_fwd(w: I.Workload) -> float:
    return I.flop_fwd(w)


def pow2_ceil(n: int) -> int:
    return 1 << max(0, math.ceil(math.log2(max(1, n))))
