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


def o_error_report(o_gpu: np.ndarray, o_ref: np.ndarray, o_absv: Optional[np.ndarray] = None) -> dict:
    """Errors of a bf16 attention output against the fp64 oracle.

    max_abs        max |O_gpu - O_ref| (the stated bar is 1e-2)
    n_over_strict  elements above 1e-2
    n_over_model   elements above max(1e-2, bound), bound = half a bf16 ulp of O_ref
                   (output rounding) + 2^-8 * (P|V|)_i (P is rounded to bf16 before the
                   PV product: relative error <= 2^-9 per probability, doubled for margin).
                   o_absv = attention output with |V| in place of V, from the oracle.
    """
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    if o_absv is None:
        o_absv = np.abs(o_ref)
    bound = np.maximum(TOL_O, 0.5 * bf16_ulp(o_ref) + 2.0 ** -8 * np.abs(o_absv) + 1e-5)
    return {"max_abs": float(err.max()) if err.size else 0.0,
            "n_over_strict": int((err > TOL_O).sum()),
            "n_over_model": int((err > bound).sum())}


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
