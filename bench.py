#!/usr/bin/env python3
"""Benchmark of the fused attention hot path (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = attn_fwd + attn_bwd over one batch of the workload (default: the
32K-token causal GQA case, Qwen2.5-7B attention shape: B=1, Hq=28, Hkv=4, D=128,
S=32768), inputs resident in HBM.  Prints ONE JSON line on rank 0.

FLOP convention: forward 4*S^2*D*Hq*B, halved when causal; backward 2.5x that.
Under torchrun (N > 1) every rank runs its own independent batch (weak scaling,
no collective on the data path); the reported time is the max over ranks.

On one GPU the line also carries "ring": the exact merge kernel of Ring attention
(attn_merge, HBM-bound, against the measured copy bandwidth) and the forward of a
4-rank ring run rank after rank on this GPU; and "ulysses": the relayout kernel around
the Ulysses all-to-alls (HBM-bound) and forward + backward of a 4-rank Ulysses group run
rank after rank on this GPU; and "decode": attention of one new token per sequence over
a 32K-token KV cache (HBM-bound); and "fp8_fwd": the e4m3 forward on the bench workload.
All are measured after the timed steps.

--impl reference times the fp64 CPU oracle (the bench's reference arm) on a
bounded sample of the same workload: the first tokens of the causal sequence form
an exact sub-problem, so each step runs the oracle's forward and backward on them.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from long_context_attention_fwd_b200 import inputs as I  # noqa: E402

METRIC = "attn fwd/bwd TFLOP/s at S=32K causal GQA bf16; % of B200 BF16 peak"
DEFAULT_WORKLOAD = "qwen2.5-7b_gqa28x4_S32768_D128"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["_source"] = "MEASURED_PEAKS.json"
        return d, "measured (MEASURED_PEAKS.json)"
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback peaks (no MEASURED_PEAKS.json)"
    return d, "fallback (no MEASURED_PEAKS.json)"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def workload_config(w: I.Workload) -> dict:
    cfg = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "D": w.D,
           "causal": w.causal, "scale": w.softmax_scale,
           "values": f"q,k,v ~ N(0,1)*{w.qkv_mult}, dO ~ N(0,1)*{w.do_mult}, seeded, bf16"}
    if w.varlen is not None:
        cfg["varlen_lengths"] = list(w.varlen)
    return cfg


# ---------------------------------------------------------------- ranks
def rank_workload(w: I.Workload, rank: int) -> I.Workload:
    """The independent batch a rank processes: the same shapes, its own seed."""
    return I.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (the job is as slow as its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


# ---------------------------------------------------------------- ncu traffic
# The sources each kernel is compiled from: a traffic record is valid only for these bytes.
KERNEL_SOURCES = {
    "attn_fwd_kernel": ("sm100_ptx.cuh", "attn_common.cuh", "attn_fwd.cuh"),
    "attn_bwd_kernel": ("sm100_ptx.cuh", "attn_common.cuh", "attn_bwd.cuh"),
    "attn_merge_kernel_4parts": ("sm100_ptx.cuh", "attn_merge.cuh"),
}


def kernel_sources_sha1(kernel: str) -> str:
    import hashlib
    h = hashlib.sha1()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "long_context_attention_fwd_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload: str, kernel: str):
    """DRAM bytes (read + write) per launch of `kernel` from the ncu capture summarised
    in profiles/traffic.json, or None when the kernel's sources changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))["workloads"][workload][kernel]
        if rec.get("sources_sha1") != kernel_sources_sha1(kernel):
            return None
        return rec["dram_bytes_per_launch"]
    except Exception:
        return None


# ---------------------------------------------------------------- clocks
CLOCK_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def summarize_clocks(lines, t0: float, t1: float) -> dict:
    """Summary of `nvidia-smi --query-gpu=CLOCK_FIELDS --format=csv,noheader,nounits` lines
    for the samples taken in the wall-clock window [t0, t1] (seconds since the epoch):
    median SM clock, the maximum SM clock, every throttle reason seen active and the
    sample count.  When no sample falls in the window (a region shorter than the sampling
    interval) the samples just around it are used, and `window` says so."""
    import datetime
    rows = []
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 10:
            continue
        try:
            ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            rows.append((ts, float(parts[2]), float(parts[3]), float(parts[4]), parts[5:]))
        except ValueError:
            continue
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
    inside = [r for r in rows if t0 <= r[0] <= t1]
    window = "timed region"
    if not inside:
        near = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))
        inside = near[:2]
        window = "nearest samples (none inside the timed region)"
    reasons = set()
    for r in inside:
        for n, v in zip(CLOCK_REASONS, r[4][1:]):
            if v.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(r[1] for r in inside),
            "sm_max_mhz": max(r[2] for r in rows),
            "reasons": sorted(reasons), "samples": len(inside),
            "power_w_max": max(r[3] for r in inside), "window": window}


class ClockSampler:
    """nvidia-smi every 50 ms, read through a pipe (no file) by a thread that keeps the
    pipe drained, and summarised over the timed region's wall-clock window."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.reader = None

    def _drain(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._drain, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None

    def stop(self, t0: float, t1: float) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)  # the sample after the region's end
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.reader.join(timeout=5)
        return summarize_clocks(list(self.lines), t0, t1)


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(w: I.Workload, tokens: int):
    """The first `tokens` tokens of the workload's first sequence: an exact causal
    sub-problem (no row sees a later key).  Returns (fwd callable, bwd callable, fwd FLOPs,
    bwd FLOPs, description)."""
    import oracle
    tokens = min(tokens, w.seq_lengths()[0] if w.varlen is not None else w.S)
    sub = I.Workload(name=w.name + "_prefix", B=1, Hq=w.Hq, Hkv=w.Hkv, S=tokens, D=w.D,
                     causal=w.causal, qkv_mult=w.qkv_mult, do_mult=w.do_mult,
                     outlier_p=w.outlier_p, outlier_mult=w.outlier_mult, seed=w.seed)
    x = I.make_inputs(sub)
    q, k, v, do = (I.bf16_bits_to_f64(x[n]) for n in ("q", "k", "v", "do"))

    def run_fwd():
        oracle.fwd(q, k, v, sub.causal, sub.softmax_scale, B=1, S=tokens)

    def run_bwd():
        oracle.bwd(q, k, v, do, sub.causal, sub.softmax_scale, B=1, S=tokens)

    desc = (f"fp64 oracle on a {tokens}-token causal prefix (exact sub-problem) "
            f"with the workload's heads (Hq={w.Hq}, Hkv={w.Hkv}, D={w.D})")
    return run_fwd, run_bwd, I.flop_fwd(sub), I.flop_bwd(sub), desc


def _time_budget(fn, budget_s: float):
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return n, time.perf_counter() - t0


def cpu_baseline(w: I.Workload, budget_s: float = 6.0, others_s: float = 1.5):
    """The oracle on the host cores: forward and backward timed separately on a prefix of
    the bench workload (`budget_s` each), and on a shorter prefix of every other workload
    (`others_s` each).  `value` is forward + backward FLOPs over their summed time."""
    import oracle
    tokens = 1024 if w.D >= 128 else 2048
    fwd, bwd, ff, fb, desc = oracle_sample(w, tokens)
    nf, tf = _time_budget(fwd, budget_s)
    nb, tb = _time_budget(bwd, budget_s)
    fwd_tf = ff * nf / tf / 1e12
    bwd_tf = fb * nb / tb / 1e12
    per_cfg = {}
    for ow in I.workloads():
        if ow.name == w.name or ow.S <= 256:
            continue
        f2, b2, ff2, fb2, _ = oracle_sample(ow, 512)
        n1, t1 = _time_budget(f2, others_s)
        n2, t2 = _time_budget(b2, others_s)
        per_cfg[ow.name] = {"fwd_tflops": ff2 * n1 / t1 / 1e12, "bwd_tflops": fb2 * n2 / t2 / 1e12,
                            "sample": "512-token causal prefix of the first sequence"}
    return {"value": (ff + fb) / (tf / nf + tb / nb) / 1e12, "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
            "sample": f"{desc}; forward {nf} run(s) in {tf:.1f} s, backward {nb} run(s) in "
                      f"{tb:.1f} s",
            "other_workloads": per_cfg}


def run_reference(args, w: I.Workload):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    tokens = 1024 if w.D >= 128 else 2048
    fwd, bwd, ff, fb, desc = oracle_sample(w, tokens)
    for _ in range(args.warmup):
        fwd()
        bwd()
    tf = tb = 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        fwd()
        t1 = time.perf_counter()
        bwd()
        tf += t1 - t0
        tb += time.perf_counter() - t1
    dt = tf + tb
    value = (ff + fb) * args.steps / dt / 1e12
    cores = oracle.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "fwd_tflops": ff * args.steps / tf / 1e12,
                         "bwd_tflops": fb * args.steps / tb / 1e12, "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def ring_measurements(wr: I.Workload, q, k, v, o, lse, stream, peaks, world=4, reps=10):
    """Measures the Ring-attention rows on one GPU, outside the timed step:
    (1) attn_merge over `world` full-size partials (HBM-bound: bytes read + written per
        launch / CUDA-event time, against the measured copy bandwidth);
    (2) the forward of a `world`-rank ring run rank after rank on this GPU (chunk partials
        from attn_fwd + attn_merge), against the single-kernel forward of the same problem.
    Every buffer is far larger than L2, so no flush is needed between launches."""
    import torch
    from long_context_attention_fwd_b200 import ops, ring

    o_parts = [o.clone() for _ in range(world)]
    lse_parts = [lse + 0.25 * j for j in range(world)]
    out, lse_out = torch.empty_like(o), torch.empty_like(lse)

    def timed(fn):
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        torch.cuda.synchronize()
        for e0, e1 in evs:
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)

    merge_ms = timed(lambda: ops.attn_merge(o_parts, lse_parts, out=out, lse=lse_out))
    row_bytes = o.numel() * o.element_size() + lse.numel() * lse.element_size()
    merge_bytes = (world + 1) * row_bytes
    hbm = float(peaks.get("hbm_gbs"))
    gbs = merge_bytes / (merge_ms * 1e-3) / 1e9
    ring_ms = timed(lambda: ring.ring_attn_fwd_single_device(q, k, v, world, wr.causal,
                                                             wr.softmax_scale))
    fwd_ms = timed(lambda: ops.attn_fwd(q, k, v, causal=wr.causal, scale=wr.softmax_scale))
    del o_parts, lse_parts, out, lse_out
    do = torch.randn(q.shape, device=q.device, dtype=torch.float32).to(q.dtype)
    ring_bwd_ms = timed(lambda: ring.ring_attn_bwd_single_device(q, k, v, o, lse, do, world,
                                                                 wr.causal, wr.softmax_scale))
    bwd_ms = timed(lambda: ops.attn_bwd(q, k, v, o, lse, do, causal=wr.causal,
                                        scale=wr.softmax_scale))
    del do
    n_fwd = sum(len(ring.ring_schedule(r, world, wr.causal)) for r in range(world))
    n_merge = sum(len(ring.ring_schedule(r, world, wr.causal)) > 1 for r in range(world))
    return {
        "merge": {"kernel": "attn_merge_kernel<%d,4,1>" % wr.D, "bound": "hbm",
                  "workload": f"{world} partials of o {list(o.shape)} bf16 + lse {list(lse.shape)} "
                              f"fp32 -> one (o, lse)",
                  "ms": merge_ms, "bytes_per_launch": merge_bytes, "achieved": gbs,
                  "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                  "traffic": (measured_traffic(wr.name, "attn_merge_kernel_4parts")
                              if world == 4 else None),
                  "peak_source": f"{peaks['_source']} hbm_gbs (copy, read+write bytes)"},
        "ring_fwd_one_gpu": {"world": world, "ms": ring_ms,
                             "tflops": I.flop_fwd(wr) / (ring_ms * 1e-3) / 1e12,
                             "single_kernel_fwd_ms": fwd_ms, "attn_fwd_launches": n_fwd,
                             "attn_merge_launches": n_merge,
                             "note": "every rank's partials and merge run one after another on "
                                     "this GPU; the K/V transfers of a real ring are not timed"},
        "ring_bwd_one_gpu": {"world": world, "ms": ring_bwd_ms,
                             "tflops": I.flop_bwd(wr) / (ring_bwd_ms * 1e-3) / 1e12,
                             "single_kernel_bwd_ms": bwd_ms,
                             "note": "block-pair attn_bwd with the merged O/LSE per scheduled pair, "
                                     "shares summed in fp32 (attn_accumulate_bf16), rounded once; "
                                     "every rank on this GPU, transfers not timed"},
    }


def ulysses_measurements(wr: I.Workload, q, k, v, do, stream, peaks, world=4, reps=10):
    """Measures the Ulysses rows on one GPU, outside the timed step:
    (1) the relayout kernel (attn_transpose_blocks) on q as one rank's send buffer for a
        `world`-rank group (HBM-bound: bytes read + written / CUDA-event time);
    (2) forward + backward of every rank of a `world`-rank group run one after another on
        this GPU (relayouts around emulated all-to-alls, attention per head group), beside
        the unsplit forward + backward."""
    import torch
    from long_context_attention_fwd_b200 import ops
    from long_context_attention_fwd_b200 import ulysses as U

    def timed(fn):
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        torch.cuda.synchronize()
        for e0, e1 in evs:
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)

    B, S, Hq, D = q.shape
    out = torch.empty_like(q)
    tr_ms = timed(lambda: ops.transpose_blocks(q, B * S, world, out=out))
    tr_bytes = 2 * q.numel() * q.element_size()
    hbm = float(peaks.get("hbm_gbs"))
    gbs = tr_bytes / (tr_ms * 1e-3) / 1e9
    del out
    uly_ms = timed(lambda: U.ulysses_attention_single_device(q, k, v, world, wr.causal,
                                                             wr.softmax_scale, do=do))

    def plain():
        o, lse = ops.attn_fwd(q, k, v, causal=wr.causal, scale=wr.softmax_scale)
        ops.attn_bwd(q, k, v, o, lse, do, causal=wr.causal, scale=wr.softmax_scale)

    plain_ms = timed(plain)
    return {
        "relayout": {"kernel": "transpose_blocks_kernel", "bound": "hbm",
                     "workload": f"q {list(q.shape)} bf16 -> send buffer of {world} head "
                                 f"groups [{world}, {B * S}, {Hq // world}, {D}]",
                     "ms": tr_ms, "bytes_per_launch": tr_bytes, "achieved": gbs, "peak": hbm,
                     "unit": "GB/s", "frac": gbs / hbm,
                     "peak_source": f"{peaks['_source']} hbm_gbs (copy, read+write bytes)"},
        "ulysses_fwd_bwd_one_gpu": {
            "world": world, "ms": uly_ms,
            "tflops": (I.flop_fwd(wr) + I.flop_bwd(wr)) / (uly_ms * 1e-3) / 1e12,
            "unsplit_fwd_bwd_ms": plain_ms,
            "note": "every rank's relayouts and head-group attention run one after another on "
                    "this GPU; the all-to-alls are plain copies here, NCCL in a real group"},
    }


def fp8_measurements(wr: I.Workload, q, k, v, stream, peaks, reps=10):
    """Measures the e4m3 forward (attn_fwd_fp8) on the bench workload, outside the timed
    step: the bf16 inputs quantised per tensor (descale = max|x| / 448) on the GPU, then
    forward TFLOP/s (same FLOP convention) against the fp8 peak, taken as the measured bf16
    peak times the nominal fp8 : bf16 ratio of 2 (4.5 vs 2.25 PFLOP/s dense)."""
    import torch
    from long_context_attention_fwd_b200 import ops

    def q8(t):
        d = float(t.abs().max().float()) / 448.0
        return (t.float() / d).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn), d

    (q8_, qd), (k8_, kd), (v8_, vd) = q8(q), q8(k), q8(v)

    def timed(fn):
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        torch.cuda.synchronize()
        for e0, e1 in evs:
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)

    fp8_ms = timed(lambda: ops.attn_fwd_fp8(q8_, k8_, v8_, qd, kd, vd, causal=wr.causal,
                                            scale=wr.softmax_scale))
    bf16_ms = timed(lambda: ops.attn_fwd(q, k, v, causal=wr.causal, scale=wr.softmax_scale))
    tf = I.flop_fwd(wr) / (fp8_ms * 1e-3) / 1e12
    peak = 2.0 * float(peaks.get("bf16_tflops"))
    return {"kernel": "attn_fwd_kernel<128, e4m3>", "bound": "tensor", "ms": fp8_ms,
            "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
            "peak_source": f"{peaks['_source']} bf16_tflops (burst) x 2, the nominal fp8:bf16 ratio",
            "bf16_fwd_ms_same_run": bf16_ms, "speedup_vs_bf16": bf16_ms / fp8_ms,
            "inputs": "the bench workload's q, k, v quantised per tensor to e4m3 on the GPU"}


def decode_measurements(dev, stream, peaks, reps=20):
    """Measures decode attention over a KV cache (attn_decode: split-KV kernel + merge) on
    the two decode workloads, outside the timed step.  HBM-bound: achieved = the cached
    K/V bytes read plus q read and o/lse written, / median CUDA-event time, against the
    measured copy bandwidth.  The cache (1.4 GB at 16 x 32K) exceeds L2, and a 256 MB buffer
    is written between launches so the single-sequence case (67 MB) starts cold too.
    Values are seeded normals drawn on the GPU (their values do not change the timing)."""
    import torch
    from long_context_attention_fwd_b200 import ops

    out = {}
    gen = torch.Generator(device=dev).manual_seed(20261212)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    hbm = float(peaks.get("hbm_gbs"))
    for w in I.decode_workloads()[1:]:
        q = torch.randn((w.B, w.Hq, w.D), generator=gen, device=dev).mul_(w.qkv_mult).bfloat16()
        k = torch.randn((w.B, w.Lmax, w.Hkv, w.D), generator=gen, device=dev).mul_(w.qkv_mult).bfloat16()
        v = torch.randn((w.B, w.Lmax, w.Hkv, w.D), generator=gen, device=dev).mul_(w.qkv_mult).bfloat16()
        cl = torch.tensor(w.lens, dtype=torch.int32, device=dev)
        ws = torch.empty(ops.attn_decode_workspace_size(q, k), dtype=torch.uint8, device=dev)
        o, lse = torch.empty_like(q), torch.empty((w.B, w.Hq), device=dev)
        for _ in range(3):
            ops.attn_decode(q, k, v, cl, scale=w.softmax_scale, out=o, lse=lse, workspace=ws)
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ops.attn_decode(q, k, v, cl, scale=w.softmax_scale, out=o, lse=lse, workspace=ws)
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        gbs = w.io_bytes() / (ms * 1e-3) / 1e9
        out[w.name] = {"kernels": "attn_decode_kernel (split-KV partials merged by the last split)",
                       "bound": "hbm", "ms": ms, "bytes": w.io_bytes(), "achieved": gbs,
                       "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                       "tokens_per_s": w.B / (ms * 1e-3),
                       "cache_lengths": f"{min(w.lens)}..{max(w.lens)} (sum {sum(w.lens)})"}
        del q, k, v, ws
    return out


def run_gpu(args, w: I.Workload):
    import torch
    from long_context_attention_fwd_b200 import ops

    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)

    # Each rank owns an independent batch: seed offset by rank.
    wr = rank_workload(w, rank)
    x = I.make_inputs(wr)
    dense = wr.varlen is None
    T = wr.tokens
    shp_q = (wr.B, wr.S, wr.Hq, wr.D) if dense else (T, wr.Hq, wr.D)
    shp_k = (wr.B, wr.S, wr.Hkv, wr.D) if dense else (T, wr.Hkv, wr.D)

    def host_bf16(bits, shape):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
        return t.view(shape).pin_memory()

    hq, hk, hv, hdo = (host_bf16(x["q"], shp_q), host_bf16(x["k"], shp_k),
                       host_bf16(x["v"], shp_k), host_bf16(x["do"], shp_q))
    q, k, v, do = (t.to(dev) for t in (hq, hk, hv, hdo))
    cu = None if dense else torch.from_numpy(x["cu_seqlens"]).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((wr.Hq, T) if not dense else (wr.B, wr.Hq, wr.S), dtype=torch.float32,
                      device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsp = torch.empty(ops.attn_bwd_workspace_size(q, cu), dtype=torch.uint8, device=dev)
    scale = wr.softmax_scale
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        ops.attn_fwd(q, k, v, causal=wr.causal, scale=scale, cu_seqlens=cu, out=o, lse=lse)
        if ev is not None:
            ev[1].record(stream)
        ops.attn_bwd(q, k, v, o, lse, do, causal=wr.causal, scale=scale, cu_seqlens=cu,
                     dq=dq, dk=dk, dv=dv, workspace=wsp)
        if ev is not None:
            ev[2].record(stream)

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(max(args.warmup, 3)):
        step()
    from long_context_attention_fwd_b200 import capi
    st, site = capi.attn_device_status(stream.cuda_stream)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {capi.strerror(st)} site={site:#x}")

    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler.start()
    time.sleep(0.3)
    barrier()
    wall0 = time.time()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    barrier()
    wall1 = time.time()
    clocks = sampler.stop(wall0, wall1)
    total_ms = t_start.elapsed_time(t_end)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    st, site = capi.attn_device_status(stream.cuda_stream)
    if st != 0:
        raise RuntimeError(f"device status after timing: {capi.strerror(st)} site={site:#x}")

    # End to end through the public API from pinned host buffers, every step's inputs
    # copied in and its results copied out inside the timed region.  The copies of
    # neighbouring steps overlap the compute on their own streams (two buffer sets):
    # step i's host->device copy runs during step i-1's compute, its device->host copy
    # during step i+1's.
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hdq = torch.empty(dq.shape, dtype=dq.dtype).pin_memory()
    hdk = torch.empty(dk.shape, dtype=dk.dtype).pin_memory()
    hdv = torch.empty(dv.shape, dtype=dv.dtype).pin_memory()
    hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    bufs = []
    for _ in range(2):
        bufs.append({"in": [torch.empty_like(t) for t in (q, k, v, do)],
                     "o": torch.empty_like(o), "lse": torch.empty_like(lse),
                     "dq": torch.empty_like(dq), "dk": torch.empty_like(dk),
                     "dv": torch.empty_like(dv),
                     "in_done": torch.cuda.Event(), "comp_done": torch.cuda.Event(),
                     "out_done": torch.cuda.Event()})

    def e2e_step(i):
        bb = bufs[i % 2]
        with torch.cuda.stream(s_in):
            s_in.wait_event(bb["comp_done"])          # step i-2 no longer reads these inputs
            for dst, src in zip(bb["in"], (hq, hk, hv, hdo)):
                dst.copy_(src, non_blocking=True)
            bb["in_done"].record(s_in)
        stream.wait_event(bb["in_done"])
        stream.wait_event(bb["out_done"])             # step i-2's results have left
        qd, kd, vd, dod = bb["in"]
        ops.attn_fwd(qd, kd, vd, causal=wr.causal, scale=scale, cu_seqlens=cu, out=bb["o"],
                     lse=bb["lse"])
        ops.attn_bwd(qd, kd, vd, bb["o"], bb["lse"], dod, causal=wr.causal, scale=scale,
                     cu_seqlens=cu, dq=bb["dq"], dk=bb["dk"], dv=bb["dv"], workspace=wsp)
        bb["comp_done"].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(bb["comp_done"])
            for h, d in ((ho, bb["o"]), (hlse, bb["lse"]), (hdq, bb["dq"]), (hdk, bb["dk"]),
                         (hdv, bb["dv"])):
                h.copy_(d, non_blocking=True)
            bb["out_done"].record(s_out)

    e2e_steps = max(2, args.steps)
    for i in range(2):                                # warm-up of both buffer sets
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)                                   # before the first copy in
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(s_out)                                  # after the last copy out
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    d2h = sum(t.numel() * t.element_size() for t in (ho, hlse, hdq, hdk, hdv))
    del bufs

    # max over ranks
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)

    fl_f, fl_b = I.flop_fwd(wr), I.flop_bwd(wr)
    ms_step = total_ms / args.steps
    value = ws * (fl_f + fl_b) * args.steps / (total_ms * 1e-3) / 1e12
    peaks, peaks_src = load_peaks()
    peak_sus = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    peak_burst = float(peaks.get("bf16_tflops"))
    f_ms, b_ms = statistics.mean(fwd_ms), statistics.mean(bwd_ms)
    fwd_tf = fl_f / (f_ms * 1e-3) / 1e12
    bwd_tf = fl_b / (b_ms * 1e-3) / 1e12

    traffic = measured_traffic(wr.name, "attn_bwd_kernel")
    ring_rows = uly_rows = None
    if ws == 1 and dense and wr.B == 1 and wr.S % 4 == 0 and not args.no_ring:
        ring_rows = ring_measurements(wr, q, k, v, o, lse, stream, peaks)
    if (ws == 1 and dense and wr.S % 4 == 0 and wr.Hq % 4 == 0 and wr.Hkv % 4 == 0
            and not args.no_ulysses):
        uly_rows = ulysses_measurements(wr, q, k, v, do, stream, peaks)
    fp8_row = None
    if ws == 1 and dense and wr.D == 128 and not args.no_fp8:
        fp8_row = fp8_measurements(wr, q, k, v, stream, peaks)
    dec_rows = None
    if ws == 1 and not args.no_decode:
        dec_rows = decode_measurements(dev, stream, peaks)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
            "config": {**workload_config(wr),
                       "l2": f"no flush: q alone is {q.numel() * 2 / 2**20:.0f} MiB > 126 MiB L2",
                       "parallelism": f"dp{ws} (independent batch per GPU)"},
            "fwd_ms": f_ms, "bwd_ms": b_ms, "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
            "fwd_frac_of_sustained_peak": fwd_tf / peak_sus,
            "bwd_frac_of_sustained_peak": bwd_tf / peak_sus,
            "fwd_frac_of_burst_peak": fwd_tf / peak_burst,
            "bwd_frac_of_burst_peak": bwd_tf / peak_burst,
            "fwd_frac_of_nominal_2250": fwd_tf / 2250.0,
            "bwd_frac_of_nominal_2250": bwd_tf / 2250.0,
            "roofline": {
                "bound": "tensor", "kernel": "attn_bwd (main kernel; time includes its two "
                                             "small helper kernels, so frac is a lower bound)",
                "achieved": bwd_tf, "peak": peak_burst, "unit": "TFLOP/s",
                "frac": bwd_tf / peak_burst,
                "frac_of_sustained_peak": bwd_tf / peak_sus,
                "peak_source": f"{peaks_src}: bf16_tflops (burst: the timed loop lasts "
                               f"{total_ms / 1e3:.2f} s, far shorter than the seconds-long "
                               f"sustained measurement)",
                "traffic": traffic,
                "algorithmic_flop_per_launch": fl_b,
            },
            "e2e": {"value": ws * (fl_f + fl_b) / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "copies": "pinned host buffers; each step's copies in and out overlap the "
                              "neighbouring steps' compute on two other streams (2 buffer "
                              "sets); timed from the first copy in to the last copy out"},
            "gpu_launches": 4 * args.steps,
            "clocks": clocks,
        }
        if ring_rows is not None:
            line["ring"] = ring_rows
        if uly_rows is not None:
            line["ulysses"] = uly_rows
        if dec_rows is not None:
            line["decode"] = dec_rows
        if fp8_row is not None:
            line["fp8_fwd"] = fp8_row
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wr)
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_profile_case(args):
    """One launch of the forward and/or backward on a reduced synthetic problem, for ncu
    captures that must stay small (a few GB on the device, one launch of each kernel):
    --profile B,Hq,Hkv,S,D [--profile-op fwd|fwd8|bwd|both|decode|merge|relayout]
    [--profile-outliers] (fwd8: two e4m3 forward launches after one bf16 one; decode: B
    sequences of S cached keys, two decode steps; merge: two merges of 4 partials shaped
    like the forward's output; relayout: q into 4 head groups, twice).  Inputs are
    drawn on the GPU (N(0,1) * 0.5, or N(0,1) with 1% of q, k entries x8); the backward
    needs the forward's output, so --profile-op bwd also launches the forward once."""
    import torch
    from long_context_attention_fwd_b200 import capi, ops
    B, Hq, Hkv, S, D = (int(x) for x in args.profile.split(","))
    dev = torch.device("cuda", 0)
    if args.profile_op == "decode":
        # one decode step: B sequences of S cached keys each
        g = torch.Generator(device=dev).manual_seed(20261203)
        q = (torch.randn((B, Hq, D), generator=g, device=dev) * 0.5).bfloat16()
        k = (torch.randn((B, S, Hkv, D), generator=g, device=dev) * 0.5).bfloat16()
        v = (torch.randn((B, S, Hkv, D), generator=g, device=dev) * 0.5).bfloat16()
        cl = torch.full((B,), S, dtype=torch.int32, device=dev)
        for _ in range(2):
            ops.attn_decode(q, k, v, cl)
        torch.cuda.synchronize()
        st, site = capi.attn_device_status(None)
        if st != capi.ATTN_OK:
            raise RuntimeError(f"device status {capi.strerror(st)} site={site:#x}")
        print(json.dumps({"profile_case": [B, Hq, Hkv, S, D], "op": "decode", "status": "ok"}))
        return 0
    if args.profile_op in ("merge", "relayout"):
        g = torch.Generator(device=dev).manual_seed(20261203)
        x = (torch.randn((B, S, Hq, D), generator=g, device=dev) * 0.5).bfloat16()
        parts = [x.clone() for _ in range(4)] if args.profile_op == "merge" else None
        lse = torch.randn((B, Hq, S), generator=g, device=dev)
        lses = [lse + 0.25 * j for j in range(4)]
        for _ in range(2):
            if args.profile_op == "merge":
                ops.attn_merge(parts, lses)
            else:
                ops.transpose_blocks(x, B * S, 4)
        torch.cuda.synchronize()
        st, site = capi.attn_device_status(None)
        if st != capi.ATTN_OK:
            raise RuntimeError(f"device status {capi.strerror(st)} site={site:#x}")
        print(json.dumps({"profile_case": [B, Hq, Hkv, S, D], "op": args.profile_op, "status": "ok"}))
        return 0
    g = torch.Generator(device=dev).manual_seed(20261203)
    mult = 1.0 if args.profile_outliers else 0.5

    def draw(H, outliers):
        x = torch.randn((B, S, H, D), generator=g, device=dev) * mult
        if outliers:
            x = torch.where(torch.rand(x.shape, generator=g, device=dev) < 0.01, x * 8, x)
        return x.bfloat16()

    q, k = draw(Hq, args.profile_outliers), draw(Hkv, args.profile_outliers)
    v, do = draw(Hkv, False), draw(Hq, False)
    scale = D ** -0.5
    o, lse = ops.attn_fwd(q, k, v, causal=True, scale=scale)
    if args.profile_op == "fwd8":
        # the e4m3 forward on the same inputs quantised per tensor (descale = max|x| / 448)
        def q8(t):
            d = float(t.abs().max().float()) / 448.0
            return (t.float() / d).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn), d
        (q8_, qd), (k8_, kd), (v8_, vd) = q8(q), q8(k), q8(v)
        for _ in range(2):
            ops.attn_fwd_fp8(q8_, k8_, v8_, qd, kd, vd, causal=True, scale=scale, out=o, lse=lse)
    if args.profile_op in ("fwd", "both"):
        ops.attn_fwd(q, k, v, causal=True, scale=scale, out=o, lse=lse)
    if args.profile_op in ("bwd", "both"):
        ops.attn_bwd(q, k, v, o, lse, do, causal=True, scale=scale)
    torch.cuda.synchronize()
    st, site = capi.attn_device_status(None)
    if st != capi.ATTN_OK:
        raise RuntimeError(f"device status {capi.strerror(st)} site={site:#x}")
    print(json.dumps({"profile_case": [B, Hq, Hkv, S, D], "op": args.profile_op,
                      "outliers": bool(args.profile_outliers), "status": "ok"}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile", default=None, metavar="B,Hq,Hkv,S,D",
                    help="one launch on a reduced synthetic problem, for ncu captures")
    ap.add_argument("--profile-op", default="both",
                    choices=["fwd", "fwd8", "bwd", "both", "decode", "merge", "relayout"])
    ap.add_argument("--profile-outliers", action="store_true")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the e4m3 forward measurement")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode-attention measurements")
    ap.add_argument("--no-ulysses", action="store_true",
                    help="skip the Ulysses measurements (relayout kernel, 1-GPU Ulysses step)")
    ap.add_argument("--no-ring", action="store_true",
                    help="skip the Ring-attention measurements (merge kernel, 1-GPU ring forward)")
    args = ap.parse_args()
    if args.profile:
        return run_profile_case(args)
    w = I.workload(args.workload)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
