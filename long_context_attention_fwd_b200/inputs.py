"""Seeded synthetic inputs shared by the CUDA path, the oracle and the bench.

This module draws numbers and nothing else: it holds none of the attention
arithmetic, so both sides of every parity check can take their inputs from it
without sharing any of the method.

Generator (stated so that anyone can reproduce the bytes):

* SplitMix64 in counter form: draw ``i`` of a stream with key ``key`` is
  ``mix64(key + (i + 1) * 0x9E3779B97F4A7C15)`` where ``mix64`` is the published
  SplitMix64 finaliser (xor-shift 30 / multiply 0xBF58476D1CE4E5B9 / xor-shift 27 /
  multiply 0x94D049BB133111EB / xor-shift 31), all modulo 2**64.
* Uniforms: ``(z >> 11) * 2**-53`` in [0, 1); Box-Muller uses ``u1 = ((z >> 11) + 1) * 2**-53``
  in (0, 1] so that ``log(u1)`` is finite.
* Normals: Box-Muller on consecutive pairs of draws, both the cosine and the sine
  output are used (element ``2p`` gets the cosine, ``2p+1`` the sine of pair ``p``).
* bf16: the fp64 value is rounded to fp32 (numpy, round-to-nearest-even), then
  to bf16 with round-to-nearest-even on the fp32 bit pattern.
* Each tensor (q, k, v, dO, lengths, outlier mask) has its own stream key derived
  from the workload seed and a fixed tag, so tensors never share draws.

Workload recipes follow the shapes of Qwen2.5-7B attention (28 query heads, 4
key/value heads, head dim 128) at the 8K and 32K lengths the long-context
fine-tuning pages train at, packed variable-length sequences, and a head-dim-64
multi-head case with outlier tails.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream tags: one per tensor kind.
TAG_Q, TAG_K, TAG_V, TAG_DO, TAG_LEN, TAG_OUT_Q, TAG_OUT_K = 1, 2, 3, 4, 5, 6, 7
TAG_CACHE_LEN = 8

_CHUNK = 1 << 22


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tag: int) -> int:
    """Key of the stream for tensor kind ``tag`` under workload ``seed``."""
    with np.errstate(over="ignore"):
        z = np.array([(seed * 0x100000001B3 + tag * 0x2545F4914F6CDD1D) & 0xFFFFFFFFFFFFFFFF],
                     dtype=np.uint64)
        return int(_mix64(z)[0])


def raw_u64(key: int, start: int, count: int) -> np.ndarray:
    """Draws ``start .. start+count-1`` of stream ``key`` as uint64."""
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix64(np.uint64(key) + idx * _GOLDEN)


def uniform(key: int, count: int, start: int = 0) -> np.ndarray:
    """``count`` uniforms in [0, 1) (fp64)."""
    z = raw_u64(key, start, count)
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _normal_pairs(key: int, p0: int, p1: int) -> np.ndarray:
    z = raw_u64(key, 2 * p0, 2 * (p1 - p0))
    u1 = ((z[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * math.pi * u2
    pair = np.empty(2 * (p1 - p0), dtype=np.float64)
    pair[0::2] = r * np.cos(t)
    pair[1::2] = r * np.sin(t)
    return pair


def normal(key: int, count: int) -> np.ndarray:
    """``count`` standard normals (fp64), Box-Muller on pairs of draws.  Chunks are
    independent (counter-based stream), so they are filled by a thread pool."""
    out = np.empty(count, dtype=np.float64)
    npairs = (count + 1) // 2
    bounds = [(p0, min(npairs, p0 + _CHUNK)) for p0 in range(0, npairs, _CHUNK)]

    def fill(b):
        p0, p1 = b
        pair = _normal_pairs(key, p0, p1)
        n = min(count - 2 * p0, pair.size)
        out[2 * p0:2 * p0 + n] = pair[:n]

    if len(bounds) > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4)) as ex:
            list(ex.map(fill, bounds))
    else:
        for b in bounds:
            fill(b)
    return out


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64/fp32 array -> bf16 bit patterns (uint16), round-to-nearest-even."""
    f = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((f >> np.uint32(16)) & np.uint32(1))
    return ((f + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16(key: int, shape, mult: float = 1.0,
                outlier_key: Optional[int] = None, outlier_p: float = 0.0,
                outlier_mult: float = 1.0) -> np.ndarray:
    """Seeded N(0,1)*mult tensor with optional Bernoulli(p) outliers scaled by
    ``outlier_mult`` (applied before rounding), returned as bf16 bits (uint16)."""
    count = int(np.prod(shape))
    out = np.empty(count, dtype=np.uint16)
    base = normal(key, count)
    if mult != 1.0:
        base *= mult
    if outlier_key is not None and outlier_p > 0.0:
        for c0 in range(0, count, _CHUNK):
            c1 = min(count, c0 + _CHUNK)
            u = uniform(outlier_key, c1 - c0, start=c0)
            seg = base[c0:c1]
            seg[u < outlier_p] *= outlier_mult
    for c0 in range(0, count, _CHUNK * 4):
        c1 = min(count, c0 + _CHUNK * 4)
        out[c0:c1] = to_bf16_bits(base[c0:c1])
    return out.reshape(shape)


def varlen_lengths(seed: int, total: int, lo: int, hi: int) -> List[int]:
    """Lengths uniform on [lo, hi] (inclusive), drawn until their sum reaches
    ``total``; the last one is cut so that the lengths sum to ``total`` exactly."""
    key = stream_key(seed, TAG_LEN)
    lens: List[int] = []
    acc = 0
    i = 0
    while acc < total:
        u = uniform(key, 1, start=i)[0]
        i += 1
        L = lo + int(math.floor(u * (hi - lo + 1)))
        L = min(L, total - acc)
        lens.append(L)
        acc += L
    return lens


def cu_seqlens_from(lengths: List[int]) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64)).astype(np.int32)
    return cu


@dataclass
class Workload:
    """One attention problem: shapes, masking and the value recipe."""
    name: str
    B: int
    Hq: int
    Hkv: int
    S: int                      # tokens per sequence (dense) or total tokens T (varlen)
    D: int
    causal: bool = True
    qkv_mult: float = 1.0
    do_mult: float = 1.0
    outlier_p: float = 0.0      # Bernoulli probability per element of q and k
    outlier_mult: float = 1.0
    varlen: Optional[List[int]] = None   # sequence lengths when packed
    seed: int = 20261202
    scale: Optional[float] = None
    extra: dict = field(default_factory=dict)

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)

    @property
    def tokens(self) -> int:
        return self.S if self.varlen is not None else self.B * self.S

    @property
    def nseq(self) -> int:
        return len(self.varlen) if self.varlen is not None else self.B

    def seq_lengths(self) -> List[int]:
        return list(self.varlen) if self.varlen is not None else [self.S] * self.B

    def cu_seqlens(self) -> Optional[np.ndarray]:
        return None if self.varlen is None else cu_seqlens_from(self.varlen)


def make_inputs(w: Workload, with_do: bool = True) -> dict:
    """bf16 bit tensors for a workload: q [T,Hq,D], k/v [T,Hkv,D], dO [T,Hq,D]
    (T = B*S for dense, the packed total otherwise), plus cu_seqlens (int32)."""
    T = w.tokens
    s = w.seed
    oq = stream_key(s, TAG_OUT_Q) if w.outlier_p > 0 else None
    ok = stream_key(s, TAG_OUT_K) if w.outlier_p > 0 else None
    q = normal_bf16(stream_key(s, TAG_Q), (T, w.Hq, w.D), w.qkv_mult, oq, w.outlier_p, w.outlier_mult)
    k = normal_bf16(stream_key(s, TAG_K), (T, w.Hkv, w.D), w.qkv_mult, ok, w.outlier_p, w.outlier_mult)
    v = normal_bf16(stream_key(s, TAG_V), (T, w.Hkv, w.D), w.qkv_mult)
    out = {"q": q, "k": k, "v": v, "cu_seqlens": w.cu_seqlens()}
    if with_do:
        out["do"] = normal_bf16(stream_key(s, TAG_DO), (T, w.Hq, w.D), w.do_mult)
    return out


def _varlen_32k_lengths() -> List[int]:
    return varlen_lengths(20261202 + 3, 32768, 512, 8192)


def workloads() -> List[Workload]:
    """The five named workloads, smallest first."""
    return [
        Workload("tiny_S256_D64_mha2", B=1, Hq=2, Hkv=2, S=256, D=64, causal=True,
                 qkv_mult=1.0, do_mult=1.0, seed=20261202 + 0),
        Workload("qwen2.5-7b_gqa28x4_S8192_D128", B=1, Hq=28, Hkv=4, S=8192, D=128,
                 causal=True, qkv_mult=0.5, do_mult=1.0, seed=20261202 + 1),
        Workload("qwen2.5-7b_gqa28x4_S32768_D128", B=1, Hq=28, Hkv=4, S=32768, D=128,
                 causal=True, qkv_mult=0.5, do_mult=1.0, seed=20261202 + 2),
        Workload("varlen_T32768_L512-8192_gqa28x4_D128", B=0, Hq=28, Hkv=4, S=32768, D=128,
                 causal=True, qkv_mult=0.5, do_mult=1.0, seed=20261202 + 3,
                 varlen=_varlen_32k_lengths()),
        Workload("mha32_B4_S16384_D64_outliers", B=4, Hq=32, Hkv=32, S=16384, D=64,
                 causal=True, qkv_mult=1.0, do_mult=1.0, outlier_p=0.01, outlier_mult=8.0,
                 seed=20261202 + 4),
    ]


def workload(name_or_index) -> Workload:
    ws = workloads()
    if isinstance(name_or_index, int):
        return ws[name_or_index]
    for w in ws:
        if w.name == name_or_index:
            return w
    raise KeyError(name_or_index)


def flop_fwd(w: Workload) -> float:
    """Forward FLOP convention: 4*S^2*D*Hq per sequence, halved when causal;
    for packed sequences the same per sequence and summed."""
    tot = 0.0
    for L in w.seq_lengths():
        f = 4.0 * L * L * w.D * w.Hq
        tot += f / 2.0 if w.causal else f
    return tot


def flop_bwd(w: Workload) -> float:
    """Backward FLOP convention: 2.5x the forward count."""
    return 2.5 * flop_fwd(w)


# ---------------------------------------------------------------- decode over a KV cache
@dataclass
class DecodeWorkload:
    """One decode step: a new query token per sequence against its key/value cache.
    q [B,Hq,D]; k/v cache [B,Lmax,Hkv,D]; cache_len [B] (entries past it are not used)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Lmax: int
    D: int
    lens: List[int]
    qkv_mult: float = 0.5
    seed: int = 20261202
    scale: Optional[float] = None

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)

    def cache_bytes(self) -> int:
        """Bytes of K and V the step must read: sum of lengths x Hkv x D x 2 bytes x 2."""
        return int(sum(self.lens)) * self.Hkv * self.D * 2 * 2

    def io_bytes(self) -> int:
        """Algorithmic bytes of one step: the cache read, q read, o and lse written."""
        return self.cache_bytes() + self.B * self.Hq * (self.D * 2 * 2 + 4)


def decode_lengths(seed: int, B: int, lo: int, hi: int) -> List[int]:
    """B cache lengths uniform on [lo, hi] (inclusive)."""
    u = uniform(stream_key(seed, TAG_CACHE_LEN), B)
    return [lo + int(math.floor(x * (hi - lo + 1))) for x in u]


def make_decode_inputs(w: DecodeWorkload, poison_tail: bool = True) -> dict:
    """bf16 bit tensors q [B,Hq,D], k/v [B,Lmax,Hkv,D] and cache_len int32 [B].  With
    poison_tail, cache entries past each length hold bf16 NaN, so that any read of them
    shows up in the output."""
    s = w.seed
    q = normal_bf16(stream_key(s, TAG_Q), (w.B, w.Hq, w.D), w.qkv_mult)
    k = normal_bf16(stream_key(s, TAG_K), (w.B, w.Lmax, w.Hkv, w.D), w.qkv_mult)
    v = normal_bf16(stream_key(s, TAG_V), (w.B, w.Lmax, w.Hkv, w.D), w.qkv_mult)
    if poison_tail:
        for b, L in enumerate(w.lens):
            k[b, L:] = 0x7FC0
            v[b, L:] = 0x7FC0
    return {"q": q, "k": k, "v": v, "cache_len": np.asarray(w.lens, dtype=np.int32)}


def decode_workloads() -> List[DecodeWorkload]:
    """Decode steps at the pages' 32K deployment context with Qwen2.5-7B attention shapes,
    and a small case whose lengths sit on and around the 128-key tile edges."""
    return [
        DecodeWorkload("decode_edges_B8_gqa8x2_D64", B=8, Hq=8, Hkv=2, Lmax=700, D=64,
                       lens=[0, 1, 127, 128, 129, 255, 700, 513], qkv_mult=1.0,
                       seed=20261202 + 10),
        DecodeWorkload("qwen2.5-7b_decode_B1_L32768", B=1, Hq=28, Hkv=4, Lmax=32768, D=128,
                       lens=[32768], seed=20261202 + 11),
        DecodeWorkload("qwen2.5-7b_decode_B16_L16K-32K", B=16, Hq=28, Hkv=4, Lmax=32768, D=128,
                       lens=decode_lengths(20261202 + 12, 16, 16384, 32768),
                       seed=20261202 + 12),
    ]


def decode_workload(name_or_index) -> DecodeWorkload:
    ws = decode_workloads()
    if isinstance(name_or_index, int):
        return ws[name_or_index]
    for w in ws:
        if w.name == name_or_index:
            return w
    raise KeyError(name_or_index)
