// attn_merge.cuh -- exact merge of partial attention results (o_p, lse_p) computed over
// disjoint key sets of the same queries.
//
// Page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠 FlashAttention
// 不够？那就加上序列并行", subsection "Ring-Attention" (and page "ms-swift支持GPU显存碎片整理
// 提升利用率", its Ring-Attention passage): the key/value sequence is split into chunks that
// travel around a ring of devices, and each device accumulates the partial attention of its
// queries over every chunk that passes by.  Because the forward kernel also returns the
// per-row natural log-sum-exp, those partials combine exactly:
//     lse = ln sum_p exp(lse_p),       o = sum_p exp(lse_p - lse) * o_p.
// A partial with lse_p = -inf saw no key and carries no weight; a row whose partials are
// all -inf gets o = 0 and lse = -inf.
//
// HBM-bound: per row it reads nparts * (2*D + 4) bytes and writes 2*D + 4.  Each row of o
// is D contiguous bf16 (2*D bytes) handled by D/8 threads with one 16-byte load per
// partial; rows are visited in memory order of o (head fastest), so every warp reads and
// writes whole contiguous 256-byte runs.  The per-row lse (fp32, 4 bytes) is read by all
// threads of the row in one broadcast load.
#pragma once

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace attn_sm100 {
namespace merge {

constexpr int kMaxParts = 16;
constexpr int kThreads = 256;

struct Params {
  const uint4* o_parts[kMaxParts];    // [T][H][D] bf16 as groups of eight
  const float* lse_parts[kMaxParts];  // [B][H][S] fp32 (lse layout of the forward)
  uint4* o;                           // [T][H][D] bf16
  float* lse;                         // [B][H][S]
  int nparts;
  unsigned H, S;                      // T = B * S tokens
  unsigned rows;                      // T * H  (< 2^31, checked on the host)
};

__device__ __forceinline__ const uint4* part_o(const Params& p, int j) { return p.o_parts[j]; }
__device__ __forceinline__ const float* part_lse(const Params& p, int j) { return p.lse_parts[j]; }

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4 x, const float w) {
  const uint32_t u[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc[2 * k] = fmaf(w, __uint_as_float(u[k] << 16), acc[2 * k]);
    acc[2 * k + 1] = fmaf(w, __uint_as_float(u[k] & 0xffff0000u), acc[2 * k + 1]);
  }
}

// Weights and weighted sum of one row.  l[u], x[u] (u < NP) hold the already loaded lse and
// o groups of partials 0..NP-1.  Only the NP = 4 shape takes more partials (the host picks
// NP = nparts below 4); it loads them here, four at a time, into x.
template <int NP>
__device__ __forceinline__ void merge_row(const Params& p, const float (&l)[NP], uint4 (&x)[NP],
                                          unsigned li, size_t off, float (&acc)[8],
                                          float& lse_out) {
  constexpr bool kMore = NP == 4;
  float m = -INFINITY;
#pragma unroll
  for (int u = 0; u < NP; ++u) m = fmaxf(m, l[u]);
  if (kMore)
    for (int j = NP; j < p.nparts; ++j) m = fmaxf(m, part_lse(p, j)[li]);
  if (m == -INFINITY) return;  // nothing visible: o = 0, lse = -inf
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < NP; ++u) s += expf(l[u] - m);  // exp(-inf) = 0 for absent partials
  if (kMore)
    for (int j = NP; j < p.nparts; ++j) s += expf(part_lse(p, j)[li] - m);
  const float inv = 1.f / s;
  lse_out = m + logf(s);
#pragma unroll
  for (int u = 0; u < NP; ++u)
    if (u < p.nparts) acc_bf16x8(acc, x[u], expf(l[u] - m) * inv);
  if (kMore)
    for (int j0 = NP; j0 < p.nparts; j0 += NP) {
#pragma unroll
      for (int u = 0; u < NP; ++u)
        if (j0 + u < p.nparts) x[u] = __ldcs(part_o(p, j0 + u) + off);
#pragma unroll
      for (int u = 0; u < NP; ++u)
        if (j0 + u < p.nparts) acc_bf16x8(acc, x[u], expf(part_lse(p, j0 + u)[li] - m) * inv);
    }
}

// Grid-stride over groups of ROWS * kThreads / (D/8) rows; each thread owns one 16-byte
// column group of ROWS rows (kThreads / (D/8) rows apart).  The lse and o loads of the first
// NP partials of all ROWS rows leave together before any of them is used, so each thread
// keeps NP * ROWS 16-byte loads in flight (the host picks NP * ROWS = 4).
// The loop bound is uniform across the block, so every thread reaches the __syncwarp.  D/8
// divides 32, so the threads of a row sit in one warp: the barrier orders every read of a
// row's partials before any write of that row, which makes o == o_parts[0] and
// lse == lse_parts[0] (exact aliasing) safe.
template <int D, int NP, int ROWS>
__global__ void __launch_bounds__(kThreads) attn_merge_kernel(const __grid_constant__ Params p) {
  static_assert(32 % (D / 8) == 0, "a row must not straddle warps");
  constexpr unsigned TPR = D / 8;
  constexpr unsigned RPB = kThreads / TPR;
  const unsigned c = threadIdx.x % TPR;
  for (unsigned r0 = blockIdx.x * (RPB * ROWS); r0 < p.rows; r0 += gridDim.x * (RPB * ROWS)) {
    float l[ROWS][NP];
    uint4 x[ROWS][NP];
    unsigned li[ROWS];
    size_t off[ROWS];
    bool valid[ROWS];
#pragma unroll
    for (int k = 0; k < ROWS; ++k) {
      const unsigned r = r0 + k * RPB + threadIdx.x / TPR;
      valid[k] = r < p.rows;
      off[k] = size_t(r) * TPR + c;
      li[k] = 0;
#pragma unroll
      for (int u = 0; u < NP; ++u) l[k][u] = -INFINITY;
      if (valid[k]) {
        const unsigned t = r / p.H, h = r - t * p.H;
        const unsigned b = t / p.S, i = t - b * p.S;
        li[k] = (b * p.H + h) * p.S + i;
#pragma unroll
        for (int u = 0; u < NP; ++u)
          if (u < p.nparts) {
            l[k][u] = part_lse(p, u)[li[k]];
            x[k][u] = __ldcs(part_o(p, u) + off[k]);
          }
      }
    }
    float acc[ROWS][8];
    float lse_out[ROWS];
#pragma unroll
    for (int k = 0; k < ROWS; ++k) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
      lse_out[k] = -INFINITY;
      if (valid[k]) merge_row<NP>(p, l[k], x[k], li[k], off[k], acc[k], lse_out[k]);
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < ROWS; ++k) {
      if (!valid[k]) continue;
      uint4 y;
      y.x = pack_bf16x2(acc[k][0], acc[k][1]);
      y.y = pack_bf16x2(acc[k][2], acc[k][3]);
      y.z = pack_bf16x2(acc[k][4], acc[k][5]);
      y.w = pack_bf16x2(acc[k][6], acc[k][7]);
      __stcs(p.o + off[k], y);
      if (c == 0) p.lse[li[k]] = lse_out[k];
    }
  }
}

// Launch shapes: (partials loaded up front, rows per thread) for 1, 2 and >= 3 partials.
// The shapes with NP < 4 handle exactly NP partials.
constexpr int kVariants = 3;
constexpr int kVariantNP[kVariants] = {1, 2, 4};
constexpr int kVariantRows[kVariants] = {4, 2, 1};
inline int variant_for(int nparts) { return nparts == 1 ? 0 : nparts == 2 ? 1 : 2; }

}  // namespace merge
}  // namespace attn_sm100
