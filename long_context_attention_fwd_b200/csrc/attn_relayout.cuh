// attn_relayout.cuh -- block transpose for the layout changes around the all-to-alls of
// Ulysses sequence parallelism.
//
// Page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠 FlashAttention
// 不够？那就加上序列并行", subsection on Ulysses (and page "ms-swift长文本训练秘诀：Ulysses
// 并行技术解析"): every device starts with a slice of the sequence for all heads; an
// all-to-all regroups the data so that every device holds the whole sequence for a subset
// of the heads, attention runs locally, and a second all-to-all restores the sequence
// split.  An all-to-all sends contiguous chunk p to rank p, so the heads destined for one
// rank must first be gathered into one chunk, and after the exchange the chunks are
// interleaved back.  Both are the same operation on a [n_outer][n_inner] grid of
// equal-size blocks:
//     out[j][i] = in[i][j]      (i < n_outer, j < n_inner, each block `vec` x 16 bytes)
//
// HBM-bound copy: reads and writes each byte once.  Threads walk the OUTPUT in order, one
// 16-byte vector each, so stores are fully coalesced and loads are coalesced within each
// block (blocks are a head's row of D bf16 values or larger, >= 128 bytes).  Four vectors
// per thread are loaded before any is stored, to keep loads in flight.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace attn_sm100 {
namespace relayout {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct Params {
  const uint4* in;
  uint4* out;
  unsigned n_outer, n_inner;  // block grid of `in`: [n_outer][n_inner]
  unsigned vec;               // 16-byte vectors per block
  unsigned total;             // n_outer * n_inner * vec  (< 2^32, checked on the host)
};

__global__ void __launch_bounds__(kThreads) transpose_blocks_kernel(const __grid_constant__ Params p) {
  const unsigned stride = gridDim.x * blockDim.x;
  for (unsigned base = blockIdx.x * blockDim.x + threadIdx.x; base < p.total;
       base += kUnroll * stride) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const unsigned idx = base + u * stride;  // output vector index
      if (idx < p.total) {
        const unsigned blk = idx / p.vec, c = idx - blk * p.vec;
        const unsigned j = blk / p.n_outer, i = blk - j * p.n_outer;  // out block (j, i)
        v[u] = __ldcs(p.in + (size_t(i) * p.n_inner + j) * p.vec + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const unsigned idx = base + u * stride;
      if (idx < p.total) __stcs(p.out + idx, v[u]);
    }
  }
}

}  // namespace relayout
}  // namespace attn_sm100
