// attn_accum.cuh -- accumulation of block gradients for the Ring-Attention backward.
//
// Page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠 FlashAttention
// 不够？那就加上序列并行", subsection "Ring-Attention": each device computes the share of
// the result that its queries and the passing key/value block contribute.  In the backward
// those shares (bf16 outputs of the block-pair backward) are summed in fp32 and rounded to
// bf16 once at the end:
//     add_bf16_to_f32:  acc[i] = (init ? 0 : acc[i]) + x[i]
//     f32_to_bf16:      out[i] = bf16(in[i])   (round to nearest even)
// HBM-bound element-wise kernels: eight elements per thread and iteration (16 bytes of bf16,
// 32 bytes of fp32), grid-stride over one wave of resident blocks.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace attn_sm100 {
namespace accum {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) add_bf16_to_f32_kernel(float4* acc, const uint4* x,
                                                                    long long n8, int init) {
  for (long long i = blockIdx.x * (long long)kThreads + threadIdx.x; i < n8;
       i += (long long)gridDim.x * kThreads) {
    const uint4 v = __ldcs(x + i);
    float4 a = init ? make_float4(0.f, 0.f, 0.f, 0.f) : acc[2 * i];
    float4 b = init ? make_float4(0.f, 0.f, 0.f, 0.f) : acc[2 * i + 1];
    a.x += __uint_as_float(v.x << 16);
    a.y += __uint_as_float(v.x & 0xFFFF0000u);
    a.z += __uint_as_float(v.y << 16);
    a.w += __uint_as_float(v.y & 0xFFFF0000u);
    b.x += __uint_as_float(v.z << 16);
    b.y += __uint_as_float(v.z & 0xFFFF0000u);
    b.z += __uint_as_float(v.w << 16);
    b.w += __uint_as_float(v.w & 0xFFFF0000u);
    acc[2 * i] = a;
    acc[2 * i + 1] = b;
  }
}

__global__ void __launch_bounds__(kThreads) f32_to_bf16_kernel(uint4* out, const float4* in,
                                                                long long n8) {
  for (long long i = blockIdx.x * (long long)kThreads + threadIdx.x; i < n8;
       i += (long long)gridDim.x * kThreads) {
    const float4 a = __ldcs(in + 2 * i), b = __ldcs(in + 2 * i + 1);
    uint4 y;
    y.x = pack_bf16x2(a.x, a.y);
    y.y = pack_bf16x2(a.z, a.w);
    y.z = pack_bf16x2(b.x, b.y);
    y.w = pack_bf16x2(b.z, b.w);
    __stcs(out + i, y);
  }
}

}  // namespace accum
}  // namespace attn_sm100
