// umma_selftest.cuh -- one-tile GEMMs that exercise, in isolation, each operand
// layout the attention kernels rely on, so that a descriptor or TMEM-layout error
// shows up as a plain matrix mismatch:
//   mode 0  C[128x128] = A[128xD] B[128xD]^T      A, B K-major via TMA (the S = Q K^T MMA)
//   mode 1  C[128xD]   = bf16(P)[128x128] V[128xD] P written to TMEM by threads,
//                                                  V MN-major via TMA (the O += P V MMA)
//   mode 2  C[128xD]   = At^T[128x128] B[128xD]   At rows written by threads into the
//                                                  swizzled MN-major layout (the dQ = dS K MMA)
// One CTA of 128 threads; every wait is bounded.
#pragma once
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"

namespace attn_sm100 {
namespace selftest {

template <int D>
__global__ void __launch_bounds__(128, 1)
umma_selftest_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     int mode, const float* __restrict__ pin, const __nv_bfloat16* __restrict__ at,
                     float* __restrict__ cout, unsigned* status, unsigned long long timeout_ns) {
  constexpr int kSlab = 128 * 128;
  constexpr int TILE = 128 * D * 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sa = smem;                        // A tile (mode 0) or At (mode 2, 32 KB)
  uint8_t* sb = smem + 32768;                // B tile
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 32768 + TILE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 3);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = threadIdx.x;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{status, abort_flag, timeout_ns};

  if (threadIdx.x == 0) {
    const uint32_t bytes = (mode == 0 ? TILE : 0) + TILE;
    mbar_arrive_expect_tx(&bars[0], bytes);
    for (int hf = 0; hf < D / 64; ++hf) {
      if (mode == 0) tma_load_3d(&tm_a, &bars[0], sa + hf * kSlab, hf * 64, 0, 0);
      tma_load_3d(&tm_b, &bars[0], sb + hf * kSlab, hf * 64, 0, 0);
    }
  }
  if (mode == 1) {
    // P row r -> TMEM lane r, columns 128..191 as bf16 pairs
    const uint32_t tp = tmem_addr(tmem, warp * 32, 128);
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t pk[16];
      for (int i = 0; i < 16; ++i)
        pk[i] = pack_bf16x2(pin[r * 128 + ch * 32 + 2 * i], pin[r * 128 + ch * 32 + 2 * i + 1]);
      tmem_st16(tp + ch * 16, pk);
    }
    tmem_wait_st();
  }
  if (mode == 2) {
    // At row r (128 bf16 along M) -> MN-major swizzled layout, 64-row M blocks 16 KB apart
    uint8_t* row = sa + (r >> 3) * 1024 + (r & 7) * 128;
    const uint4* src = reinterpret_cast<const uint4*>(at + r * 128);
    for (int c16 = 0; c16 < 16; ++c16) {
      const int blk = c16 >> 3, chunk = c16 & 7;
      *reinterpret_cast<uint4*>(row + blk * 16384 + ((chunk ^ (r & 7)) << 4)) = src[c16];
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  bool ok = true;
  if (threadIdx.x == 0) {
    ok = mbar_wait(&bars[0], 0, wc, 0x300);
    if (ok) {
      tc_fence_after();
      const uint32_t ab = smem_u32(sa), bb = smem_u32(sb);
      if (mode == 0) {
        constexpr uint32_t id = idesc_bf16_f32(128, 128, 0, 0);
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
          mma_ss(tmem, sdesc_sw128(ab + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024), id, kk > 0);
        }
      } else if (mode == 1) {
        constexpr uint32_t id = idesc_bf16_f32(128, D, 0, 1);
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem, tmem + 128 + kk * 8, sdesc_sw128(bb + kk * 2048, kSlab, 1024), id, kk > 0);
      } else {
        constexpr uint32_t id = idesc_bf16_f32(128, D, 1, 1);
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem, sdesc_sw128(ab + kk * 2048, 16384, 1024), sdesc_sw128(bb + kk * 2048, kSlab, 1024),
                 id, kk > 0);
      }
    }
    mma_commit(&bars[1]);
  }
  ok = __all_sync(0xffffffffu, mbar_wait(&bars[1], 0, wc, 0x301));
  if (ok) {
    tc_fence_after();
    const int ncol = (mode == 0) ? 128 : D;
    const uint32_t tc = tmem_addr(tmem, warp * 32, 0);
    for (int ch = 0; ch < ncol / 32; ++ch) {
      uint32_t u[32];
      tmem_ld32(tc + ch * 32, u);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) cout[r * ncol + ch * 32 + i] = __uint_as_float(u[i]);
    }
  }
  if (threadIdx.x == 0) mbar_drain(&bars[0], 0, timeout_ns);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// e4m3 (kind::f8f6f4) layouts at D = 128, one 128 x 128 tile:
//   mode 3  C = A8 B8^T                A, B e4m3 [128 rows][128], K-major via TMA: four
//                                      MMAs of K = 32 (the S = Q K^T MMA of the fp8 forward)
//   mode 4  C = e4m3(256 P) V8          P fp32 [128][128] quantised and packed four per TMEM
//                                      column by the threads, V e4m3 [128 keys][128] MN-major
//                                      via TMA (the O += P V MMA); pq receives the e4m3 values
//                                      of 256 P as the threads read them back.
__global__ void __launch_bounds__(128, 1)
umma_selftest_fp8_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         int mode, const float* __restrict__ pin, float* __restrict__ pq,
                         float* __restrict__ cout, unsigned* status, unsigned long long timeout_ns) {
  constexpr int TILE = 128 * 128;  // bytes of one e4m3 tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sa = smem;
  uint8_t* sb = smem + TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * TILE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 3);
  const int warp = threadIdx.x >> 5, r = threadIdx.x;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{status, abort_flag, timeout_ns};

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bars[0], (mode == 3 ? TILE : 0) + TILE);
    if (mode == 3) tma_load_3d(&tm_a, &bars[0], sa, 0, 0, 0);
    tma_load_3d(&tm_b, &bars[0], sb, 0, 0, 0);
  }
  if (mode == 4) {
    // P row r -> TMEM lane r, columns 128..159: four e4m3 keys per 32-bit column
    const uint32_t tp = tmem_addr(tmem, warp * 32, 128);
    for (int ch = 0; ch < 2; ++ch) {
      uint32_t pk[16];
      for (int i = 0; i < 16; ++i) {
        const float* x = pin + r * 128 + ch * 64 + 4 * i;
        pk[i] = pack_e4m3x2(256.f * x[0], 256.f * x[1]) | (pack_e4m3x2(256.f * x[2], 256.f * x[3]) << 16);
        float a0, a1, a2, a3;
        unpack_e4m3x2(pk[i], a0, a1);
        unpack_e4m3x2(pk[i] >> 16, a2, a3);
        float* q = pq + r * 128 + ch * 64 + 4 * i;
        q[0] = a0; q[1] = a1; q[2] = a2; q[3] = a3;
      }
      tmem_st16(tp + ch * 16, pk);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  bool ok = true;
  if (threadIdx.x == 0) {
    ok = mbar_wait(&bars[0], 0, wc, 0x310);
    if (ok) {
      tc_fence_after();
      const uint32_t ab = smem_u32(sa), bb = smem_u32(sb);
      if (mode == 3) {
        constexpr uint32_t id = idesc_e4m3_f32(128, 128, 0, 0);
        for (int kk = 0; kk < 4; ++kk)
          mma_ss_f8(tmem, sdesc_sw128(ab + kk * 32, 16, 1024), sdesc_sw128(bb + kk * 32, 16, 1024), id, kk > 0);
      } else {
        constexpr uint32_t id = idesc_e4m3_f32(128, 128, 0, 1);
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_f8(tmem, tmem + 128 + kk * 8, sdesc_sw128(bb + kk * 4096, 16384, 1024), id, kk > 0);
      }
    }
    mma_commit(&bars[1]);
  }
  ok = __all_sync(0xffffffffu, mbar_wait(&bars[1], 0, wc, 0x311));
  if (ok) {
    tc_fence_after();
    const uint32_t tc = tmem_addr(tmem, warp * 32, 0);
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t u[32];
      tmem_ld32(tc + ch * 32, u);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) cout[r * 128 + ch * 32 + i] = __uint_as_float(u[i]);
    }
  }
  if (threadIdx.x == 0) mbar_drain(&bars[0], 0, timeout_ns);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace selftest
}  // namespace attn_sm100
