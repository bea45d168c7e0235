// attn_bwd.cuh -- fused attention backward for sm_100a.
//
// The page "ms-swift集成FlashAttention 2/3" (section "为什么传统注意力这么'吃'显存",
// why standard attention eats so much memory) notes that the backward pass of the
// native implementation needs the S x S intermediates again, cached or recomputed;
// the fused kernel (section "FlashAttention 如何破局") keeps none of them in HBM.
// Here the backward recomputes the probabilities tile by tile from the per-row
// log-sum-exp the forward saved:
//     P = exp(scale * Q K^T - LSE),  dP = dO V^T,  Delta = rowsum(dO * O),
//     dS = P * (dP - Delta),  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// Kernels:
//   bwd_preprocess  -Delta and -LSE*log2(e) per query row into a tile-padded workspace
//                   (rows past a sequence end get LSE = +inf, so their P is exactly 0),
//                   and zeroes the fp32 dQ accumulator rows.
//   attn_bwd_kernel KV-stationary: one CTA holds a 128-key tile of one kv head (K, V in
//                   shared memory, dK/dV accumulators in TMEM) and loops over the query
//                   heads of its group and the 128-row query tiles that see it.
//                   Per query tile: S^T = K Q^T, dP^T = V dO^T, dV += P^T dO (P^T read
//                   from TMEM as bf16), dK += dS^T Q and dQ_tile = dS K (both reading the
//                   one bf16 dS buffer in shared memory, K-major and MN-major), and dQ_tile
//                   is reduced into the fp32 accumulator with coalesced vector reductions.
//                   dK/dV stay deterministic.
//   dq_convert      dq = bf16(scale * accumulator).
//
// Warps: 0-3 and 4-7 compute P^T and dS^T (one thread per key row; warps 0-3 take query
// columns 0-63 of the tile, warps 4-7 columns 64-127, which halves the per-thread chain
// that paces the loop), 8-11 drain dQ from TMEM and reduce it into the accumulator,
// 12 is the TMA producer, 13 issues the MMAs, 14-15 only complete the control warpgroup
// for the register split.
#pragma once
#include <cuda_bf16.h>
#include "attn_common.cuh"
#include "sm100_ptx.cuh"

namespace attn_sm100 {
namespace bwd {

constexpr int kThreads = 512;    // 16 warps; warps 14-15 only complete the control warpgroup
constexpr int kWarpTMA = 12;
constexpr int kWarpMMA = 13;
// Register split (setmaxnreg): the launch gives every thread 128 registers
// (512 x 128 = 65536); the control warpgroup (warps 12-15) drops to 72 and the three
// compute warpgroups (P/dS, P/dS, dQ drain) rise to 144:
// 128 x 72 + 384 x 144 = 64512 <= 65536 (the smallest split ptxas compiles without spills).
constexpr int kRegsLaunch = 128;
constexpr int kRegsControl = 72;
constexpr int kRegsCompute = 144;
static_assert(128 * kRegsControl + 384 * kRegsCompute <= kThreads * kRegsLaunch, "register split");
constexpr int kSlab = 128 * 128;
// The P/dS warpgroups hand dS over in four chunks of 32 query columns (1), so that the dK
// MMA runs while the later chunks are computed, or all at once (0).
#ifndef ATTN_BWD_DSCHUNK
#define ATTN_BWD_DSCHUNK 1
#endif
constexpr int kDsChunks = ATTN_BWD_DSCHUNK ? 4 : 1;
// At D = 128 (dQ in the dP^T columns), dQ is issued as soon as the last dS chunk lands,
// before that chunk's dK steps (1), so the dQ drain -- which the next tile's dP^T waits
// for -- starts earlier; or after all of dK (0).  At D = 64 dQ has columns of its own and
// always comes after dK.
#ifndef ATTN_BWD_DQFIRST
#define ATTN_BWD_DQFIRST 1
#endif

struct Params {
  SeqView sv;
  float* dq_acc;          // [Hq][ntile][D/4][128][4] fp32: one contiguous block per query tile
  const float* lse2;      // [Hq][ntile][128]: -LSE * log2(e) (negated: the P step adds it)
  const float* delta;     // [Hq][ntile][128]: -Delta (negated: the dS step adds it)
  __nv_bfloat16* dk;      // [T][Hkv][D]
  __nv_bfloat16* dv;
  int Hq, Hkv, G, T, causal;
  int ntile;              // tiles per head in the workspace = (T >> 7) + nseq
  int group_major;        // CTA order: 1 = kv head outermost, 0 = kv head innermost
  float scale_log2;
  float scale;
  unsigned* status;
  unsigned long long timeout_ns;
};

template <int D>
struct Cfg {
  static constexpr int TILE = 128 * D * 2;  // one 128-row bf16 tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;        // 2 stages
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;   // 2 stages
  static constexpr int OFF_DS = OFF_DO + 2 * TILE;  // 128 x 128 bf16, MN-major for the dQ MMA
  static constexpr int OFF_LSE = OFF_DS + 128 * 128 * 2;  // 2 stages x 128 fp32
  static constexpr int OFF_DELTA = OFF_LSE + 2 * 512;
  static constexpr int OFF_BAR = OFF_DELTA + 2 * 512;
  // kv_full, q_full[2], q_empty[2], do_full[2], do_empty[2], s_full, dp_full, p_full,
  // dq_full, dq_free, dkv_final, drain, ds_full[kDsChunks]
  static constexpr int NBAR = 16 + kDsChunks;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int kMaxDyn = 232448;
  static constexpr int SLACK = (SMEM_BYTES + 1024 <= kMaxDyn) ? 1024 : (kMaxDyn - SMEM_BYTES);
  static constexpr int SMEM_ALLOC = SMEM_BYTES + SLACK;
  static constexpr uint32_t TMEM_COLS = 512;
  // D = 128 fills TMEM with S^T, dP^T, dV, dK, so the dQ tile shares dP^T's columns and
  // the next dP^T waits for the dQ drain.  D = 64 leaves room for dQ columns of its own.
  static constexpr bool DQ_ALIAS = D == 128;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  static constexpr uint32_t COL_DQ = DQ_ALIAS ? COL_DP : 256 + 2 * D;
  static_assert(COL_DQ + D <= TMEM_COLS && (DQ_ALIAS || COL_DQ >= COL_DK + D), "TMEM budget");
  static_assert(SMEM_BYTES <= kMaxDyn, "shared memory budget");
};

enum : unsigned {
  kSiteKV = 0x200, kSiteQEmpty, kSiteQFull, kSiteSFull, kSiteDpFull, kSitePFull, kSiteDsFull,
  kSiteDqFull, kSiteDqFree, kSiteFinal, kSiteDoEmpty, kSiteDoFull
};

// dQ tile layout (workspace): element (row r, column d) of a 128-row tile lives at float
// offset ((d / 4) * 128 + r) * 4 + d % 4, so the 32 threads of a warp, which own 32
// consecutive rows, reduce 16-byte chunks into 512 contiguous bytes at a time.
__host__ __device__ constexpr size_t dq_tile_offset(int r, int d) {
  return (size_t(d >> 2) * 128 + r) * 4 + (d & 3);
}

// ---------------------------------------------------------------- preprocess
// grid (ntile, Hq), 128 threads: one thread per query row of one 128-row tile.
// Writes -Delta_i = -(dO_i . O_i) and -LSE_i * log2(e) into the tile-padded workspace
// (0 / -inf for rows past the sequence end, so their probabilities are exactly 0)
// and zeroes the tile's fp32 dQ block.  Both are stored negated because the main
// kernel adds them (one packed FMA / add, with no separate negation).
template <int D>
__global__ void __launch_bounds__(128)
bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                      const float* __restrict__ lse, float* __restrict__ lse2,
                      float* __restrict__ delta, float* __restrict__ dq_acc, SeqView sv, int Hq,
                      int T, int ntile) {
  int seq, m, start, len;
  if (!locate_block<7>(sv, blockIdx.x, seq, m, start, len)) return;
  const int h = blockIdx.y;
  const int r = threadIdx.x;
  const int qpos = m * 128 + r;
  float dl = 0.f, l2 = INFINITY;
  if (qpos < len) {
    const size_t row = (size_t(start + qpos) * Hq + h) * D;
    const uint4* po = reinterpret_cast<const uint4*>(o + row);
    const uint4* pd = reinterpret_cast<const uint4*>(dout + row);
    float acc = 0.f;
#pragma unroll 4
    for (int i = 0; i < D / 8; ++i) {
      const uint4 a = __ldg(po + i), b = __ldg(pd + i);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 fa = __bfloat1622float2(a2[k]);
        const float2 fb = __bfloat1622float2(b2[k]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
    dl = acc;
    const size_t li = sv.cu ? size_t(h) * T + start + qpos : (size_t(seq) * Hq + h) * sv.S + qpos;
    l2 = lse[li] * 1.4426950408889634f;
  }
  const size_t wi = (size_t(h) * ntile + blockIdx.x) * 128 + r;
  lse2[wi] = -l2;
  delta[wi] = -dl;
  float4* z = reinterpret_cast<float4*>(dq_acc + (size_t(h) * ntile + blockIdx.x) * 128 * D);
#pragma unroll 4
  for (int i = 0; i < D / 4; ++i) z[i * 128 + r] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------- dq convert
// grid (ntile, Hq), 256 threads: dq[t][h][:] = bf16(scale * dQ tile rows), 8 columns per item.
template <int D>
__global__ void __launch_bounds__(256)
dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, SeqView sv,
                  int Hq, int ntile, float scale) {
  int seq, m, start, len;
  if (!locate_block<7>(sv, blockIdx.x, seq, m, start, len)) return;
  const int h = blockIdx.y;
  const float4* blk = reinterpret_cast<const float4*>(acc + (size_t(h) * ntile + blockIdx.x) * 128 * D);
  constexpr int G8 = D / 8;
  for (int idx = threadIdx.x; idx < 128 * G8; idx += 256) {
    const int r = idx / G8, c8 = idx % G8;
    const int qpos = m * 128 + r;
    if (qpos >= len) continue;
    const float4 a = __ldg(blk + (2 * c8) * 128 + r);
    const float4 b = __ldg(blk + (2 * c8 + 1) * 128 + r);
    uint4 out;
    out.x = pack_bf16x2(a.x * scale, a.y * scale);
    out.y = pack_bf16x2(a.z * scale, a.w * scale);
    out.z = pack_bf16x2(b.x * scale, b.y * scale);
    out.w = pack_bf16x2(b.z * scale, b.w * scale);
    *reinterpret_cast<uint4*>(dq + (size_t(start + qpos) * Hq + h) * D + 8 * c8) = out;
  }
}

// ---------------------------------------------------------------- main kernel
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad > uint32_t(C::SLACK)) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (sequence, kv head, 128-key tile); low tiles (most query tiles) first.
  // Two orders of the same items.  Kv head innermost keeps the longest tiles of every
  // group in the first wave.  Kv head outermost (dense batches only) keeps the CTAs
  // resident at a time within one or two groups, so the dQ tiles they reduce into stay
  // in L2 while the CTAs drift apart along the queries; the host takes it when one
  // group's tiles fill a wave, so the longest tiles of later groups do not start late.
  // Within a group of a dense batch the sequences are innermost (tile n of every
  // sequence before tile n + 1); packed batches go sequence by sequence.
  const unsigned nt = unsigned(p.ntile);
  const int g = p.group_major ? int(blockIdx.x / nt) : int(blockIdx.x % unsigned(p.Hkv));
  const int tix = p.group_major ? int(blockIdx.x % nt) : int(blockIdx.x / unsigned(p.Hkv));
  int seq, n, start, len;
  if (p.sv.cu) {
    if (!locate_block<7>(p.sv, tix, seq, n, start, len)) return;
  } else {
    seq = tix % p.sv.nseq;
    n = tix / p.sv.nseq;
    start = seq * p.sv.S;
    len = p.sv.S;
    if (n >= (len + 127) >> 7) return;
  }
  const int nq = (len + 127) >> 7;
  const int m0 = p.causal ? n : 0;
  const int per_head = nq - m0;
  const int iters = p.G * per_head;
  const int tile_base = (start >> 7) + seq;  // workspace tile index of query tile 0
  // Iteration order: query tiles from the last one down to m0, the group's query heads
  // innermost.  CTAs of one wave then start on the same tile and advance in step, so
  // the dQ tiles they reduce into (and the Q/dO tiles they read) stay in L2.

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;     // [2] Q tile + LSE + Delta of a stage landed
  uint64_t* q_empty = bars + 3;    // [2] the stage's Q buffer may be refilled
  uint64_t* do_full = bars + 5;    // [2] dO tile landed
  uint64_t* do_empty = bars + 7;   // [2] the stage's dO buffer may be refilled
  uint64_t* s_full = bars + 9;
  uint64_t* dp_full = bars + 10;
  uint64_t* p_full = bars + 11;
  uint64_t* dq_full = bars + 12;
  uint64_t* dq_free = bars + 13;   // dQ columns of TMEM read out
  uint64_t* dkv_final = bars + 14;
  uint64_t* drain = bars + 15;
  uint64_t* ds_full = bars + 16;   // [kDsChunks] chunk c of dS is in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* lse_s = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* delta_s = reinterpret_cast<float*>(smem + C::OFF_DELTA);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&do_full[i], 1);
      mbar_init(&do_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 8);
    for (int c = 0; c < kDsChunks; ++c) mbar_init(&ds_full[c], kDsChunks == 1 ? 8 : 4);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);
    mbar_init(dkv_final, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == kWarpMMA) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kWarpTMA && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.status, abort_flag, p.timeout_ns};

  if (warp >= 12) {
    reg_dealloc<kRegsControl>();
    if (warp == kWarpTMA && lane == 0) {
      // ---------------------------------------------------------- producer
      int nq_issued = 0, ndo_issued = 0;
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
      for (int hf = 0; hf < D / 64; ++hf) {
        tma_load_3d(&tm_k, kv_full, smem + C::OFF_K + hf * kSlab, hf * 64, g, start + 128 * n);
        tma_load_3d(&tm_v, kv_full, smem + C::OFF_V + hf * kSlab, hf * 64, g, start + 128 * n);
      }
      for (int it = 0; it < iters; ++it) {
        const int st = it & 1;
        const uint32_t ph = ((it >> 1) & 1) ^ 1;
        const int hq = g * p.G + it % p.G;
        const int m = nq - 1 - it / p.G;
        // dO first: its stage frees at the dP MMA, earlier than Q's (freed at the dK MMA).
        if (!mbar_wait(&do_empty[st], ph, wc, kSiteDoEmpty)) break;
        mbar_arrive_expect_tx(&do_full[st], C::TILE);
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_3d(&tm_do, &do_full[st], smem + C::OFF_DO + st * C::TILE + hf * kSlab, hf * 64,
                      hq, start + 128 * m);
        ++ndo_issued;
        if (!mbar_wait(&q_empty[st], ph, wc, kSiteQEmpty)) break;
        mbar_arrive_expect_tx(&q_full[st], C::TILE + 1024);
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_3d(&tm_q, &q_full[st], smem + C::OFF_Q + st * C::TILE + hf * kSlab, hf * 64, hq,
                      start + 128 * m);
        const size_t wi = (size_t(hq) * p.ntile + tile_base + m) * 128;
        bulk_load(lse_s + st * 128, p.lse2 + wi, 512, &q_full[st]);
        bulk_load(delta_s + st * 128, p.delta + wi, 512, &q_full[st]);
        ++nq_issued;
      }
      mbar_drain(kv_full, 0, drain_ns(abort_flag, p.timeout_ns));
      for (int st = 0; st < 2; ++st) {
        const int cq = nq_issued > st ? (nq_issued - 1 - st) / 2 + 1 : 0;
        const int cd = ndo_issued > st ? (ndo_issued - 1 - st) / 2 + 1 : 0;
        if (cq) mbar_drain(&q_full[st], (cq - 1) & 1, drain_ns(abort_flag, p.timeout_ns));
        if (cd) mbar_drain(&do_full[st], (cd - 1) & 1, drain_ns(abort_flag, p.timeout_ns));
      }
    } else if (warp == kWarpMMA && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);   // S^T, dP^T
      constexpr uint32_t idKV = idesc_bf16_f32(128, D, 0, 1);    // dV, dK (A from TMEM)
      constexpr uint32_t idQ = idesc_bf16_f32(128, D, 1, 1);     // dQ (A = dS, MN-major)
      const uint32_t kb = smem_u32(smem + C::OFF_K);
      const uint32_t vb = smem_u32(smem + C::OFF_V);
      const uint32_t dsb = smem_u32(smem + C::OFF_DS);
      auto issue_T = [&](uint32_t col, uint32_t ab, uint32_t bb) {  // [128 x 128] = A B^T over D
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
          mma_ss(tmem + col, sdesc_sw128(ab + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024), idS,
                 kk > 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(kv_full, 0, wc, kSiteKV) && mbar_wait(&q_full[0], 0, wc, kSiteQFull);
      if (ok && iters > 0) {
        tc_fence_after();
        issue_T(C::COL_S, kb, smem_u32(smem + C::OFF_Q));
        mma_commit(s_full);
      }
      // P^T halves sit in TMEM columns [0, 32) and [96, 128) of the S^T region (warps 0-3 /
      // warps 4-7, bf16 pairs): A-operand column of 16-row step kk.
      auto a_col = [](int kk) -> uint32_t { return kk < 4 ? kk * 8 : 96 + (kk - 4) * 8; };
      // Per query tile: dP^T first (it needs neither P nor dS, so the dS step can start as
      // soon as P is done), then dV, the next S^T, dK and dQ.
      for (int it = 0; it < iters && ok; ++it) {
        const int st = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        const uint32_t qb = smem_u32(smem + C::OFF_Q + st * C::TILE);
        const uint32_t dob = smem_u32(smem + C::OFF_DO + st * C::TILE);
        if (!(ok = mbar_wait(&do_full[st], ph, wc, kSiteDoFull))) break;
        if (C::DQ_ALIAS && it > 0 && !(ok = mbar_wait(dq_free, (it - 1) & 1, wc, kSiteDqFree))) break;
        tc_fence_after();
        issue_T(C::COL_DP, vb, dob);  // dP^T = V dO^T (over dS^T of the previous tile, or dQ)
        mma_commit(dp_full);
        if (!(ok = mbar_wait(p_full, it & 1, wc, kSitePFull))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dV += P^T dO
          mma_ts(tmem + C::COL_DV, tmem + C::COL_S + a_col(kk), sdesc_sw128(dob + kk * 2048, kSlab, 1024),
                 idKV, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&do_empty[st]);
        if (it + 1 < iters) {
          if (!(ok = mbar_wait(&q_full[st ^ 1], ((it + 1) >> 1) & 1, wc, kSiteQFull))) break;
          tc_fence_after();
          issue_T(C::COL_S, kb, smem_u32(smem + C::OFF_Q + (st ^ 1) * C::TILE));  // next S^T
          mma_commit(s_full);
        }
        // dK += dS^T Q (dS^T K-major in shared memory), chunk by chunk as dS arrives:
        // chunk c covers query K steps 2c, 2c + 1 (warpgroup c / 2, local half c % 2).  The
        // two warpgroups run side by side, so their first halves are taken first.
        auto chunk_of = [](int j) { return kDsChunks == 4 ? ((j & 1) << 1) | (j >> 1) : 0; };
        auto issue_dK = [&](int c) {
#pragma unroll
          for (int k2 = 0; k2 < 8 / kDsChunks; ++k2) {
            const int kk = c * (8 / kDsChunks) + k2;
            mma_ss(tmem + C::COL_DK, sdesc_sw128(dsb + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024),
                   sdesc_sw128(qb + kk * 2048, kSlab, 1024), idKV, (it > 0 || kk > 0) ? 1u : 0u);
          }
        };
        constexpr bool kDqFirst = ATTN_BWD_DQFIRST && C::DQ_ALIAS;
        constexpr int kEarly = kDqFirst ? kDsChunks - 1 : kDsChunks;  // dK chunks before dQ
        for (int j = 0; j < kDsChunks && ok; ++j) {
          if (!(ok = mbar_wait(&ds_full[chunk_of(j)], it & 1, wc, kSiteDsFull))) break;
          tc_fence_after();
          if (j < kEarly) issue_dK(chunk_of(j));
        }
        if (!ok) break;
        if (!kDqFirst) mma_commit(&q_empty[st]);
        if (!C::DQ_ALIAS && it > 0 && !(ok = mbar_wait(dq_free, (it - 1) & 1, wc, kSiteDqFree))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dQ_tile = dS K
          mma_ss(tmem + C::COL_DQ, sdesc_sw128(dsb + kk * 2048, 16384, 1024),
                 sdesc_sw128(kb + kk * 2048, kSlab, 1024), idQ, kk > 0 ? 1u : 0u);
        mma_commit(dq_full);
        if (kDqFirst) {
          // the last chunk's dK steps; q_empty then also tells the P/dS warps that every
          // read of this tile's dS buffer has been issued and completed
          issue_dK(chunk_of(kDsChunks - 1));
          mma_commit(&q_empty[st]);
        }
      }
      if (ok) mma_commit(dkv_final);
      mma_commit(drain);
      mbar_drain(drain, 0, drain_ns(abort_flag, p.timeout_ns));
    }
  } else if (warp < 8) {
    reg_alloc<kRegsCompute>();
    // ------------------------------------------------------------ P^T and dS^T
    // Warpgroup wg takes query columns cb .. cb+63 of the tile (cb = 64 wg); thread r owns
    // key row r.  P^T is stored in place as bf16, packed two per 32-bit column, inside the
    // columns its own warpgroup reads: S^T columns cb + 32 wg .. + 31 (0-31 and 96-127),
    // so neither warpgroup overwrites a column the other has yet to read.  dS^T goes to
    // shared memory only.
    const int wg = warp >> 2;
    const int qw = warp & 3;
    const int cb = wg * 64;
    const int r = qw * 32 + lane;      // key row in the tile
    const int kpos = n * 128 + r;
    const bool key_ok = p.causal || kpos < len;
    const float c = p.scale_log2;
    const uint32_t tS = tmem_addr(tmem, qw * 32, C::COL_S + cb);
    const uint32_t tPst = tmem_addr(tmem, qw * 32, C::COL_S + cb + 32 * wg);
    const uint32_t tP = tmem_addr(tmem, qw * 32, C::COL_DP + cb);
    uint8_t* ds_row = smem + C::OFF_DS + wg * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
    bool ok = true;
    for (int it = 0; it < iters; ++it) {
      const int st = it & 1;
      const int m = nq - 1 - it / p.G;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, it & 1, wc, kSiteSFull) &&
                                       mbar_wait(&q_full[st], (it >> 1) & 1, wc, kSiteQFull));
      if (!ok) break;
      tc_fence_after();
      const float* lse_t = lse_s + st * 128 + cb;
      const float* dlt_t = delta_s + st * 128 + cb;
      // The second 32 columns of S^T load while the first 32 are exponentiated.
      float pr[64];
      uint32_t us[64];
      auto half_s = [&](int hf) -> uint32_t(&)[32] {
        return *reinterpret_cast<uint32_t(*)[32]>(us + 32 * hf);
      };
      tmem_ld32(tS + 0, half_s(0));
      tmem_wait_ld_regs(half_s(0));
      tmem_ld32(tS + 32, half_s(1));
      const bool diag = p.causal && m == n;
      const float4* lse4 = reinterpret_cast<const float4*>(lse_t);
      const uint64_t cc = f2_pack(c, c);
      // Only the diagonal tile (causal) and keys past a sequence's end (full mask) need
      // the per-element select; every other tile takes the unmasked path.
      const bool masked = diag || !key_ok;
      auto p_quads = [&](int i4_0, bool msk) {
#pragma unroll
        for (int i4 = i4_0; i4 < i4_0 + 8; ++i4) {
#pragma unroll
          for (int u = 0; u < 4; ++u) pr[4 * i4 + u] = __uint_as_float(us[4 * i4 + u]);
          const float4 l4 = lse4[i4];
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(pr[4 * i4], pr[4 * i4 + 1]), cc, f2_pack(l4.x, l4.y)), x0, x1);
          f2_unpack(f2_fma(f2_pack(pr[4 * i4 + 2], pr[4 * i4 + 3]), cc, f2_pack(l4.z, l4.w)), x2, x3);
          const float xv[4] = {x0, x1, x2, x3};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = 4 * i4 + u;
            const float e = ex2_approx(xv[u]);
            pr[i] = msk ? ((key_ok && !(diag && cb + i < r)) ? e : 0.f) : e;
          }
        }
      };
      if (masked) p_quads(0, true); else p_quads(0, false);
      tmem_wait_ld_regs(half_s(1));
      if (masked) p_quads(8, true); else p_quads(8, false);
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pr[ch * 32 + 2 * i], pr[ch * 32 + 2 * i + 1]);
        tmem_st16(tPst + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);

      // dS^T = P^T * (dP^T - Delta), written as bf16 into shared memory once the previous
      // dQ MMA has finished reading that buffer.  The one buffer is the A operand of both
      // MMAs that use dS: MN-major dS for dQ = dS K, K-major dS^T for dK += dS^T Q.
      // The dS buffer is free once the previous tile's dQ (and, with dQ first, its last dK
      // steps: q_empty of that tile) have read it.
      ok = __all_sync(0xffffffffu,
                      mbar_wait(dp_full, it & 1, wc, kSiteDpFull) &&
                      (it == 0 || mbar_wait(dq_full, (it - 1) & 1, wc, kSiteDqFull)) &&
                      (!(ATTN_BWD_DQFIRST && C::DQ_ALIAS) || it == 0 ||
                       mbar_wait(&q_empty[(it - 1) & 1], ((it - 1) >> 1) & 1, wc, kSiteQEmpty)));
      if (!ok) break;
      tc_fence_after();
      // dP^T in two halves: the second loads while the first half's dS^T is computed.
      uint32_t u[64];
      auto half_p = [&](int hf) -> uint32_t(&)[32] {
        return *reinterpret_cast<uint32_t(*)[32]>(u + 32 * hf);
      };
      tmem_ld32(tP + 0, half_p(0));
      tmem_wait_ld_regs(half_p(0));
      tmem_ld32(tP + 32, half_p(1));
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        if (ch == 1) tmem_wait_ld_regs(half_p(1));
        uint32_t pk[16];
        const float4* dl4 = reinterpret_cast<const float4*>(dlt_t + ch * 32);
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 d4 = dl4[i4];
          const int c0 = ch * 32 + 4 * i4;
          float a0, a1, a2, a3;
          f2_unpack(f2_mul(f2_pack(pr[c0], pr[c0 + 1]),
                           f2_add(f2_pack(__uint_as_float(u[c0]), __uint_as_float(u[c0 + 1])),
                                  f2_pack(d4.x, d4.y))), a0, a1);
          f2_unpack(f2_mul(f2_pack(pr[c0 + 2], pr[c0 + 3]),
                           f2_add(f2_pack(__uint_as_float(u[c0 + 2]), __uint_as_float(u[c0 + 3])),
                                  f2_pack(d4.z, d4.w))), a2, a3);
          pk[2 * i4] = pack_bf16x2(a0, a1);
          pk[2 * i4 + 1] = pack_bf16x2(a2, a3);
        }
        // shared memory: this warpgroup's 64 query rows are 64-row block wg; local rows
        // ch*32 .. ch*32+31 are 16-byte chunks ch*4 .. ch*4+3 of the key row's line
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = ch * 4 + q4;
          *reinterpret_cast<uint4*>(ds_row + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
        if (kDsChunks == 4) {
          // The dK MMA may read this chunk now.  The last chunk also orders both halves'
          // TMEM loads before the hand-over, since the dQ MMA (after every chunk) writes
          // over the dP^T columns at D = 128.
          fence_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ds_full[wg * 2 + ch]);
        }
      }
      if (kDsChunks == 1) {
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_full[0]);
      }
    }
    // epilogue: dV rows (warps 0-3), dK rows scaled (warps 4-7)
    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(dkv_final, 0, wc, kSiteFinal));
      if (ok) {
        tc_fence_after();
        const uint32_t tO = tmem_addr(tmem, qw * 32, wg == 0 ? C::COL_DV : C::COL_DK);
        const float mul = wg == 0 ? 1.f : p.scale;
        __nv_bfloat16* dst = (wg == 0 ? p.dv : p.dk) + (size_t(start + kpos) * p.Hkv + g) * D;
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t v32[32];
          tmem_ld32(tO + ch * 32, v32);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(v32[2 * i]) * mul, __uint_as_float(v32[2 * i + 1]) * mul);
          if (kpos < len) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
    }
  } else {
    reg_alloc<kRegsCompute>();
    // ------------------------------------------------------------ dQ drain (warps 8-11)
    // Per query tile: read dQ_tile from TMEM (thread = row), free those columns, and
    // add the rows into the fp32 workspace tile with vector reductions.  In the tile
    // layout [D/4][128][4] the 32 rows of a warp are 32 consecutive 16-byte chunks, so
    // each warp-wide reduction covers 512 contiguous bytes (four full lines), and the
    // reductions are fire-and-forget: nothing else waits for them.  The tile is read in
    // two halves (register budget): the first half's reductions are issued before the
    // second half is read and the columns are freed.
    const int qw = warp & 3;
    const int r = qw * 32 + lane;      // query row of the tile
    const uint32_t tQ = tmem_addr(tmem, qw * 32, C::COL_DQ);
    constexpr int HALF = D / 2;
    bool ok = true;
    for (int it = 0; it < iters; ++it) {
      const int hq = g * p.G + it % p.G;
      const int m = nq - 1 - it / p.G;
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full, it & 1, wc, kSiteDqFull));
      if (!ok) break;
      tc_fence_after();
      float4* gdst = reinterpret_cast<float4*>(p.dq_acc + (size_t(hq) * p.ntile + tile_base + m) * 128 * D);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t acc[HALF];
#pragma unroll
        for (int ch = 0; ch < HALF / 32; ++ch)
          tmem_ld32(tQ + hf * HALF + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(acc + ch * 32));
        tmem_wait_ld();
        if (hf == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dq_free);
        }
#pragma unroll
        for (int c4 = 0; c4 < HALF / 4; ++c4)
          atomicAdd(gdst + (hf * HALF / 4 + c4) * 128 + r,
                    make_float4(__uint_as_float(acc[4 * c4]), __uint_as_float(acc[4 * c4 + 1]),
                                __uint_as_float(acc[4 * c4 + 2]), __uint_as_float(acc[4 * c4 + 3])));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace bwd
}  // namespace attn_sm100
