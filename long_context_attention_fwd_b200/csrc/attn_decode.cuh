// attn_decode.cuh -- decode attention over a key/value cache for sm_100a (split-KV).
//
// One new query token per sequence attends to every cached key of its sequence (page
// "ms-swift长文本训练秘诀：Ulysses并行技术解析", section 5: the fine-tuned model is served
// with a 32K-token context; the arithmetic is the standard attention of page
// "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "为什么传统注意力这么'吃'显存",
// computed tile by tile with the online softmax of section "FlashAttention 如何破局").
// The cache of a long sequence is cut into splits; each CTA streams one split's K/V tiles
// and writes partial results (o_p, lse_p) that attn_merge combines exactly.
//
// Decode reads every cached key and value once and does little arithmetic per byte, so
// the kernel is bound by HBM bandwidth.  Mapping (one CTA = one sequence b, one kv head g,
// one split of its cache):
//   Q tile      the G query heads of kv head g are G consecutive rows of q [B*Hq][D]; the
//               128-row tile starting there is loaded once (rows >= G belong to other heads
//               or are zero-filled past the end; their results are never read).
//   warp 8      TMA producer: K_j / V_j tiles of the split into a ring of NS stages (3 for
//               D = 128, 6 for D = 64: the loads, not the math, must stay in flight).
//   warp 9      MMA issuer: S_t = Q K_j^T and O_t += P_t V_j, exactly the operand layouts of
//               the prefill forward kernel.
//   warps 0-3 / 4-7   online softmax of two independent streams: stream 0 takes the split's
//               even tiles, stream 1 the odd ones, each with its own S and O in tensor memory,
//               so one stream's exponentials overlap the other's MMAs.  Only the warps that
//               own rows < G do any work.  Each stream writes its own partial result.
// Cache rows past a sequence's length are never used: their scores are masked to -inf, and
// the rows of the last V tile past the length are zeroed in shared memory before its PV
// product (whatever the cache holds there, 0 * NaN would otherwise poison O).
//
// Each CTA first combines its two streams into one partial (o_s, lse_s).  The last CTA of
// a (sequence, kv head) to finish then combines the partials of every split into o and
// lse (the exact log-sum-exp rule of attn_merge), so a decode step is one launch.  The
// CTAs find the last one without a counter: each writes a flag word carrying the call's
// tag into the caller's workspace (which may hold anything when the call starts), fences,
// and reads the flags of every split of its group; a CTA that sees them all tagged
// merges.  With sequentially consistent fences at least one CTA sees all the others'
// flags; when two do, both write the same result.  The merging CTA clears the flags, so
// a replay of the same launch (same tag) starts clean.
#pragma once
#include <cuda_bf16.h>
#include "attn_merge.cuh"
#include "sm100_ptx.cuh"

namespace attn_sm100 {
namespace decode {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 384;
constexpr int kWarpTMA = 8;
constexpr int kWarpMMA = 9;
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 72;
constexpr int kRegsCompute = 216;
static_assert(128 * kRegsControl + 256 * kRegsCompute <= kThreads * kRegsLaunch, "register split");
constexpr float kRescaleThreshold = 8.0f;
constexpr int kSlab = 128 * 128;
constexpr int kMaxSplits = 128;  // splits (and partials) per (sequence, kv head)

struct Params {
  const int32_t* cache_len;  // [B] (device); clamped to [0, Lmax]
  __nv_bfloat16* o_part;     // [nsplit][B*Hq][D]: one partial per split
  float* lse_part;           // [nsplit][B*Hq]
  int Hq, G, Hkv, Lmax;
  int nsplit, tps;           // splits per (sequence, kv head); tiles per split
  int rows;                  // B * Hq (row stride between partials)
  unsigned long long* flags; // [B * Hkv][nsplit] done flags (caller workspace, any initial value)
  unsigned long long tag;    // this call's tag (nonzero)
  __nv_bfloat16* o;          // [B * Hq][D] result
  float* lse;                // [B * Hq]
  float scale_log2;
  unsigned* status;
  unsigned long long timeout_ns;
};

template <int D>
struct Cfg {
  static constexpr int NS = (D == 128) ? 3 : 6;
  static constexpr int QT_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QT_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
  // q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], v_raw, s_full[2], p_full[2],
  // o_final[2], drain, x_full
  static constexpr int NBAR = 1 + 4 * NS + 1 + 8;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_X = OFF_MISC + 16;    // stream 1's (m, l, lb) per row: 3 x 128 fp32
  static constexpr int SMEM_BYTES = OFF_X + 3 * 128 * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
};

enum : unsigned {
  kSiteKEmpty = 0x300, kSiteVEmpty, kSiteQFull, kSiteKFull, kSiteVFull, kSitePFull, kSiteSFull,
  kSiteOFinal, kSiteVRaw, kSiteDrainQ, kSiteDrainK, kSiteDrainV, kSiteDrainVRaw, kSiteDrainMMA,
  kSiteXFull
};

// Combines the nparts partials of rows row0 .. row0 + G - 1 into p.o and p.lse, with all
// kThreads threads of the CTA: LSE = ln sum_j exp(LSE_j), O = sum_j exp(LSE_j - LSE) O_j
// (weights and sums in fp32, one bf16 rounding).  Partials are read through L2 (another
// CTA wrote most of them).  `scratch` is shared memory the kernel no longer uses.
template <int D>
__device__ void merge_rows(const Params& p, int row0, int G, int nparts, uint8_t* scratch) {
  constexpr int TPR = D / 8;               // threads per row: one 16-byte column group each
  constexpr int NGRP = kThreads / TPR;     // thread groups
  float* s_m = reinterpret_cast<float*>(scratch);   // [128] row maximum of the partial LSEs
  float* s_inv = s_m + 128;                          // [128] 1 / sum of the weights
  float* s_acc = s_inv + 128;                        // [NGRP][TPR][8] partial sums
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Per row (one warp each): the largest partial LSE, and the weight sum relative to it.
  for (int r = warp; r < G; r += kThreads / 32) {
    const int row = row0 + r;
    float m = -INFINITY;
    for (int j = lane; j < nparts; j += 32) m = fmaxf(m, __ldcg(p.lse_part + size_t(j) * p.rows + row));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    if (m != -INFINITY)
      for (int j = lane; j < nparts; j += 32) l += expf(__ldcg(p.lse_part + size_t(j) * p.rows + row) - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      s_m[r] = m;
      s_inv[r] = (m == -INFINITY) ? 0.f : 1.f / l;
      p.lse[row] = (m == -INFINITY) ? -INFINITY : m + logf(l);
    }
  }
  __syncthreads();
  // Rows in passes of rp; the partials of a row are spread over nsub thread groups.
  const int rp = G < NGRP ? G : NGRP;
  const int nsub = NGRP / rp;
  const int grp = threadIdx.x / TPR, c = threadIdx.x % TPR;
  const size_t pstride = size_t(p.rows) * TPR;  // uint4 stride between partials
  for (int r0 = 0; r0 < G; r0 += rp) {
    const int r = r0 + grp % rp, sub = grp / rp;
    if (sub < nsub && r < G) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const float m = s_m[r];
      if (m != -INFINITY) {
        const uint4* ob = reinterpret_cast<const uint4*>(p.o_part) + size_t(row0 + r) * TPR + c;
        const float* lb = p.lse_part + row0 + r;
#pragma unroll 4
        for (int j = sub; j < nparts; j += nsub)
          merge::acc_bf16x8(acc, __ldcg(ob + size_t(j) * pstride), expf(__ldcg(lb + size_t(j) * p.rows) - m));
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) s_acc[(grp * TPR + c) * 8 + e] = acc[e];
    }
    __syncthreads();
    if (grp < rp && r0 + grp < G) {
      const int rr = r0 + grp;
      float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int k = 0; k < nsub; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] += s_acc[((grp + k * rp) * TPR + c) * 8 + e];
      const float inv = s_inv[rr];
      uint4 y;
      y.x = pack_bf16x2(o[0] * inv, o[1] * inv);
      y.y = pack_bf16x2(o[2] * inv, o[3] * inv);
      y.z = pack_bf16x2(o[4] * inv, o[5] * inv);
      y.w = pack_bf16x2(o[6] * inv, o[7] * inv);
      reinterpret_cast<uint4*>(p.o + size_t(row0 + rr) * D)[c] = y;
    }
    __syncthreads();
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (sequence b, kv head g, split s)
  const int s = blockIdx.x % p.nsplit;
  const int bg = blockIdx.x / p.nsplit;
  const int g = bg % p.Hkv;
  const int b = bg / p.Hkv;
  const int L = min(max(__ldg(p.cache_len + b), 0), p.Lmax);
  const int ntile = (L + BN - 1) / BN;
  const int j0 = s * p.tps;
  const int n = max(0, min(ntile - j0, p.tps));         // tiles of this split
  const int n_t[2] = {(n + 1) >> 1, n >> 1};             // even / odd tiles
  const int last_valid = L - BN * (ntile - 1);           // keys in the sequence's last tile
  const bool partial_last = n > 0 && j0 + n == ntile && last_valid < BN;
  const long long tok0 = (long long)b * p.Lmax + (long long)j0 * BN;
  const int row0 = b * p.Hq + g * p.G;                   // first q row of this kv head

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::NS;
  uint64_t* v_full = k_empty + C::NS;
  uint64_t* v_empty = v_full + C::NS;
  uint64_t* v_raw = v_empty + C::NS;
  uint64_t* s_full = v_raw + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_final = p_full + 2;
  uint64_t* drain = o_final + 2;
  uint64_t* x_full = drain + 1;    // stream 1's row statistics are in shared memory
  float* x_m = reinterpret_cast<float*>(smem + C::OFF_X);
  float* x_l = x_m + 128;
  float* x_lb = x_l + 128;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const int nw = (p.G + 31) >> 5;  // softmax warps per stream that own rows < G

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(q_full, 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(v_raw, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], nw);
      mbar_init(&o_final[t], 1);
    }
    mbar_init(drain, 1);
    mbar_init(x_full, nw);
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.status, abort_flag, p.timeout_ns};

  if (warp >= 8) {
   reg_dealloc<kRegsControl>();
   if (warp == kWarpTMA && n > 0) {
    // ------------------------------------------------------------ producer
    // The last V tile of a sequence whose length is not a tile multiple is loaded on its
    // own barrier, then the whole warp zeroes its rows past the length and hands the
    // tile to the MMA warp with a plain arrive on v_full.
    const int n_plain_v = partial_last ? n - 1 : n;
    int nk = 0, nv = 0;
    bool ok = true;
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, C::QT_BYTES);
      for (int hf = 0; hf < D / 64; ++hf)
        tma_load_3d(&tm_q, q_full, smem + C::OFF_Q + hf * kSlab, hf * 64, 0, row0);
      for (int j = 0; j < n && ok; ++j) {
        const int st = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        if (!(ok = mbar_wait(&k_empty[st], ph ^ 1, wc, kSiteKEmpty))) break;
        mbar_arrive_expect_tx(&k_full[st], C::KV_BYTES);
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_3d(&tm_k, &k_full[st], smem + C::OFF_K + st * C::KV_BYTES + hf * kSlab,
                      hf * 64, g, int(tok0 + BN * j));
        ++nk;
        if (!(ok = mbar_wait(&v_empty[st], ph ^ 1, wc, kSiteVEmpty))) break;
        if (j < n_plain_v) {
          mbar_arrive_expect_tx(&v_full[st], C::KV_BYTES);
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_3d(&tm_v, &v_full[st], smem + C::OFF_V + st * C::KV_BYTES + hf * kSlab,
                        hf * 64, g, int(tok0 + BN * j));
          ++nv;
        } else {
          mbar_arrive_expect_tx(v_raw, C::KV_BYTES);
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_3d(&tm_v, v_raw, smem + C::OFF_V + st * C::KV_BYTES + hf * kSlab,
                        hf * 64, g, int(tok0 + BN * j));
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (partial_last) {
      const int st = (n - 1) % C::NS;
      // Every lane waits for the raw tile (it was issued unless the loop stopped early).
      bool landed = ok && __all_sync(0xffffffffu, mbar_wait(v_raw, 0, wc, kSiteVRaw));
      if (landed) {
        // Rows last_valid..127 of each 64-column slab: whole 128-byte lines, so the
        // swizzle (which only permutes 16-byte chunks inside a line) does not matter.
        const int nrows = BN - last_valid;
        for (int idx = lane; idx < nrows * (D / 64) * 8; idx += 32) {
          const int chunk = idx & 7, rr = (idx >> 3) % nrows, hf = (idx >> 3) / nrows;
          uint4* dst = reinterpret_cast<uint4*>(smem + C::OFF_V + st * C::KV_BYTES + hf * kSlab +
                                                (last_valid + rr) * 128 + chunk * 16);
          *dst = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_async_smem();  // generic-proxy writes -> visible to the tensor core
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&v_full[st]);
          ++nv;  // v_full of the last tile's stage has completed one more phase
        }
      } else if (lane == 0 && ok) {
        mbar_drain_checked(v_raw, 0, wc, kSiteDrainVRaw);
      }
    }
    if (lane == 0) {
      // Drain: every issued copy must land before shared memory is released.  Tiles
      // 0..nk-1 (K) and 0..nv-1 (V) completed their stage's barrier in order, so the
      // last phase of stage st is the count of those tiles in that stage, minus one.
      mbar_drain_checked(q_full, 0, wc, kSiteDrainQ);
      for (int st = 0; st < C::NS; ++st) {
        const int ck = nk > st ? (nk - 1 - st) / C::NS + 1 : 0;
        const int cv = nv > st ? (nv - 1 - st) / C::NS + 1 : 0;
        if (ck) mbar_drain_checked(&k_full[st], (ck - 1) & 1, wc, kSiteDrainK);
        if (cv) mbar_drain_checked(&v_full[st], (cv - 1) & 1, wc, kSiteDrainV);
      }
    }
   } else if (warp == kWarpMMA && n > 0) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idPV = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t qb = smem_u32(smem + C::OFF_Q);
      const uint32_t colS[2] = {C::COL_S0, C::COL_S1};
      const uint32_t colO[2] = {C::COL_O0, C::COL_O1};
      auto issue_S = [&](int t, int st) {
        const uint32_t kb = smem_u32(smem + C::OFF_K + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
          mma_ss(tmem + colS[t], sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                 idS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_PV = [&](int t, int st, bool acc) {
        const uint32_t vb = smem_u32(smem + C::OFF_V + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(tmem + colO[t], tmem + colS[t] + kk * 8, sdesc_sw128(vb + kk * 2048, kSlab, 1024),
                 idPV, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(q_full, 0, wc, kSiteQFull);
      for (int t = 0; t < 2 && t < n && ok; ++t) {
        if (!(ok = mbar_wait(&k_full[t], 0, wc, kSiteKFull))) break;
        tc_fence_after();
        issue_S(t, t);
        mma_commit(&s_full[t]);
        mma_commit(&k_empty[t]);
      }
      for (int j = 0; j < n && ok; ++j) {
        const int t = j & 1;
        const int st = j % C::NS;
        if (!(ok = mbar_wait(&v_full[st], (j / C::NS) & 1, wc, kSiteVFull))) break;
        if (!(ok = mbar_wait(&p_full[t], (j >> 1) & 1, wc, kSitePFull))) break;
        tc_fence_after();
        issue_PV(t, st, j >= 2);
        mma_commit(&v_empty[st]);
        if (j + 2 >= n) mma_commit(&o_final[t]);
        if (j + 2 < n) {
          const int st2 = (j + 2) % C::NS;
          if (!(ok = mbar_wait(&k_full[st2], ((j + 2) / C::NS) & 1, wc, kSiteKFull))) break;
          tc_fence_after();
          issue_S(t, st2);
          mma_commit(&s_full[t]);
          mma_commit(&k_empty[st2]);
        }
      }
      mma_commit(drain);
      mbar_drain_checked(drain, 0, wc, kSiteDrainMMA);
    }
   }
   // Back to the launch budget for the merge below, which every warp runs (this waits
   // for the softmax warpgroups' matching decrease).
   reg_alloc<kRegsLaunch>();
  } else {
    reg_alloc<kRegsCompute>();
    // ------------------------------------------------------------ softmax + partial output
    const int t = warp >> 2;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    if (qw < nw) {
      const int nt = t ? n_t[1] : n_t[0];
      const float c = p.scale_log2;
      const uint32_t colS = t ? C::COL_S1 : C::COL_S0;
      const uint32_t colO = t ? C::COL_O1 : C::COL_O0;
      const uint32_t tS = tmem_addr(tmem, qw * 32, colS);
      const uint32_t tO = tmem_addr(tmem, qw * 32, colO);
      float m_run = -INFINITY, l_run = 0.f, lb_run = 0.f;
      bool ok = true;
      for (int i = 0; i < nt; ++i) {
        const int j = 2 * i + t;  // tile index within the split
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], i & 1, wc, kSiteSFull));
        if (!ok) break;
        tc_fence_after();
        float sc[128];
        {
          uint32_t u0[32], u1[32], u2[32], u3[32];
          tmem_ld32(tS + 0, u0);
          tmem_ld32(tS + 32, u1);
          tmem_ld32(tS + 64, u2);
          tmem_ld32(tS + 96, u3);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            sc[k] = __uint_as_float(u0[k]);
            sc[32 + k] = __uint_as_float(u1[k]);
            sc[64 + k] = __uint_as_float(u2[k]);
            sc[96 + k] = __uint_as_float(u3[k]);
          }
        }
        if (partial_last && j == n - 1) {
#pragma unroll
          for (int k = 0; k < 128; ++k)
            if (k >= last_valid) sc[k] = -INFINITY;
        }
        float mx;
        {
          float m4[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
          for (int k = 4; k < 124; k += 8) {
            m4[0] = fmax3(m4[0], sc[k], sc[k + 4]);
            m4[1] = fmax3(m4[1], sc[k + 1], sc[k + 5]);
            m4[2] = fmax3(m4[2], sc[k + 2], sc[k + 6]);
            m4[3] = fmax3(m4[3], sc[k + 3], sc[k + 7]);
          }
          m4[0] = fmax3(m4[0], sc[124], sc[125]);
          m4[1] = fmax3(m4[1], sc[126], sc[127]);
          mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
        }
        const float mx2 = mx * c;
        const bool need = mx2 > m_run + kRescaleThreshold;
        const float m_new = need ? mx2 : m_run;
        const float alpha = need ? ex2_approx(m_run - m_new) : 1.f;
        if (i > 0 && __any_sync(0xffffffffu, need)) {
          uint32_t u[32];
#pragma unroll 1
          for (int ch = 0; ch < D / 32; ++ch) {
            tmem_ld32(tO + ch * 32, u);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) u[k] = __float_as_uint(__uint_as_float(u[k]) * alpha);
            tmem_st32(tO + ch * 32, u);
          }
        }
        l_run *= alpha;
        lb_run *= alpha;
        m_run = m_new;
        const float mneg = (m_run == -INFINITY) ? 0.f : -m_run;
        const uint64_t cc = f2_pack(c, c), mm = f2_pack(mneg, mneg);
        uint64_t sf[4] = {0, 0, 0, 0}, sb[4] = {0, 0, 0, 0};
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(sc[ch * 32 + 2 * k], sc[ch * 32 + 2 * k + 1]), cc, mm), x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            const uint32_t bb = pack_bf16x2(p0, p1);
            pk[k] = bb;
            sf[k & 3] = f2_add(sf[k & 3], f2_pack(p0, p1));
            sb[k & 3] = f2_add(sb[k & 3], f2_pack(__uint_as_float(bb << 16),
                                                  __uint_as_float(bb & 0xFFFF0000u)));
          }
          tmem_st16(tS + ch * 16, pk);
        }
        {
          float a0, a1, b0, b1;
          f2_unpack(f2_add(f2_add(sf[0], sf[1]), f2_add(sf[2], sf[3])), a0, a1);
          f2_unpack(f2_add(f2_add(sb[0], sb[1]), f2_add(sb[2], sb[3])), b0, b1);
          l_run += a0 + a1;
          lb_run += b0 + b1;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t]);
      }
      // One partial per split: stream 1 hands its row statistics to stream 0 through
      // shared memory, and stream 0 combines both accumulators (each relative to its own
      // running maximum) into o_s = (a0 O0 + a1 O1) / (a0 lb0 + a1 lb1) and
      // lse_s = ln(a0 l0 + a1 l1) + M, with a_t = 2^(m_t - M), M = max(m0, m1).  A stream
      // with no tile has m = -inf, weight 0, and its accumulator is never read.
      if (ok && nt > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&o_final[t], 0, wc, kSiteOFinal));
        if (ok) tc_fence_after();
      }
      if (t == 1) {
        if (r < 128) {
          x_m[r] = m_run;
          x_l[r] = l_run;
          x_lb[r] = lb_run;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(x_full);
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(x_full, 0, wc, kSiteXFull)) && ok;
        tc_fence_after();
        const bool valid = r < p.G;
        __nv_bfloat16* orow = p.o_part + (size_t(s) * p.rows + row0 + r) * D;
        float* lrow = p.lse_part + size_t(s) * p.rows + row0 + r;
        const float m1 = x_m[r], l1 = x_l[r], lb1 = x_lb[r];
        const float M = fmaxf(m_run, m1);
        if (nt == 0 || M == -INFINITY) {
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0u, 0u, 0u, 0u);
            *lrow = -INFINITY;
          }
        } else if (ok) {
          const bool has1 = n_t[1] > 0;
          const float a0 = ex2_approx(m_run - M);
          const float a1 = has1 ? ex2_approx(m1 - M) : 0.f;
          const float inv = 1.f / (a0 * lb_run + a1 * lb1);
          const float w0 = a0 * inv, w1 = a1 * inv;
          const uint32_t tO1 = tmem_addr(tmem, qw * 32, C::COL_O1);
#pragma unroll 1
          for (int ch = 0; ch < D / 16; ++ch) {
            uint32_t u[16], u1[16];
            tmem_ld16(tO + ch * 16, u);
            if (has1) tmem_ld16(tO1 + ch * 16, u1);
            tmem_wait_ld();
            uint32_t pk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              float e0 = __uint_as_float(u[2 * k]) * w0, e1 = __uint_as_float(u[2 * k + 1]) * w0;
              if (has1) {
                e0 = fmaf(__uint_as_float(u1[2 * k]), w1, e0);
                e1 = fmaf(__uint_as_float(u1[2 * k + 1]), w1, e1);
              }
              pk[k] = pack_bf16x2(e0, e1);
            }
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + ch * 16);
              dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
          if (valid) *lrow = (M + __log2f(a0 * l_run + a1 * l1)) * 0.69314718055994530942f;
        }
      }
    }
    reg_dealloc<kRegsLaunch>();
  }

  // ---- teardown: every role has drained; release tensor memory.
  if (warp < 4 && warp < nw) __threadfence();  // the partial's writers: visible before the flag
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }

  // ---- done flag; the CTA that sees every split of its group done merges the partials.
  volatile int* s_merge = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  if (warp == 0) {
    volatile unsigned long long* fl = p.flags + size_t(bg) * p.nsplit;
    if (lane == 0) fl[s] = p.tag;
    __syncwarp();
    __threadfence();  // sequentially consistent: this flag is ordered before the reads below
    bool all = true;
    for (int i = lane; i < p.nsplit; i += 32) all = all && fl[i] == p.tag;
    all = __all_sync(0xffffffffu, all);
    if (all) {
      for (int i = lane; i < p.nsplit; i += 32) fl[i] = 0ull;  // a replay starts clean
    }
    if (lane == 0) *s_merge = all;
  }
  __syncthreads();
  if (*s_merge) {
    __threadfence();
    merge_rows<D>(p, row0, p.G, p.nsplit, smem + C::OFF_K);  // K/V stages are free now
  }
}

}  // namespace decode
}  // namespace attn_sm100
