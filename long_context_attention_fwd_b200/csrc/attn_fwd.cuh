// attn_fwd.cuh -- fused attention forward for sm_100a.
//
// Follows the fused, tiled scheme of the page "ms-swift集成FlashAttention 2/3，长文本训练更高效"
// [ms-swift integrates FlashAttention 2/3], section "FlashAttention 如何破局"
// [how FlashAttention breaks the deadlock]: Q, K, V are cut into tiles along the
// sequence, a block holds its Q tile and streams the K/V tiles of the same sequence
// through on-chip memory, runs QK^T -> softmax -> PV there with an online softmax
// (running maximum and normaliser per row), and writes only the output (plus the
// row log-sum-exp kept for the backward pass).
//
// Blackwell mapping (one CTA = 256 query rows of one head, as two 128-row tiles):
//   warp 8      TMA producer: Q tiles once, then K_j / V_j into a ring of NS stages.
//   warp 9      MMA issuer (one thread): S_t = Q_t K_j^T (SS, fp32 in TMEM) and
//               O_t += P_t V_j (P read from TMEM as bf16, V from shared memory; at D = 64
//               also the row sums of P against the ones columns).
//   warps 10-11 idle (they complete the control warpgroup for the register split).
//   warps 0-3   softmax for tile 0, warps 4-7 for tile 1: one thread per query row,
//               reads S from TMEM, exp2-based online max/sum, writes P (bf16) back
//               into the S columns, rescales O in TMEM when the running max grows by
//               more than 2^8, and finally normalises O and stores O and LSE.
// The two tiles ping-pong: while softmax works on one tile the tensor core runs the
// other tile's PV and the next S, so MMA and exponentials overlap.
//
// The exponentials and the MMAs of a tile take about equally long at D = 128, and the
// exponentials twice as long at D = 64, so the softmax chain paces the loop.  At D = 64
// two changes take work off the softmax threads and start the PV product sooner:
//   - the normaliser over the bf16 weights comes out of the PV MMA itself, as 16 extra
//     accumulator columns against a column of ones in shared memory;
//   - P is handed to the MMA warp in four chunks of 32 keys, so the PV MMAs of the first
//     keys run while the later ones are exponentiated (at D = 128 the extra barrier
//     round trips cost more than the overlap gains, so P goes over as one tile there).
// A share of the exponentials (Cfg::EMU pairs of every 16, in tiles without masked
// scores) can also be evaluated by a polynomial on the FMA pipe (exp2_poly_x2); the share
// is 0 by default, since no share measured faster at either head dim.
//
// FP8 = true is the e4m3 variant (D = 128): Q, K, V are e4m3 with per-tensor descale
// factors folded into the softmax scale (q, k) and the epilogue (v); the MMAs are
// kind::f8f6f4 (K = 32 per instruction, twice the bf16 rate); P is quantised as
// e4m3(256 p) -- the factor 256 keeps probabilities down to 2^-14 in e4m3's normal range
// -- and O is divided by the sum of exactly those quantised weights, so the factor cancels.
#pragma once
#include <cuda_bf16.h>
#include <type_traits>
#include "attn_common.cuh"
#include "sm100_ptx.cuh"

namespace attn_sm100 {
namespace fwd {

constexpr int BM = 128;                // query rows per tile
constexpr int BN = 128;                // keys per K/V tile
constexpr int kThreads = 384;          // 12 warps; warps 10-11 only complete the control warpgroup
constexpr int kWarpTMA = 8;
constexpr int kWarpMMA = 9;
// Register split (setmaxnreg), as in the backward kernel: 168 at launch, 88 for the
// control warpgroup (the producer and MMA loops carry the item loop's state), 208 for the
// two softmax warpgroups (128*88 + 256*208 = 384*168); ptxas spills nothing at this split.
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 88;
constexpr int kRegsCompute = 208;
static_assert(128 * kRegsControl + 256 * kRegsCompute <= kThreads * kRegsLaunch, "register split");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when max grows > 2^8
constexpr int kSlab = 128 * 128;       // one 128-row x 64-column bf16 swizzled slab (16 KB)
// Share of the exponentials (pairs out of 16) computed on the FMA pipe, per head dim.
#ifndef ATTN_FWD_EMU64
#define ATTN_FWD_EMU64 0
#endif
#ifndef ATTN_FWD_EMU128
#define ATTN_FWD_EMU128 0
#endif
#ifndef ATTN_FWD_EMU_FP8
#define ATTN_FWD_EMU_FP8 0
#endif
// The softmax warps hand P to the MMA warp in chunks (1), so that a tile's PV product
// starts on the first keys while the later ones are still being exponentiated, or as
// one tile (0), per head dim.
// Row sums of the rounded weights by mixed-precision adds (bf16 or f16 operand, fp32
// accumulator) instead of unpacking to fp32 first (1), or by unpacking (0).
#ifndef ATTN_FWD_MIXADD
#define ATTN_FWD_MIXADD 1
#endif
// e4m3: the factor 256 of P = e4m3(256 p) folded into the exponent, exp2(x + 8) (1), or
// applied by a multiply (0).
#ifndef ATTN_FWD_FP8FOLD
#define ATTN_FWD_FP8FOLD 1
#endif
#ifndef ATTN_FWD_PCHUNK64
#define ATTN_FWD_PCHUNK64 1
#endif
#ifndef ATTN_FWD_PCHUNK128
#define ATTN_FWD_PCHUNK128 0
#endif
#ifndef ATTN_FWD_PCHUNK_FP8
#define ATTN_FWD_PCHUNK_FP8 1
#endif

struct Params {
  SeqView sv;
  __nv_bfloat16* o;
  float* lse;
  int Hq, G, T;                        // query heads, query heads per kv head, total tokens
  int causal;
  float scale_log2;                    // softmax scale * log2(e) (* q, k descale for e4m3)
  float o_scale;                       // 1, or the v descale for e4m3
  int nblk;                            // (T >> 8) + nseq: upper bound of 256-row blocks
  int nitems;                          // nblk * Hq work items
  unsigned* status;
  unsigned long long timeout_ns;
};

constexpr float kP8Scale = 256.0f;      // e4m3 P = e4m3(256 p)
// e4m3 saturates at 448, so 256 p must stay below it: p is relative to the running maximum,
// which the lazy rescale lets lag the true one by up to the threshold.  2^0.5 * 256 = 362.
constexpr float kRescaleThresholdFp8 = 0.5f;

template <int D, bool FP8 = false>
struct Cfg {
  // D = 64 (bf16): TMEM has room for 16 more accumulator columns per tile, so the PV MMA
  // also sums the bf16 weights of every row against a column of ones (N = D + 16): the
  // normaliser then comes from the tensor core, accumulated and rescaled exactly like O,
  // instead of a second running sum in the softmax threads.
  static constexpr bool ONES = !FP8 && D == 64;
  static constexpr int NPV = ONES ? D + 16 : D;          // N of the PV MMA
  // Of every 16 probability pairs, EMU are exponentiated on the FMA pipe (exp2_poly_x2)
  // instead of the MUFU unit, in tiles without masked scores.
  static constexpr int EMU = FP8 ? ATTN_FWD_EMU_FP8 : (D == 64 ? ATTN_FWD_EMU64 : ATTN_FWD_EMU128);
  static constexpr int ES = FP8 ? 1 : 2;                 // bytes per element
  static constexpr int NS = FP8 ? 4 : ((D == 128) ? 2 : 4);
  static constexpr int SLABS = D * ES / 128;             // 128-byte swizzle rows per tile row
  static constexpr int KSTEPS = D * ES / 32;             // MMAs over D (32 bytes of K each)
  static constexpr int PSTEPS = BN * ES / 32;            // MMAs over the keys of a tile
  static constexpr int SMCH = FP8 ? 2 : 4;               // softmax chunks of 16 P columns
  static constexpr int PCH =                              // P hand-overs per tile
      (FP8 ? ATTN_FWD_PCHUNK_FP8 : (D == 64 ? ATTN_FWD_PCHUNK64 : ATTN_FWD_PCHUNK128)) ? SMCH : 1;
  static constexpr int QT_BYTES = BM * D * ES;
  static constexpr int KV_BYTES = BN * D * ES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * QT_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_ONES = OFF_V + NS * KV_BYTES;  // 128 x 64 bf16 slab (ONES only)
  static constexpr int OFF_BAR = OFF_ONES + (ONES ? kSlab : 0);
  // q_full, q_empty, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2],
  // p_full[2][PCH], o_final[2], drain
  static constexpr int NBAR = 2 + 4 * NS + 5 + 2 * PCH;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = ONES ? 384 : 256 + D;
  static_assert(COL_O1 + NPV <= TMEM_COLS, "TMEM budget");
};

// a += low bf16 of v, b += high bf16 of v: each bf16 taken exactly, one fp32 rounding per add
// (mixed-precision add, no unpacking).
__device__ __forceinline__ void add_bf16x2_f32(uint32_t v, float& a, float& b) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
      : "+f"(a), "+f"(b) : "r"(v));
}
// The same for two f16 values.
__device__ __forceinline__ void add_f16x2_f32(uint32_t v, float& a, float& b) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.f16 %0, lo, %0;\n\tadd.rn.f32.f16 %1, hi, %1;\n\t}"
      : "+f"(a), "+f"(b) : "r"(v));
}
// The two e4m3 values of the low 16 bits of `v`, exactly, as an f16x2 (low byte in the low half).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(uint16_t(v & 0xFFFFu)));
  return h2;
}

// Pair i (0..15) of a 32-score chunk is exponentiated on the FMA pipe when this holds:
// EMU of every 16 pairs, spread evenly.
template <int EMU>
__device__ __forceinline__ constexpr bool emu_pair(int i) {
  return EMU > 0 && ((i + 1) * EMU) / 16 != (i * EMU) / 16;
}

// Wait-site codes reported in the status word when a wait times out.
enum : unsigned {
  kSiteKEmpty = 0x100, kSiteVEmpty, kSiteQFull, kSiteKFull, kSiteVFull, kSitePFull, kSiteSFull,
  kSiteOFinal, kSiteQEmpty
};

// One work item: 256 query rows (two 128-row tiles) of one head of one sequence.
struct Item {
  int h, g, seq, start, len, q_row0, jmax;
  int n_t[2];  // K/V tiles each query tile sees (0: the tile lies past the sequence end)
};

// The k-th item of this CTA.  Items are numbered longest causal block first, heads
// fastest.  The grid is persistent (one CTA per SM, or fewer when there are fewer items):
// CTA c takes items c, 2G-1-c, 2G+c, 4G-1-c, ... of a G-CTA grid -- rounds of G items in
// alternating direction, so that over two rounds every CTA gets one of the longer and one
// of the shorter blocks.  A grid of one CTA per item gives each CTA exactly one item.
__device__ __forceinline__ int item_index(int k) {
  const int G = int(gridDim.x), c = int(blockIdx.x);
  return k * G + ((k & 1) ? G - 1 - c : c);
}

// Fills `it` for item w; false for an index in the slack after a sequence's last block.
__device__ __forceinline__ bool item_at(const Params& p, int w, Item& it) {
  it.h = w % p.Hq;
  int mb;
  if (!locate_block<8>(p.sv, p.nblk - 1 - w / p.Hq, it.seq, mb, it.start, it.len)) return false;
  it.g = it.h / p.G;
  it.q_row0 = mb * 256;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r0 = it.q_row0 + BM * t;
    if (r0 >= it.len) it.n_t[t] = 0;
    else if (p.causal) it.n_t[t] = (min(r0 + BM - 1, it.len - 1) >> 7) + 1;
    else it.n_t[t] = (it.len + BN - 1) >> 7;
  }
  it.jmax = max(it.n_t[0], it.n_t[1]);
  return true;
}

template <int D, bool FP8 = false>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Params p) {
  static_assert(!FP8 || D == 128, "the e4m3 variant is built for D = 128");
  using C = Cfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;    // the item's last S MMA has read the Q tiles
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + C::NS;
  uint64_t* v_full = k_empty + C::NS;
  uint64_t* v_empty = v_full + C::NS;
  uint64_t* s_full = v_empty + C::NS;
  uint64_t* p_full = s_full + 2;           // [2][PCH]: chunk c of tile t's P is in TMEM
  uint64_t* o_final = p_full + 2 * C::PCH;
  uint64_t* drain = o_final + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      for (int c = 0; c < C::PCH; ++c) mbar_init(&p_full[t * C::PCH + c], 4);
      mbar_init(&o_final[t], 1);
    }
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
  }
  if constexpr (C::ONES) {
    // The ones operand of the row-sum columns: 128 key rows of 64 bf16 (one 128-byte
    // swizzle row each), element 0 = 1 and the rest 0.  With the 128-byte swizzle the
    // 16-byte chunk c of row r sits at chunk position c ^ (r % 8), so element 0 of row r
    // lies at byte 16 * (r % 8) of the row.
    uint4* ones = reinterpret_cast<uint4*>(smem + C::OFF_ONES);
    for (int i = threadIdx.x; i < kSlab / 16; i += kThreads) {
      const int r = i >> 3, c = i & 7;
      ones[i] = make_uint4(c == (r & 7) ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    fence_async_smem();  // generic-proxy writes, read by the tensor core
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.status, abort_flag, p.timeout_ns};

  if (warp >= 8) {
   reg_dealloc<kRegsControl>();
   if (warp == kWarpTMA) {
    // ------------------------------------------------------------ producer
    // Per item: the two Q tiles (once the previous item's last S MMA has read the
    // buffer), then K_j / V_j into the ring, whose position carries over from item to
    // item, so the next item's tiles load while this one finishes.
    if (lane == 0) {
      int nq = 0, nk = 0, nv = 0;  // Q loads, K tiles, V tiles issued
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int w = item_index(k);
        if (w >= p.nitems) break;
        Item it;
        if (!item_at(p, w, it)) continue;
        if (nq > 0 && !(ok = mbar_wait(q_empty, (nq - 1) & 1, wc, kSiteQEmpty))) break;
        const uint32_t qbytes = (it.n_t[0] > 0 ? C::QT_BYTES : 0) + (it.n_t[1] > 0 ? C::QT_BYTES : 0);
        mbar_arrive_expect_tx(q_full, qbytes);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (it.n_t[t] == 0) continue;
          for (int hf = 0; hf < C::SLABS; ++hf)
            tma_load_3d(&tm_q, q_full, smem + C::OFF_Q + t * C::QT_BYTES + hf * kSlab,
                        hf * (128 / C::ES), it.h, it.start + it.q_row0 + BM * t);
        }
        ++nq;
        for (int j = 0; j < it.jmax; ++j) {
          const int st = nk % C::NS;
          const uint32_t ph = (nk / C::NS) & 1;
          if (!(ok = mbar_wait(&k_empty[st], ph ^ 1, wc, kSiteKEmpty))) break;
          mbar_arrive_expect_tx(&k_full[st], C::KV_BYTES);
          for (int hf = 0; hf < C::SLABS; ++hf)
            tma_load_3d(&tm_k, &k_full[st], smem + C::OFF_K + st * C::KV_BYTES + hf * kSlab,
                        hf * (128 / C::ES), it.g, it.start + BN * j);
          ++nk;
          if (!(ok = mbar_wait(&v_empty[st], ph ^ 1, wc, kSiteVEmpty))) break;
          mbar_arrive_expect_tx(&v_full[st], C::KV_BYTES);
          for (int hf = 0; hf < C::SLABS; ++hf)
            tma_load_3d(&tm_v, &v_full[st], smem + C::OFF_V + st * C::KV_BYTES + hf * kSlab,
                        hf * (128 / C::ES), it.g, it.start + BN * j);
          ++nv;
        }
      }
      // Drain: every issued copy must land before shared memory is released.
      if (nq) mbar_drain(q_full, (nq - 1) & 1, drain_ns(abort_flag, p.timeout_ns));
      for (int st = 0; st < C::NS; ++st) {
        const int ck = nk > st ? (nk - 1 - st) / C::NS + 1 : 0;
        const int cv = nv > st ? (nv - 1 - st) / C::NS + 1 : 0;
        if (ck) mbar_drain(&k_full[st], (ck - 1) & 1, drain_ns(abort_flag, p.timeout_ns));
        if (cv) mbar_drain(&v_full[st], (cv - 1) & 1, drain_ns(abort_flag, p.timeout_ns));
      }
    }
   } else if (warp == kWarpMMA) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = FP8 ? idesc_e4m3_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idPV = FP8 ? idesc_e4m3_f32(128, D, 0, 1) : idesc_bf16_f32(128, C::NPV, 0, 1);
      const uint32_t qb[2] = {smem_u32(smem + C::OFF_Q), smem_u32(smem + C::OFF_Q + C::QT_BYTES)};
      const uint32_t colS[2] = {C::COL_S0, C::COL_S1};
      const uint32_t colO[2] = {C::COL_O0, C::COL_O1};
      auto issue_S = [&](int t, int st) {
        const uint32_t kb = smem_u32(smem + C::OFF_K + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * kSlab + (kk & 3) * 32;
          if constexpr (FP8)
            mma_ss_f8(tmem + colS[t], sdesc_sw128(qb[t] + off, 16, 1024),
                      sdesc_sw128(kb + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
          else
            mma_ss(tmem + colS[t], sdesc_sw128(qb[t] + off, 16, 1024),
                   sdesc_sw128(kb + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
      };
      // O_t (+)= P_t V over the tile's keys, chunk by chunk as the softmax warps hand the
      // chunks of P over (parity `ph` of this tile's hand-overs); false if a wait failed.
      auto issue_PV = [&](int t, int st, bool acc, uint32_t ph) -> bool {
        const uint32_t vb = smem_u32(smem + C::OFF_V + st * C::KV_BYTES);
        // MN-major V: 64-element N blocks kSlab apart; with the ones columns the second
        // N block is the ones slab, which lies after every V stage.
        constexpr uint32_t kLbo0 = C::ONES ? uint32_t(C::OFF_ONES - C::OFF_V) : uint32_t(kSlab);
        const uint32_t lbo = C::ONES ? kLbo0 - uint32_t(st * C::KV_BYTES) : kLbo0;
        constexpr int KPC = C::PSTEPS / C::PCH;  // K steps per hand-over
#pragma unroll
        for (int c = 0; c < C::PCH; ++c) {
          if (!mbar_wait(&p_full[t * C::PCH + c], ph, wc, kSitePFull)) return false;
          tc_fence_after();
#pragma unroll
          for (int k2 = 0; k2 < KPC; ++k2) {
            const int kk = c * KPC + k2;
            // K step: 32 bytes of keys = 32 / ES key rows of 128 bytes in the MN-major V tile
            const uint64_t bdesc = sdesc_sw128(vb + kk * (4096 / C::ES), lbo, 1024);
            if constexpr (FP8)
              mma_ts_f8(tmem + colO[t], tmem + colS[t] + kk * 8, bdesc, idPV, (acc || kk > 0) ? 1u : 0u);
            else
              mma_ts(tmem + colO[t], tmem + colS[t] + kk * 8, bdesc, idPV, (acc || kk > 0) ? 1u : 0u);
          }
        }
        return true;
      };
      // Phase counts carry over from item to item: nq items' Q tiles consumed, kv the
      // ring position of the item's first K/V tile, pc[t] P tiles of query tile t used.
      // A new item's first S overwrites the previous item's last P only after the PV
      // that read it (MMAs complete in order); its first PV overwrites O only after the
      // softmax warps signalled the new item's first P, which they do after their
      // epilogue of the previous item has read O.
      int nq = 0, kv = 0, pc[2] = {0, 0};
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int w = item_index(k);
        if (w >= p.nitems) break;
        Item it;
        if (!item_at(p, w, it)) continue;
        const int n_t[2] = {it.n_t[0], it.n_t[1]};
        const int jmax = it.jmax;
        if (!(ok = mbar_wait(q_full, nq & 1, wc, kSiteQFull))) break;
        ++nq;
        if (!(ok = mbar_wait(&k_full[kv % C::NS], (kv / C::NS) & 1, wc, kSiteKFull))) break;
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (n_t[t] > 0) {
            issue_S(t, kv % C::NS);
            mma_commit(&s_full[t]);
          }
        mma_commit(&k_empty[kv % C::NS]);
        if (jmax == 1) mma_commit(q_empty);  // the item's last S has been issued
        for (int j = 0; j < jmax && ok; ++j) {
          const int st = (kv + j) % C::NS;
          if (!(ok = mbar_wait(&v_full[st], ((kv + j) / C::NS) & 1, wc, kSiteVFull))) break;
          tc_fence_after();
          if (j < n_t[0]) {
            if (!(ok = issue_PV(0, st, j > 0, pc[0] & 1))) break;
            ++pc[0];
            if (j == n_t[0] - 1) mma_commit(&o_final[0]);
          }
          const bool nxt = j + 1 < jmax;
          const int st1 = (kv + j + 1) % C::NS;
          if (nxt) {
            if (!(ok = mbar_wait(&k_full[st1], ((kv + j + 1) / C::NS) & 1, wc, kSiteKFull))) break;
            tc_fence_after();
            if (j + 1 < n_t[0]) {
              issue_S(0, st1);
              mma_commit(&s_full[0]);
            }
          }
          if (j < n_t[1]) {
            if (!(ok = issue_PV(1, st, j > 0, pc[1] & 1))) break;
            ++pc[1];
            if (j == n_t[1] - 1) mma_commit(&o_final[1]);
          }
          mma_commit(&v_empty[st]);
          if (nxt) {
            if (j + 1 < n_t[1]) {
              issue_S(1, st1);
              mma_commit(&s_full[1]);
            }
            mma_commit(&k_empty[st1]);
            if (j + 2 == jmax) mma_commit(q_empty);  // the item's last S has been issued
          }
        }
        kv += jmax;
      }
      // Drain: all MMAs must finish before TMEM and shared memory are released.
      mma_commit(drain);
      mbar_drain(drain, 0, drain_ns(abort_flag, p.timeout_ns));
    }
   }
  } else {
    reg_alloc<kRegsCompute>();
    // ------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    const float c = p.scale_log2;
    const uint32_t colS = t ? C::COL_S1 : C::COL_S0;
    const uint32_t colO = t ? C::COL_O1 : C::COL_O0;
    const uint32_t tS = tmem_addr(tmem, qw * 32, colS);
    const uint32_t tO = tmem_addr(tmem, qw * 32, colO);
    int sc = 0, oc = 0;  // S tiles and epilogues of this query tile so far (barrier phases)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int w = item_index(k);
      if (w >= p.nitems) break;
      Item it;
      if (!item_at(p, w, it)) continue;
      const int n = t ? it.n_t[1] : it.n_t[0];
      if (n == 0) continue;
      const int rpos = it.q_row0 + BM * t + r;
      const int len = it.len;
      float m_run = -INFINITY;  // reference maximum (log2 units) the accumulator is scaled to
      float l_run = 0.f;        // running normaliser relative to m_run (fp32 probabilities)
      float lb_run = 0.f;       // the same over the bf16-rounded probabilities fed to PV
      for (int j = 0; j < n; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], sc & 1, wc, kSiteSFull));
        if (!ok) break;
        ++sc;
        tc_fence_after();
        float s[128];
        {
          uint32_t u0[32], u1[32], u2[32], u3[32];
          tmem_ld32(tS + 0, u0);
          tmem_ld32(tS + 32, u1);
          tmem_ld32(tS + 64, u2);
          tmem_ld32(tS + 96, u3);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(u0[i]);
            s[32 + i] = __uint_as_float(u1[i]);
            s[64 + i] = __uint_as_float(u2[i]);
            s[96 + i] = __uint_as_float(u3[i]);
          }
        }
        if (j == n - 1) {
          // Last tile of the row's range: causal diagonal, or the sequence's key bound.
          const int lim = p.causal ? rpos : (len - 1);
          const int cmax = lim - BN * j;
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i > cmax) s[i] = -INFINITY;
        }
        float mx;
        {
          float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
          for (int i = 4; i < 124; i += 8) {  // elements 4 .. 123
            m4[0] = fmax3(m4[0], s[i], s[i + 4]);
            m4[1] = fmax3(m4[1], s[i + 1], s[i + 5]);
            m4[2] = fmax3(m4[2], s[i + 2], s[i + 6]);
            m4[3] = fmax3(m4[3], s[i + 3], s[i + 7]);
          }
          m4[0] = fmax3(m4[0], s[124], s[125]);
          m4[1] = fmax3(m4[1], s[126], s[127]);
          mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
        }
        const float mx2 = mx * c;
        const bool need = mx2 > m_run + (FP8 ? kRescaleThresholdFp8 : kRescaleThreshold);
        const float m_new = need ? mx2 : m_run;
        const float alpha = need ? ex2_approx(m_run - m_new) : 1.f;
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          uint32_t u[32];
#pragma unroll 1
          for (int ch = 0; ch < (C::NPV + 31) / 32; ++ch) {  // O, and the row-sum columns
            tmem_ld32(tO + ch * 32, u);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            tmem_st32(tO + ch * 32, u);
          }
        }
        l_run *= alpha;
        lb_run *= alpha;
        m_run = m_new;
        const float mneg = (m_run == -INFINITY) ? 0.f : -m_run;
        const uint64_t cc = f2_pack(c, c), mm = f2_pack(mneg, mneg);
        // e4m3: exp2(x + 8) = 256 exp2(x), the scaled weight that is quantised
        constexpr float kFold = (FP8 && ATTN_FWD_FP8FOLD) ? 8.0f : 0.0f;
        const uint64_t mm8 = f2_pack(mneg + kFold, mneg + kFold);
        // Two running sums: of the fp32 probabilities (for the log-sum-exp) and of
        // their bf16 roundings (the values the PV MMA consumes), so that O is
        // normalised by exactly the weights it was accumulated with.  With the ones
        // columns the second sum comes out of the PV MMA instead.
        uint64_t sf[4] = {0, 0, 0, 0}, sb[4] = {0, 0, 0, 0};
        float sbf[4] = {0.f, 0.f, 0.f, 0.f};  // the rounded weights' sum, mixed-precision adds
        // Hands chunk ch of P to the MMA warp once its TMEM stores have completed (after
        // every chunk, or after the last one when P goes over as one tile).
        auto publish = [&](int ch) {
          constexpr int per = C::SMCH / C::PCH;
          if ((ch + 1) % per != 0) return;
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[t * C::PCH + ch / per]);
        };
        if constexpr (!FP8) {
          // Tiles with no masked score hand a share of the exponentials to the FMA pipe.
          auto exps = [&](auto emu_tag) {
            constexpr bool kEmu = decltype(emu_tag)::value;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const uint64_t x2 = f2_fma(f2_pack(s[ch * 32 + 2 * i], s[ch * 32 + 2 * i + 1]), cc, mm);
                float x0, x1, p0, p1;
                f2_unpack(x2, x0, x1);
                if (kEmu && emu_pair<C::EMU>(i)) {
                  f2_unpack(exp2_poly_x2(x0, x1), p0, p1);
                } else {
                  p0 = ex2_approx(x0);
                  p1 = ex2_approx(x1);
                }
                const uint32_t b = pack_bf16x2(p0, p1);
                pk[i] = b;
                sf[i & 3] = f2_add(sf[i & 3], f2_pack(p0, p1));
                if constexpr (!C::ONES) {
                  if constexpr (ATTN_FWD_MIXADD)
                    add_bf16x2_f32(b, sbf[(i & 1) * 2], sbf[(i & 1) * 2 + 1]);
                  else
                    sb[i & 3] = f2_add(sb[i & 3], f2_pack(__uint_as_float(b << 16),
                                                          __uint_as_float(b & 0xFFFF0000u)));
                }
              }
              tmem_st16(tS + ch * 16, pk);
              publish(ch);
            }
          };
          if (C::EMU > 0 && j < n - 1) exps(std::true_type{});
          else exps(std::false_type{});
        } else {
          // e4m3: four keys per 32-bit column, 256 p quantised; sb sums the quantised values
          auto exps8 = [&](auto emu_tag) {
            constexpr bool kEmu = decltype(emu_tag)::value;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int k0 = ch * 64 + 4 * i;
                float x0, x1, x2, x3, p0, p1, p2, p3;
                f2_unpack(f2_fma(f2_pack(s[k0], s[k0 + 1]), cc, mm8), x0, x1);
                f2_unpack(f2_fma(f2_pack(s[k0 + 2], s[k0 + 3]), cc, mm8), x2, x3);
                if (kEmu && emu_pair<C::EMU>(i)) {
                  f2_unpack(exp2_poly_x2(x0, x1), p0, p1);
                  f2_unpack(exp2_poly_x2(x2, x3), p2, p3);
                } else {
                  p0 = ex2_approx(x0);
                  p1 = ex2_approx(x1);
                  p2 = ex2_approx(x2);
                  p3 = ex2_approx(x3);
                }
                // with the fold, p is already 256 p (and so are both sums)
                constexpr float ps = ATTN_FWD_FP8FOLD ? 1.0f : kP8Scale;
                const uint32_t lo = pack_e4m3x2(ps * p0, ps * p1);
                const uint32_t hi = pack_e4m3x2(ps * p2, ps * p3);
                pk[i] = lo | (hi << 16);
                sf[i & 3] = f2_add(sf[i & 3], f2_add(f2_pack(p0, p1), f2_pack(p2, p3)));
                if constexpr (ATTN_FWD_MIXADD) {
                  add_f16x2_f32(e4m3x2_to_f16x2(lo), sbf[0], sbf[1]);
                  add_f16x2_f32(e4m3x2_to_f16x2(hi), sbf[2], sbf[3]);
                } else {
                  float q0, q1, q2, q3;
                  unpack_e4m3x2(lo, q0, q1);
                  unpack_e4m3x2(hi, q2, q3);
                  sb[i & 3] = f2_add(sb[i & 3], f2_add(f2_pack(q0, q1), f2_pack(q2, q3)));
                }
              }
              tmem_st16(tS + ch * 16, pk);
              publish(ch);
            }
          };
          if (C::EMU > 0 && j < n - 1) exps8(std::true_type{});
          else exps8(std::false_type{});
        }
        {
          float a0, a1, b0, b1;
          f2_unpack(f2_add(f2_add(sf[0], sf[1]), f2_add(sf[2], sf[3])), a0, a1);
          f2_unpack(f2_add(f2_add(sb[0], sb[1]), f2_add(sb[2], sb[3])), b0, b1);
          l_run += a0 + a1;
          lb_run += (b0 + b1) + ((sbf[0] + sbf[1]) + (sbf[2] + sbf[3]));
        }
      }
      if (ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(&o_final[t], oc & 1, wc, kSiteOFinal));
        ++oc;
        if (ok) {
          tc_fence_after();
          // lb_run sums the weights the PV MMA used (for e4m3 in units of 1/256, which the
          // division cancels); with the ones columns that sum is O's column D.  o_scale is
          // 1, or the v descale.
          float wsum = lb_run;
          if constexpr (C::ONES) {
            uint32_t u[32];
            tmem_ld32(tO + D, u);
            tmem_wait_ld();
            wsum = __uint_as_float(u[0]);
          }
          const float inv = p.o_scale / wsum;
          const bool valid = rpos < len;
          __nv_bfloat16* orow = p.o + (size_t(it.start + rpos) * p.Hq + it.h) * D;
#pragma unroll 1
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t u[32];
            tmem_ld32(tO + ch * 32, u);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(u[2 * i]) * inv, __uint_as_float(u[2 * i + 1]) * inv);
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
          if (valid) {
            // with the e4m3 fold, l_run sums 256 p
            constexpr float kLFold = (FP8 && ATTN_FWD_FP8FOLD) ? 8.0f : 0.0f;
            const float lse = (m_run + __log2f(l_run) - kLFold) * 0.69314718055994530942f;
            const size_t li = p.sv.cu ? size_t(it.h) * p.T + it.start + rpos
                                      : (size_t(it.seq) * p.Hq + it.h) * p.sv.S + rpos;
            p.lse[li] = lse;
          }
        }
      }
    }  // items
  }

  // ---- teardown: every role has drained; release tensor memory.
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fwd
}  // namespace attn_sm100
