// attn_lib.cu -- host side of libattn.so: argument validation, TMA descriptors,
// launch configuration and the device status word.  The kernels live in the
// included headers; this is the only translation unit of the library.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <chrono>
#include <unistd.h>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "attn_accum.cuh"
#include "attn_bwd.cuh"
#include "attn_decode.cuh"
#include "attn_fwd.cuh"
#include "attn_merge.cuh"
#include "attn_relayout.cuh"
#include "umma_selftest.cuh"

using namespace attn_sm100;

static_assert(merge::kMaxParts == ATTN_MERGE_MAX_PARTS, "merge part limit out of sync");
static_assert(decode::kRegsLaunch == fwd::kRegsLaunch, "register split of the decode kernel");

// Sticky device status: [0] status bits, [1] site code of the first timeout.
static __device__ unsigned g_attn_status[2];

namespace {

// Description of the last failing CUDA call made by this library on this thread.
thread_local char g_last_error[256] = "";

attn_status fail_cuda(const char* where, cudaError_t e) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e), int(e));
  return ATTN_ERR_CUDA;
}
attn_status fail_cu(const char* where, CUresult r) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: CUresult %d", where, int(r));
  return ATTN_ERR_CUDA;
}
attn_status check_launch(const char* where) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ATTN_OK : fail_cuda(where, e);
}

constexpr int kMaxDevices = 64;
std::atomic<unsigned long long> g_timeout_ns{2000000000ull};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
  bool ready = false;
  bool sm100 = false;
  unsigned* status = nullptr;
  unsigned merge_grid[2][merge::kVariants] = {};  // resident blocks per merge kernel (D 64/128)
  unsigned relayout_grid = 0;                     // resident blocks of transpose_blocks_kernel
  unsigned sms = 0;                               // SM count (grid size of element-wise kernels)
};
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

// The calling thread's current device.  Entry points make the device that owns their
// tensors current (launches and kernel attributes need it) and give the caller's choice
// back when they return.  The previous device is only made current again when its
// primary context is already active: cudaSetDevice would otherwise create a context,
// and take its memory, on a device this process never used.
typedef CUresult (*DeviceGetFn)(CUdevice*, int);
typedef CUresult (*PrimaryCtxStateFn)(CUdevice, unsigned int*, int*);
std::once_flag g_ctx_fns_once;
DeviceGetFn g_device_get = nullptr;
PrimaryCtxStateFn g_primary_ctx_state = nullptr;

bool primary_context_active(int ordinal) {
  std::call_once(g_ctx_fns_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuDeviceGet", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_device_get = reinterpret_cast<DeviceGetFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuDevicePrimaryCtxGetState", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_primary_ctx_state = reinterpret_cast<PrimaryCtxStateFn>(fn);
    (void)cudaGetLastError();
  });
  if (!g_device_get || !g_primary_ctx_state) return false;
  CUdevice d;
  if (g_device_get(&d, ordinal) != CUDA_SUCCESS) return false;
  unsigned flags = 0;
  int active = 0;
  return g_primary_ctx_state(d, &flags, &active) == CUDA_SUCCESS && active != 0;
}

struct DeviceRestore {
  int prev = -1;
  DeviceRestore() {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      prev = -1;
      (void)cudaGetLastError();
    }
  }
  ~DeviceRestore() {
    int cur = -1;
    if (prev < 0 || cudaGetDevice(&cur) != cudaSuccess || cur == prev) return;
    if (primary_context_active(prev) && cudaSetDevice(prev) != cudaSuccess)
      (void)cudaGetLastError();  // leave no stale error for the caller's next check
  }
  DeviceRestore(const DeviceRestore&) = delete;
  DeviceRestore& operator=(const DeviceRestore&) = delete;
};

// Per-device set-up (once): capability check, status-word address, kernel attributes.
// `ptr` (optional) is a device pointer of the call: its device is made current on the
// calling thread first, so that a call from any host thread (autograd's worker thread,
// for one) runs on the device that owns the tensors with its context current.
attn_status device_setup(DeviceState** out, const void* ptr = nullptr) {
  int dev = 0;
  cudaError_t e0 = cudaSuccess;
  if (ptr) {
    cudaPointerAttributes attr;
    e0 = cudaPointerGetAttributes(&attr, ptr);
    if (e0 != cudaSuccess) return fail_cuda("cudaPointerGetAttributes", e0);
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
      return fail_cuda("tensor pointer is not device memory", cudaErrorInvalidValue);
    e0 = cudaSetDevice(attr.device);
    if (e0 != cudaSuccess) return fail_cuda("cudaSetDevice", e0);
  }
  e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return fail_cuda("cudaGetDevice", e0);
  if (dev < 0 || dev >= kMaxDevices) return fail_cuda("device index", cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp prop;
    if ((e0 = cudaGetDeviceProperties(&prop, dev)) != cudaSuccess)
      return fail_cuda("cudaGetDeviceProperties", e0);
    d.sm100 = (prop.major == 10 && prop.minor == 0);
    if (d.sm100) {
      if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        e0 = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e0 != cudaSuccess) return fail_cuda("cudaGetDriverEntryPoint", e0);
        if (q != cudaDriverEntryPointSuccess || !fn)
          return fail_cuda("cuTensorMapEncodeTiled lookup", cudaErrorSymbolNotFound);
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
      if ((e0 = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_attn_status)) !=
          cudaSuccess)
        return fail_cuda("cudaGetSymbolAddress(status)", e0);
      cudaError_t e = cudaSuccess;
      e = e ? e : cudaFuncSetAttribute(fwd::attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, fwd::Cfg<64>::SMEM_ALLOC);
      e = e ? e : cudaFuncSetAttribute(fwd::attn_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, fwd::Cfg<128>::SMEM_ALLOC);
      e = e ? e : cudaFuncSetAttribute(fwd::attn_fwd_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, fwd::Cfg<128, true>::SMEM_ALLOC);
      e = e ? e : cudaFuncSetAttribute(bwd::attn_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, bwd::Cfg<64>::SMEM_ALLOC);
      e = e ? e : cudaFuncSetAttribute(bwd::attn_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, bwd::Cfg<128>::SMEM_ALLOC);
      e = e ? e : cudaFuncSetAttribute(decode::attn_decode_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, decode::Cfg<64>::SMEM_ALLOC);
      e = e ? e : cudaFuncSetAttribute(decode::attn_decode_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, decode::Cfg<128>::SMEM_ALLOC);
      e = e ? e : cudaFuncSetAttribute(selftest::umma_selftest_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, 32768 + 128 * 64 * 2 + 2048);
      e = e ? e : cudaFuncSetAttribute(selftest::umma_selftest_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, 32768 + 128 * 128 * 2 + 2048);
      if (e != cudaSuccess) return fail_cuda("cudaFuncSetAttribute", e);
      // The kernels re-split registers between warpgroups with setmaxnreg; that is only
      // safe when each thread starts with exactly the budget the split was sized for.
      const void* split_kernels[7] = {
          reinterpret_cast<const void*>(fwd::attn_fwd_kernel<64>),
          reinterpret_cast<const void*>(fwd::attn_fwd_kernel<128>),
          reinterpret_cast<const void*>(fwd::attn_fwd_kernel<128, true>),
          reinterpret_cast<const void*>(bwd::attn_bwd_kernel<64>),
          reinterpret_cast<const void*>(bwd::attn_bwd_kernel<128>),
          reinterpret_cast<const void*>(decode::attn_decode_kernel<64>),
          reinterpret_cast<const void*>(decode::attn_decode_kernel<128>)};
      const int split_regs[7] = {fwd::kRegsLaunch, fwd::kRegsLaunch, fwd::kRegsLaunch,
                                 bwd::kRegsLaunch, bwd::kRegsLaunch, decode::kRegsLaunch,
                                 decode::kRegsLaunch};
      for (int i = 0; i < 7; ++i) {
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, split_kernels[i])) != cudaSuccess)
          return fail_cuda("cudaFuncGetAttributes", e);
        if (fa.numRegs != split_regs[i]) {
          snprintf(g_last_error, sizeof(g_last_error),
                   "kernel %d compiled with %d registers per thread, register split needs %d", i,
                   fa.numRegs, split_regs[i]);
          return ATTN_ERR_UNSUPPORTED;
        }
      }
      // The merge kernels are grid-stride: one wave of resident blocks.
      const void* merge_kernels[2][merge::kVariants] = {
          {reinterpret_cast<const void*>(merge::attn_merge_kernel<64, 1, 4>),
           reinterpret_cast<const void*>(merge::attn_merge_kernel<64, 2, 2>),
           reinterpret_cast<const void*>(merge::attn_merge_kernel<64, 4, 1>)},
          {reinterpret_cast<const void*>(merge::attn_merge_kernel<128, 1, 4>),
           reinterpret_cast<const void*>(merge::attn_merge_kernel<128, 2, 2>),
           reinterpret_cast<const void*>(merge::attn_merge_kernel<128, 4, 1>)}};
      for (int i = 0; i < 2; ++i)
        for (int v = 0; v < merge::kVariants; ++v) {
          int per_sm = 0;
          if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, merge_kernels[i][v],
                                                                 merge::kThreads, 0)) != cudaSuccess)
            return fail_cuda("cudaOccupancyMaxActiveBlocksPerMultiprocessor", e);
          d.merge_grid[i][v] = unsigned(prop.multiProcessorCount) * unsigned(per_sm > 0 ? per_sm : 1);
        }
      {
        int per_sm = 0;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                 &per_sm, relayout::transpose_blocks_kernel, relayout::kThreads, 0)) != cudaSuccess)
          return fail_cuda("cudaOccupancyMaxActiveBlocksPerMultiprocessor", e);
        d.relayout_grid = unsigned(prop.multiProcessorCount) * unsigned(per_sm > 0 ? per_sm : 1);
      }
    }
    d.sms = unsigned(prop.multiProcessorCount);
    d.ready = true;
  }
  if (!d.sm100) return ATTN_ERR_UNSUPPORTED;
  *out = &d;
  return ATTN_OK;
}

// 3-D view (D, H, T) of a [T][H][D] bf16 tensor; box 64 x 1 x 128, 128-byte swizzle.
attn_status make_map(CUtensorMap* m, const void* base, int D, int H, long long T) {
  const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(T)};
  const cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(H) * D * 2};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                              strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : fail_cu("cuTensorMapEncodeTiled", r);
}

// 3-D view (D, H, T) of a [T][H][D] 1-byte (e4m3) tensor; box 128 x 1 x 128, 128-byte swizzle.
attn_status make_map_u8(CUtensorMap* m, const void* base, int D, int H, long long T) {
  const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(T)};
  const cuuint64_t strides[2] = {cuuint64_t(D), cuuint64_t(H) * D};
  const cuuint32_t box[3] = {128, 1, 128};
  const cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                              strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : fail_cu("cuTensorMapEncodeTiled (u8)", r);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

attn_status check_sizes(int B, int Hq, int Hkv, int S, int D, float scale, bool varlen,
                        long long* T) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  const long long t = varlen ? (long long)S : (long long)B * S;
  // token coordinates are int32 in the kernels; keep every row index in range
  if (t >= (1ll << 31) - 512 || ((t >> 7) + B + 1) * (long long)Hq >= (1ll << 31))
    return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  *T = t;
  return ATTN_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Grid of the forward kernel.  Dense batches at D = 128: persistent, one CTA per SM (its
// shared memory admits one), each taking a fixed share of the items -- their lengths are
// known from the item index alone, so the alternating rounds balance them.  Otherwise one
// CTA per item, and the hardware block scheduler hands out the next item as an SM frees
// up: packed lengths sit in device memory, where the host cannot see them, and at D = 64
// the dynamic order measured faster (interleaved medians on the MHA D=64 16K shape:
// 6.85 ms against 7.04 ms persistent; at the 32K D=128 shape 7.42 against 7.44, equal).
unsigned fwd_grid(unsigned nitems, unsigned sms, bool packed, int D) {
  if (packed || D != 128) return nitems;
  return nitems < sms ? nitems : sms;
}

struct WsLayout {
  size_t dq_acc, lse2, delta, total;
  int ntile;
};
WsLayout ws_layout(int B, int Hq, long long T, int D) {
  WsLayout w;
  w.ntile = int((T >> 7) + B);
  w.dq_acc = 0;
  w.lse2 = round_up(size_t(Hq) * w.ntile * 128 * D * sizeof(float), 256);
  w.delta = w.lse2 + round_up(size_t(Hq) * w.ntile * 128 * sizeof(float), 256);
  w.total = w.delta + round_up(size_t(Hq) * w.ntile * 128 * sizeof(float), 256);
  return w;
}

// Split plan of decode: tiles per split and splits per (sequence, kv head), a function
// of the shapes only (so the workspace size needs no device query).  Aims at about four
// CTAs per SM of a 148-SM B200 in total (one CTA is resident per SM, so later CTAs fill
// the gaps that uneven sequence lengths leave), with at least four 128-key tiles per
// split.  When that gives less than two waves, one exact wave is better: every CTA then
// starts at once and no SM waits on a second round.  At most decode_max_splits()
// partial results.  (Measured on 16 x 16K-32K keys: 140 us with this plan, 161 us with
// two CTAs per SM; on one 32K sequence: 34 us in one wave, 38 us in 1.7 waves.)
constexpr int kPlanSMs = 148;
int decode_max_splits() { return decode::kMaxSplits; }
void decode_plan(int B, int Hkv, int Lmax, int* nsplit, int* tps) {
  const long long ntile = (Lmax + 127) / 128;
  const long long units = (long long)B * Hkv;
  long long t = (units * ntile + 4 * kPlanSMs - 1) / (4 * kPlanSMs);
  if (t < 4) t = 4;
  if (t > ntile) t = ntile;
  long long ns = (ntile + t - 1) / t;
  if (units * ns < 2 * kPlanSMs) {
    long long ns1 = kPlanSMs / units;
    if (ns1 < 1) ns1 = 1;
    t = (ntile + ns1 - 1) / ns1;
    if (t < 4) t = 4;
    if (t > ntile) t = ntile;
    ns = (ntile + t - 1) / t;
  }
  if (ns > decode_max_splits()) {
    ns = decode_max_splits();
    t = (ntile + ns - 1) / ns;
    ns = (ntile + t - 1) / t;
  }
  *nsplit = int(ns);
  *tps = int(t);
}
struct DecodeWs {
  size_t o_part, lse_part, flags, total;
  int nsplit, tps, nparts;
};
DecodeWs decode_ws(int B, int Hq, int Hkv, int Lmax, int D) {
  DecodeWs w;
  decode_plan(B, Hkv, Lmax, &w.nsplit, &w.tps);
  w.nparts = w.nsplit;  // each split combines its two streams into one partial
  const size_t rows = size_t(B) * Hq;
  w.o_part = 0;
  w.lse_part = round_up(size_t(w.nparts) * rows * D * 2, 256);
  w.flags = w.lse_part + round_up(size_t(w.nparts) * rows * 4, 256);
  w.total = w.flags + round_up(size_t(B) * Hkv * w.nsplit * 8, 256);
  return w;
}

// Tag of a decode call (64 bits, nonzero): a split's done flag counts only when it holds
// the current call's tag.  The sequence starts at a value drawn from the clock and the
// process id, so that workspaces written by other processes are unlikely to hold a live
// tag.
unsigned long long next_decode_tag() {
  static std::atomic<unsigned long long> ctr{0};
  static const unsigned long long base = [] {
    unsigned long long x = static_cast<unsigned long long>(
        std::chrono::high_resolution_clock::now().time_since_epoch().count());
    x ^= static_cast<unsigned long long>(getpid()) << 32;
    x += 0x9E3779B97F4A7C15ull;  // SplitMix64 finaliser, to spread nearby seeds
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
  }();
  const unsigned long long t = base + ctr.fetch_add(1);
  return t ? t : 1;
}
attn_status check_decode_sizes(int B, int Hq, int Hkv, int Lmax, int D, float scale) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 1) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || Hq / Hkv > 128) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * Lmax >= (1ll << 31) - 256 || (long long)B * Hq >= (1ll << 31) - 256)
    return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_version(void) { return 100; }

const char* attn_last_error(void) { return g_last_error; }

const char* attn_strerror(attn_status s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported (head dim must be 64 or 128 on an sm_100 device)";
    case ATTN_ERR_MISALIGNED: return "misaligned pointer";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

void attn_set_wait_timeout_ns(unsigned long long ns) { g_timeout_ns.store(ns ? ns : 1); }

attn_status attn_check_cu_seqlens(const int32_t* cu, int B, int S) {
  if (!cu || B < 1 || S < 0) return ATTN_ERR_INVALID_ARG;
  if (cu[0] != 0 || cu[B] != S) return ATTN_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (cu[b + 1] < cu[b]) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int S, int D, int causal, float scale,
                     const int32_t* cu_seqlens, void* stream) {
  DeviceRestore restore_device;
  long long T = 0;
  attn_status st = check_sizes(B, Hq, Hkv, S, D, scale, cu_seqlens != nullptr, &T);
  if (st != ATTN_OK) return st;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || (cu_seqlens && !aligned(cu_seqlens, 4)))
    return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  if ((st = device_setup(&dev, q)) != ATTN_OK) return st;

  CUtensorMap mq, mk, mv;
  if (make_map(&mq, q, D, Hq, T) || make_map(&mk, k, D, Hkv, T) || make_map(&mv, v, D, Hkv, T))
    return ATTN_ERR_CUDA;  // reason recorded by make_map
  fwd::Params p;
  p.sv = SeqView{cu_seqlens, B, cu_seqlens ? int(T) : S, int(T)};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.T = int(T);
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_scale = 1.f;
  p.nblk = int((T >> 8) + B);
  p.nitems = p.nblk * Hq;
  p.status = dev->status;
  p.timeout_ns = g_timeout_ns.load();
  const dim3 grid(fwd_grid(unsigned(p.nitems), dev->sms, cu_seqlens != nullptr, D));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (D == 64)
    fwd::attn_fwd_kernel<64><<<grid, fwd::kThreads, fwd::Cfg<64>::SMEM_ALLOC, s>>>(mq, mk, mv, p);
  else
    fwd::attn_fwd_kernel<128><<<grid, fwd::kThreads, fwd::Cfg<128>::SMEM_ALLOC, s>>>(mq, mk, mv, p);
  return check_launch("attn_fwd_kernel launch");
}

attn_status attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int Hq, int Hkv, int S, int D, int causal, float scale, float q_descale,
                         float k_descale, float v_descale, const int32_t* cu_seqlens,
                         void* stream) {
  DeviceRestore restore_device;
  long long T = 0;
  attn_status st = check_sizes(B, Hq, Hkv, S, D, scale, cu_seqlens != nullptr, &T);
  if (st != ATTN_OK) return st;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(q_descale) || !std::isfinite(k_descale) || !std::isfinite(v_descale) ||
      !std::isfinite(scale * q_descale * k_descale))
    return ATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || (cu_seqlens && !aligned(cu_seqlens, 4)))
    return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  if ((st = device_setup(&dev, q)) != ATTN_OK) return st;
  CUtensorMap mq, mk, mv;
  if (make_map_u8(&mq, q, D, Hq, T) || make_map_u8(&mk, k, D, Hkv, T) || make_map_u8(&mv, v, D, Hkv, T))
    return ATTN_ERR_CUDA;
  fwd::Params p;
  p.sv = SeqView{cu_seqlens, B, cu_seqlens ? int(T) : S, int(T)};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.T = int(T);
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * q_descale * k_descale * 1.4426950408889634f;
  p.o_scale = v_descale;
  p.nblk = int((T >> 8) + B);
  p.nitems = p.nblk * Hq;
  p.status = dev->status;
  p.timeout_ns = g_timeout_ns.load();
  const dim3 grid(fwd_grid(unsigned(p.nitems), dev->sms, cu_seqlens != nullptr, D));
  fwd::attn_fwd_kernel<128, true><<<grid, fwd::kThreads, fwd::Cfg<128, true>::SMEM_ALLOC,
                                    static_cast<cudaStream_t>(stream)>>>(mq, mk, mv, p);
  return check_launch("attn_fwd_kernel<fp8> launch");
}

size_t attn_bwd_workspace_size(int B, int Hq, int S, int D, const int32_t* cu_seqlens) {
  long long T = 0;
  if (check_sizes(B, Hq, 1, S, D, 1.f, cu_seqlens != nullptr, &T) != ATTN_OK) return 0;
  return ws_layout(B, Hq, T, D).total;
}

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                     int Hq, int Hkv, int S, int D, int causal, float scale,
                     const int32_t* cu_seqlens, void* workspace, size_t workspace_bytes,
                     void* stream) {
  DeviceRestore restore_device;
  long long T = 0;
  attn_status st = check_sizes(B, Hq, Hkv, S, D, scale, cu_seqlens != nullptr, &T);
  if (st != ATTN_OK) return st;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return ATTN_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(B, Hq, T, D);
  if (workspace_bytes < w.total) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || !aligned(workspace, 256) || (cu_seqlens && !aligned(cu_seqlens, 4)))
    return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  if ((st = device_setup(&dev, q)) != ATTN_OK) return st;

  CUtensorMap mq, mk, mv, mdo;
  if (make_map(&mq, q, D, Hq, T) || make_map(&mk, k, D, Hkv, T) || make_map(&mv, v, D, Hkv, T) ||
      make_map(&mdo, dout, D, Hq, T))
    return ATTN_ERR_CUDA;  // reason recorded by make_map
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws + w.dq_acc);
  float* lse2 = reinterpret_cast<float*>(ws + w.lse2);
  float* delta = reinterpret_cast<float*>(ws + w.delta);
  const SeqView sv{cu_seqlens, B, cu_seqlens ? int(T) : S, int(T)};
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const dim3 pgrid(unsigned(w.ntile), unsigned(Hq));
  if (D == 64)
    bwd::bwd_preprocess_kernel<64><<<pgrid, 128, 0, s>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, lse2,
        delta, dq_acc, sv, Hq, int(T), w.ntile);
  else
    bwd::bwd_preprocess_kernel<128><<<pgrid, 128, 0, s>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, lse2,
        delta, dq_acc, sv, Hq, int(T), w.ntile);
  if ((st = check_launch("bwd_preprocess_kernel launch")) != ATTN_OK) return st;

  bwd::Params p;
  p.sv = sv;
  p.dq_acc = dq_acc;
  p.lse2 = lse2;
  p.delta = delta;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.T = int(T);
  p.causal = causal ? 1 : 0;
  p.ntile = w.ntile;
  // Group-major CTA order once one kv head's tiles fill a wave of the GPU (measured on
  // 28/4 heads, D = 128: 32K tokens 23.2 -> 22.4 ms; at 8K, 65 tiles a group, it would
  // start the longest tiles of the last groups late: 1.51 -> 2.02 ms).
  p.group_major = (!cu_seqlens && unsigned(w.ntile) >= dev->sms) ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.scale = scale;
  p.status = dev->status;
  p.timeout_ns = g_timeout_ns.load();
  const dim3 grid(unsigned(w.ntile) * unsigned(Hkv));
  if (D == 64)
    bwd::attn_bwd_kernel<64><<<grid, bwd::kThreads, bwd::Cfg<64>::SMEM_ALLOC, s>>>(mq, mk, mv, mdo, p);
  else
    bwd::attn_bwd_kernel<128><<<grid, bwd::kThreads, bwd::Cfg<128>::SMEM_ALLOC, s>>>(mq, mk, mv, mdo, p);
  if ((st = check_launch("attn_bwd_kernel launch")) != ATTN_OK) return st;

  if (D == 64)
    bwd::dq_convert_kernel<64><<<pgrid, 256, 0, s>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), sv, Hq,
                                                    w.ntile, scale);
  else
    bwd::dq_convert_kernel<128><<<pgrid, 256, 0, s>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), sv,
                                                     Hq, w.ntile, scale);
  return check_launch("dq_convert_kernel launch");
}

attn_status attn_merge(const void* const* o_parts, const float* const* lse_parts, int nparts,
                       void* o, float* lse, int B, int H, int S, int D, void* stream) {
  DeviceRestore restore_device;
  if (nparts < 1 || nparts > ATTN_MERGE_MAX_PARTS || !o_parts || !lse_parts || !o || !lse)
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || S < 1) return ATTN_ERR_INVALID_ARG;
  const long long rows = (long long)B * S * H;
  if (rows >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  merge::Params p;
  for (int j = 0; j < nparts; ++j) {
    if (!o_parts[j] || !lse_parts[j]) return ATTN_ERR_INVALID_ARG;
    if (!aligned(o_parts[j], 16) || !aligned(lse_parts[j], 4)) return ATTN_ERR_MISALIGNED;
    p.o_parts[j] = static_cast<const uint4*>(o_parts[j]);
    p.lse_parts[j] = lse_parts[j];
  }
  for (int j = nparts; j < merge::kMaxParts; ++j) {
    p.o_parts[j] = nullptr;
    p.lse_parts[j] = nullptr;
  }
  if (!aligned(o, 16) || !aligned(lse, 4)) return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev, o);
  if (st != ATTN_OK) return st;
  p.o = static_cast<uint4*>(o);
  p.lse = lse;
  p.nparts = nparts;
  p.H = unsigned(H);
  p.S = unsigned(S);
  p.rows = unsigned(rows);
  const int var = merge::variant_for(nparts);
  const unsigned rows_per_block =
      unsigned(merge::kThreads / (D / 8)) * unsigned(merge::kVariantRows[var]);
  const unsigned need = unsigned((rows + rows_per_block - 1) / rows_per_block);
  const unsigned wave = dev->merge_grid[D == 64 ? 0 : 1][var];
  const dim3 grid(need < wave ? need : wave);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned thr = merge::kThreads;
  if (D == 64) {
    if (var == 0) merge::attn_merge_kernel<64, 1, 4><<<grid, thr, 0, s>>>(p);
    else if (var == 1) merge::attn_merge_kernel<64, 2, 2><<<grid, thr, 0, s>>>(p);
    else merge::attn_merge_kernel<64, 4, 1><<<grid, thr, 0, s>>>(p);
  } else {
    if (var == 0) merge::attn_merge_kernel<128, 1, 4><<<grid, thr, 0, s>>>(p);
    else if (var == 1) merge::attn_merge_kernel<128, 2, 2><<<grid, thr, 0, s>>>(p);
    else merge::attn_merge_kernel<128, 4, 1><<<grid, thr, 0, s>>>(p);
  }
  return check_launch("attn_merge_kernel launch");
}

size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int D) {
  if (check_decode_sizes(B, Hq, Hkv, Lmax, D, 1.f) != ATTN_OK) return 0;
  return decode_ws(B, Hq, Hkv, Lmax, D).total;
}

attn_status attn_decode(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* cache_len, void* o, float* lse, int B, int Hq, int Hkv,
                        int Lmax, int D, float scale, void* workspace, size_t workspace_bytes,
                        void* stream) {
  DeviceRestore restore_device;
  attn_status st = check_decode_sizes(B, Hq, Hkv, Lmax, D, scale);
  if (st != ATTN_OK) return st;
  if (!q || !k_cache || !v_cache || !cache_len || !o || !lse || !workspace)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
      !aligned(workspace, 256) || !aligned(lse, 4) || !aligned(cache_len, 4))
    return ATTN_ERR_MISALIGNED;
  const DecodeWs w = decode_ws(B, Hq, Hkv, Lmax, D);
  if (workspace_bytes < w.total) return ATTN_ERR_INVALID_ARG;
  DeviceState* dev = nullptr;
  if ((st = device_setup(&dev, q)) != ATTN_OK) return st;

  CUtensorMap mq, mk, mv;
  if (make_map(&mq, q, D, 1, (long long)B * Hq) || make_map(&mk, k_cache, D, Hkv, (long long)B * Lmax) ||
      make_map(&mv, v_cache, D, Hkv, (long long)B * Lmax))
    return ATTN_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  decode::Params p;
  p.cache_len = cache_len;
  p.o_part = reinterpret_cast<__nv_bfloat16*>(ws + w.o_part);
  p.lse_part = reinterpret_cast<float*>(ws + w.lse_part);
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.Hkv = Hkv;
  p.Lmax = Lmax;
  p.nsplit = w.nsplit;
  p.tps = w.tps;
  p.rows = B * Hq;
  p.flags = reinterpret_cast<unsigned long long*>(ws + w.flags);
  p.tag = next_decode_tag();
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = dev->status;
  p.timeout_ns = g_timeout_ns.load();
  const long long nblocks = (long long)B * Hkv * w.nsplit;
  if (nblocks >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (D == 64)
    decode::attn_decode_kernel<64><<<unsigned(nblocks), decode::kThreads, decode::Cfg<64>::SMEM_ALLOC, s>>>(mq, mk, mv, p);
  else
    decode::attn_decode_kernel<128><<<unsigned(nblocks), decode::kThreads, decode::Cfg<128>::SMEM_ALLOC, s>>>(mq, mk, mv, p);
  return check_launch("attn_decode_kernel launch");
}

attn_status attn_accumulate_bf16(float* acc, const void* x, long long n, int init, void* stream) {
  DeviceRestore restore_device;
  if (!acc || !x || n < 1) return ATTN_ERR_INVALID_ARG;
  if (n % 8) return ATTN_ERR_INVALID_ARG;
  if (!aligned(acc, 16) || !aligned(x, 16)) return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev, acc);
  if (st != ATTN_OK) return st;
  const long long n8 = n / 8;
  const long long need = (n8 + accum::kThreads - 1) / accum::kThreads;
  const long long wave = (long long)dev->sms * 8;
  accum::add_bf16_to_f32_kernel<<<unsigned(need < wave ? need : wave), accum::kThreads, 0,
                                  static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<float4*>(acc), static_cast<const uint4*>(x), n8, init ? 1 : 0);
  return check_launch("add_bf16_to_f32_kernel launch");
}

attn_status attn_convert_f32_bf16(void* out, const float* in, long long n, void* stream) {
  DeviceRestore restore_device;
  if (!out || !in || n < 1) return ATTN_ERR_INVALID_ARG;
  if (n % 8) return ATTN_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(in, 16)) return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev, in);
  if (st != ATTN_OK) return st;
  const long long n8 = n / 8;
  const long long need = (n8 + accum::kThreads - 1) / accum::kThreads;
  const long long wave = (long long)dev->sms * 8;
  accum::f32_to_bf16_kernel<<<unsigned(need < wave ? need : wave), accum::kThreads, 0,
                              static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(out), reinterpret_cast<const float4*>(in), n8);
  return check_launch("f32_to_bf16_kernel launch");
}

attn_status attn_transpose_blocks(const void* in, void* out, long long n_outer, long long n_inner,
                                  long long block_bytes, void* stream) {
  DeviceRestore restore_device;
  if (!in || !out || n_outer < 1 || n_inner < 1 || block_bytes < 16) return ATTN_ERR_INVALID_ARG;
  if (block_bytes % 16) return ATTN_ERR_MISALIGNED;
  if (!aligned(in, 16) || !aligned(out, 16)) return ATTN_ERR_MISALIGNED;
  const long long vec = block_bytes / 16;
  if (n_outer >= (1ll << 31) || n_inner >= (1ll << 31) || vec >= (1ll << 31) ||
      (double)n_outer * (double)n_inner * (double)vec >= 2147483648.0)
    return ATTN_ERR_INVALID_ARG;
  const long long total = n_outer * n_inner * vec;
  const uintptr_t a = reinterpret_cast<uintptr_t>(in), b = reinterpret_cast<uintptr_t>(out);
  const uintptr_t span = uintptr_t(total) * 16;
  if (a < b + span && b < a + span) return ATTN_ERR_INVALID_ARG;  // in and out overlap
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev, in);
  if (st != ATTN_OK) return st;
  relayout::Params p;
  p.in = static_cast<const uint4*>(in);
  p.out = static_cast<uint4*>(out);
  p.n_outer = unsigned(n_outer);
  p.n_inner = unsigned(n_inner);
  p.vec = unsigned(vec);
  p.total = unsigned(total);
  const long long per_pass = (long long)relayout::kThreads * relayout::kUnroll;
  const unsigned need = unsigned((total + per_pass - 1) / per_pass);
  const dim3 grid(need < dev->relayout_grid ? need : dev->relayout_grid);
  relayout::transpose_blocks_kernel<<<grid, relayout::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return check_launch("transpose_blocks_kernel launch");
}

attn_status attn_device_status(void* stream, unsigned* site) {
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda("cudaStreamSynchronize", e);
  unsigned word[2] = {0, 0};
  if ((e = cudaMemcpy(word, dev->status, sizeof(word), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return fail_cuda("cudaMemcpy(status)", e);
  if (site) *site = word[1];
  if (word[0] == 0) return ATTN_OK;
  const unsigned zero[2] = {0, 0};
  if ((e = cudaMemcpy(dev->status, zero, sizeof(zero), cudaMemcpyHostToDevice)) != cudaSuccess)
    return fail_cuda("cudaMemcpy(status reset)", e);
  return (word[0] & kStatusTimeout) ? ATTN_ERR_TIMEOUT : ATTN_ERR_CUDA;
}

}  // extern "C"

// ------------------------------------------------------------------ self-tests
static __global__ void wait_timeout_kernel(unsigned* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl wc{status, &abort_flag, timeout_ns};
    mbar_wait(&bar, 0, wc, 0x400);  // nothing ever arrives: the wait gives up
  }
}

extern "C" attn_status attn_selftest_wait_timeout(unsigned long long timeout_ns, void* stream) {
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev->status, timeout_ns);
  return check_launch("wait_timeout_kernel launch");
}

extern "C" attn_status attn_selftest_umma(int mode, int D, const void* a, const void* b,
                                          const float* pin, const void* at, float* c,
                                          void* stream) {
  DeviceRestore restore_device;
  if (mode < 0 || mode > 2) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (!b || !c || (mode == 0 && !a) || (mode == 1 && !pin) || (mode == 2 && !at))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned(b, 16) || (a && !aligned(a, 16)) || (at && !aligned(at, 16)) ||
      (pin && !aligned(pin, 16)) || !aligned(c, 16))
    return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev, b);
  if (st != ATTN_OK) return st;
  CUtensorMap ma, mb;
  if (make_map(&ma, a ? a : b, D, 1, 128) || make_map(&mb, b, D, 1, 128)) return ATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned long long to = g_timeout_ns.load();
  if (D == 64)
    selftest::umma_selftest_kernel<64><<<1, 128, 32768 + 128 * 64 * 2 + 2048, s>>>(
        ma, mb, mode, pin, static_cast<const __nv_bfloat16*>(at), c, dev->status, to);
  else
    selftest::umma_selftest_kernel<128><<<1, 128, 32768 + 128 * 128 * 2 + 2048, s>>>(
        ma, mb, mode, pin, static_cast<const __nv_bfloat16*>(at), c, dev->status, to);
  return check_launch("umma_selftest_kernel launch");
}

extern "C" attn_status attn_selftest_umma_fp8(int mode, const void* a, const void* b,
                                              const float* pin, float* pq, float* c, void* stream) {
  DeviceRestore restore_device;
  if (mode != 3 && mode != 4) return ATTN_ERR_INVALID_ARG;
  if (!b || !c || (mode == 3 && !a) || (mode == 4 && (!pin || !pq))) return ATTN_ERR_INVALID_ARG;
  if (!aligned(b, 16) || (a && !aligned(a, 16)) || (pin && !aligned(pin, 16)) ||
      (pq && !aligned(pq, 16)) || !aligned(c, 16))
    return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev, b);
  if (st != ATTN_OK) return st;
  CUtensorMap ma, mb;
  if (make_map_u8(&ma, a ? a : b, 128, 1, 128) || make_map_u8(&mb, b, 128, 1, 128))
    return ATTN_ERR_CUDA;
  selftest::umma_selftest_fp8_kernel<<<1, 128, 2 * 128 * 128 + 2048, static_cast<cudaStream_t>(stream)>>>(
      ma, mb, mode, pin, pq, c, dev->status, g_timeout_ns.load());
  return check_launch("umma_selftest_fp8_kernel launch");
}

static __global__ void exp2_selftest_kernel(const float2* __restrict__ x, float2* __restrict__ y,
                                            long long n2) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n2;
       i += (long long)gridDim.x * blockDim.x) {
    const float2 a = x[i];
    float r0, r1;
    f2_unpack(exp2_poly_x2(a.x, a.y), r0, r1);
    y[i] = make_float2(r0, r1);
  }
}

extern "C" attn_status attn_selftest_exp2(const float* x, float* y, long long n, void* stream) {
  DeviceRestore restore_device;
  if (!x || !y || n < 2 || (n & 1)) return ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16)) return ATTN_ERR_MISALIGNED;
  DeviceState* dev = nullptr;
  attn_status st = device_setup(&dev, x);
  if (st != ATTN_OK) return st;
  const long long n2 = n / 2;
  const long long need = (n2 + 255) / 256;
  const long long wave = (long long)dev->sms * 8;
  exp2_selftest_kernel<<<unsigned(need < wave ? need : wave), 256, 0,
                         static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float2*>(x), reinterpret_cast<float2*>(y), n2);
  return check_launch("exp2_selftest_kernel launch");
}

// ------------------------------------------------------------------ backward without allocation
// Some callers cannot hand this library a workspace: they have no device allocator at the
// call site (a plugin interface that passes only the tensors of one operation), or their
// runtime reserves all device memory at start-up and forbids allocation afterwards.  For
// them attn_bwd_noalloc runs the same backward on a fixed scratch array that lives in the
// library itself.  Every GPU that loads the library keeps this array until the process
// exits, so its size is kept modest; problems whose workspace is larger are refused.
static __device__ __align__(256) uint8_t g_bwd_scratch[ATTN_BWD_NOALLOC_MAX_BYTES];

namespace {
void* g_scratch_ptr[kMaxDevices] = {};  // device address of g_bwd_scratch, per device
std::mutex g_scratch_mu;
}  // namespace

extern "C" attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                        const void* o, const float* lse, const void* dout,
                                        void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                                        int S, int D, int causal, float scale,
                                        const int32_t* cu_seqlens, void* stream) {
  DeviceRestore restore_device;
  const size_t need = attn_bwd_workspace_size(B, Hq, S, D, cu_seqlens);
  if (need == 0) {  // the same size checks attn_bwd applies
    snprintf(g_last_error, sizeof(g_last_error),
             "attn_bwd_noalloc: invalid sizes (B=%d Hq=%d S=%d D=%d)", B, Hq, S, D);
    return ATTN_ERR_INVALID_ARG;
  }
  if (need > size_t(ATTN_BWD_NOALLOC_MAX_BYTES)) {
    snprintf(g_last_error, sizeof(g_last_error),
             "attn_bwd_noalloc: workspace of %zu bytes exceeds the static scratch of %zu bytes",
             need, size_t(ATTN_BWD_NOALLOC_MAX_BYTES));
    return ATTN_ERR_INVALID_ARG;
  }
  if (!q) {
    snprintf(g_last_error, sizeof(g_last_error), "attn_bwd_noalloc: q is a null pointer");
    return ATTN_ERR_INVALID_ARG;
  }
  // Set-up, once per device and with that device current: the array's name is only a
  // host-side stand-in, so its device address is looked up and cached.
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, q);
  if (e != cudaSuccess) return fail_cuda("cudaPointerGetAttributes", e);
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail_cuda("tensor pointer is not device memory", cudaErrorInvalidValue);
  if (attr.device < 0 || attr.device >= kMaxDevices)
    return fail_cuda("device index", cudaErrorInvalidDevice);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[attr.device]) {
      if ((e = cudaSetDevice(attr.device)) != cudaSuccess) return fail_cuda("cudaSetDevice", e);
      void* ptr = nullptr;
      if ((e = cudaGetSymbolAddress(&ptr, g_bwd_scratch)) != cudaSuccess)
        return fail_cuda("cudaGetSymbolAddress(scratch)", e);
      g_scratch_ptr[attr.device] = ptr;
    }
    scratch = g_scratch_ptr[attr.device];
  }
  // Nothing in the scratch needs clearing: the backward's first kernel rewrites every
  // byte the later kernels read (dQ accumulator tiles, LSE and Delta) on each call.
  return attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, causal, scale, cu_seqlens,
                  scratch, size_t(ATTN_BWD_NOALLOC_MAX_BYTES), stream);
}
