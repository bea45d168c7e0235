// attn_common.cuh -- work decomposition shared by the forward and backward kernels.
//
// Sequences: dense batches are treated as packed sequences of equal length S that
// start at b*S; packed batches take their starts from the device array cu_seqlens.
// Tiles never straddle two sequences: sequence s is cut into blocks of 2^LOG rows
// counted from its own start.  Block m of sequence s gets the global index
//     base(s) + m,   base(s) = (start(s) >> LOG) + s,
// which is strictly increasing in s and never collides (ceil(L/2^LOG) blocks fit
// between base(s) and base(s+1)), so a grid of (T >> LOG) + nseq indices covers
// every block without a host-side prefix sum or a device-to-host copy.
#pragma once
#include <cstdint>

namespace attn_sm100 {

// Packed offsets are clamped to [0, T] so that a malformed cu_seqlens array can
// never send a load or store outside the tensors.
struct SeqView {
  const int32_t* cu;  // nullptr: dense
  int nseq;
  int S;              // dense sequence length (ignored when cu != nullptr)
  int T;              // total tokens
  __device__ __forceinline__ int start(int s) const {
    return cu ? min(max(cu[s], 0), T) : s * S;
  }
  __device__ __forceinline__ int len(int s) const {
    if (!cu) return S;
    const int a = start(s);
    return min(max(cu[s + 1], a), T) - a;
  }
};

// Maps a global block index to (sequence, block-in-sequence). Returns false when the
// index falls in the slack after a sequence's last block (no work).
template <int LOG>
__device__ __forceinline__ bool locate_block(const SeqView& sv, int idx, int& seq, int& blk,
                                             int& start, int& len) {
  if (idx < 0) return false;
  int lo = 0, hi = sv.nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((sv.start(mid) >> LOG) + mid <= idx) lo = mid;
    else hi = mid - 1;
  }
  seq = lo;
  start = sv.start(lo);
  len = sv.len(lo);
  blk = idx - ((start >> LOG) + lo);
  const int nblk = (len + (1 << LOG) - 1) >> LOG;
  return blk >= 0 && blk < nblk;
}

}  // namespace attn_sm100
