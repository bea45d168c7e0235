/*
 * attn.h -- C ABI of libattn.so: exact scaled-dot-product attention, forward and
 * backward, as fused tiled kernels for NVIDIA B200 (sm_100a).
 *
 * What is computed (page "ms-swift集成FlashAttention 2/3，长文本训练更高效"
 * [ms-swift integrates FlashAttention 2/3]): the standard attention of section
 * "为什么传统注意力这么'吃'显存" -- S = scale * Q K^T, a row softmax, O = P V -- computed
 * the way section "FlashAttention 如何破局" describes: Q/K/V tiled along the
 * sequence, an online softmax keeping a running maximum and normaliser per row,
 * and only the output (plus the per-row log-sum-exp) written to global memory.
 * The S x S score matrix never reaches HBM in either direction.
 *
 * Conventions shared by every entry point
 *   - All tensors are row-major and contiguous, bf16 unless stated.
 *     Dense batches (cu_seqlens == NULL): q, o, dO, dq are [B][S][Hq][D];
 *     k, v, dk, dv are [B][S][Hkv][D]; lse is fp32 [B][Hq][S].
 *     Packed batches (cu_seqlens != NULL): B is the number of sequences and S the
 *     total token count T; q is [T][Hq][D], k/v [T][Hkv][D], lse [Hq][T];
 *     cu_seqlens is a DEVICE array of B+1 int32 offsets, 0 = cu[0] <= ... <= cu[B] = T.
 *     Sequences never attend to each other; positions count from each sequence's start.
 *   - Grouped-query attention: query head h reads key/value head h / (Hq/Hkv).
 *   - causal != 0 masks key j for query i when j > i (positions within the sequence).
 *   - lse[i] = ln sum_j exp(scale * q_i . k_j) over the visible keys (natural log).
 *   - D must be 64 or 128; Hq must be a multiple of Hkv; B, Hq, Hkv, S >= 1.
 *   - Every tensor pointer is a device pointer owned by the caller; tensor pointers
 *     must be 16-byte aligned (lse and cu_seqlens 4-byte aligned).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     asynchronous on that stream; arguments are validated synchronously before
 *     anything is launched, and nothing is launched when validation fails.
 *   - Work runs on the device that owns the first tensor argument; the entry point
 *     makes that device current for its launches and, on return, makes the calling
 *     thread's previous device current again when that device's primary context is
 *     active (no context is created on a device the process has not used).  The
 *     stream must belong to the tensors' device.
 *   - No entry point allocates device memory, and no per-call state is kept; the one
 *     exception to "caller-owned memory" is the fixed scratch array attn_bwd_noalloc
 *     works in, which is part of the loaded library.
 *   - A packed batch whose cu_seqlens break the rules above cannot make a kernel read
 *     or write outside the tensors (every sequence is clamped to [0, T)), but its
 *     results are undefined; attn_check_cu_seqlens validates a host copy.
 *   - Device-side waits are bounded; a wait that times out makes the kernel skip
 *     its remaining work and records the event in a sticky status word that
 *     attn_device_status reports.
 *   - The library looks up the device addresses of its own device-side variables (the
 *     status word, attn_bwd_noalloc's scratch array) once per device and keeps them;
 *     a cudaDeviceReset between calls is not supported.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,   /* bad size, null pointer, Hq % Hkv != 0, scale not finite,
                                 workspace too small, malformed host cu_seqlens */
  ATTN_ERR_UNSUPPORTED = 2,   /* D not in {64, 128}, or the device is not sm_100 */
  ATTN_ERR_MISALIGNED = 3,    /* a pointer breaks the alignment rules above */
  ATTN_ERR_CUDA = 4,          /* a CUDA runtime/driver call or a launch failed */
  ATTN_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up (see attn_device_status) */
} attn_status;

/* Forward pass (page section "FlashAttention 如何破局": tiled QK^T -> online softmax -> PV).
 * Writes o (same layout as q) and lse. */
attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int S, int D, int causal, float scale,
                     const int32_t* cu_seqlens, void* stream);

/* FP8 forward (page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section
 * "FlashAttention 如何破局": FlashAttention-3 adds FP8 computation on Hopper; this is the
 * same idea on B200's fifth-generation tensor cores).  q, k, v hold e4m3 values (1 byte,
 * same [T][H][D] layouts as attn_fwd) with per-tensor descale factors: the attention of
 * (q_descale * q, k_descale * k, v_descale * v) is computed, i.e.
 *     s_ij = scale * q_descale * k_descale * (q8_i . k8_j),   o_i = v_descale * sum_j P_ij v8_j.
 * The probabilities are quantised for the P V product as e4m3(256 p) (the factor keeps
 * probabilities down to 2^-14 in e4m3's normal range and cancels in the normalisation,
 * which divides by the sum of exactly the quantised weights).  o is bf16, lse fp32 as in
 * attn_fwd (computed from the unquantised probabilities).  D must be 128
 * (ATTN_ERR_UNSUPPORTED otherwise); descale factors and their product with scale must be
 * finite.  Everything else (masks, GQA, packed batches, errors) as attn_fwd. */
attn_status attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int Hq, int Hkv, int S, int D, int causal, float scale, float q_descale,
                         float k_descale, float v_descale, const int32_t* cu_seqlens,
                         void* stream);

/* Bytes of device workspace attn_bwd needs for these arguments (same meaning as in
 * attn_bwd; only whether cu_seqlens is NULL matters).  Holds, per query head and
 * 128-row query tile, the fp32 dQ accumulator tile, Delta = rowsum(dO * O) and
 * LSE*log2(e); there are (T / 128) + B tiles per head (T = total tokens).
 * Returns 0 for invalid sizes. */
size_t attn_bwd_workspace_size(int B, int Hq, int S, int D, const int32_t* cu_seqlens);

/* Backward pass (page section "为什么传统注意力这么'吃'显存": the intermediates are
 * recomputed, not stored -- P is rebuilt tile by tile from lse).
 * Inputs q, k, v, o, lse (from attn_fwd with the same arguments) and dout = dL/dO;
 * outputs dq, dk, dv (layouts of q, k, v).  dk/dv are summed over the query heads of
 * each group.  `workspace` (>= attn_bwd_workspace_size bytes, 256-byte aligned) is
 * scratch owned by the caller; its contents need no initialisation.
 * dq is accumulated with fp32 atomics, so its last bits can differ run to run;
 * o, lse, dk and dv are deterministic. */
attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                     int Hq, int Hkv, int S, int D, int causal, float scale,
                     const int32_t* cu_seqlens, void* workspace, size_t workspace_bytes,
                     void* stream);

/* Size in bytes of the scratch array attn_bwd_noalloc works in (64 MiB). */
#define ATTN_BWD_NOALLOC_MAX_BYTES (64u << 20)

/* attn_bwd for callers that cannot allocate device memory.  The pages have no
 * counterpart: this exists for integrations that have no device allocator where they
 * call the backward (for example a plugin interface that passes only the tensors of
 * one operation) or whose runtime reserves all device memory up front and forbids
 * allocating later.  Arguments are those of attn_bwd without the workspace; the
 * caller still passes every input and output.
 *   - The scratch is a fixed array of ATTN_BWD_NOALLOC_MAX_BYTES inside the library,
 *     held on every GPU that loads the library until the process exits.  Problems
 *     whose attn_bwd_workspace_size exceeds it are refused with ATTN_ERR_INVALID_ARG
 *     (attn_last_error says why); attn_bwd with a caller workspace has no such limit.
 *   - The first call on a device looks up the array's device address (a set-up step
 *     done once per device, under a lock); make that first call before any stream
 *     capture.  This function allocates nothing and frees nothing.
 *   - All calls share the one array, and each call leaves its contents behind; the
 *     backward rewrites everything it reads, so nothing needs clearing between calls.
 *     Calls whose work overlaps on the GPU (different streams, or different host
 *     threads without ordering) race on the array and corrupt each other's results:
 *     serialise them. */
attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             int B, int Hq, int Hkv, int S, int D, int causal, float scale,
                             const int32_t* cu_seqlens, void* stream);

/* Bytes of device workspace attn_decode needs (0 for invalid sizes).  It holds the
 * per-split partial results, nsplit partials of B*Hq rows (bf16 o and fp32 lse) where
 * nsplit is fixed by (B, Hkv, Lmax), and one 8-byte done flag per split. */
size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int D);

/* Decode attention over a key/value cache: one new query token per sequence attends to
 * all cache_len[b] cached keys of its sequence (page "ms-swift长文本训练秘诀：Ulysses并行技术
 * 解析", section 5: serving the fine-tuned model with a 32K-token context; the arithmetic
 * is the standard attention of page "ms-swift集成FlashAttention 2/3，长文本训练更高效",
 * section "为什么传统注意力这么'吃'显存", one query row against the cache).
 *     o[b][h] = sum_j softmax_j(scale * q[b][h] . k[b][j][g]) v[b][j][g],  g = h / (Hq/Hkv)
 *     lse[b][h] = ln sum_j exp(scale * q[b][h] . k[b][j][g])
 *   - q, o: bf16 [B][Hq][D]; k_cache, v_cache: bf16 [B][Lmax][Hkv][D]; lse: fp32 [B][Hq];
 *     cache_len: DEVICE int32 [B], each clamped to [0, Lmax].  Cache rows at or past
 *     cache_len[b] are never used, whatever they hold.  cache_len[b] = 0 gives o = 0 and
 *     lse = -inf.
 *   - The cache is split along the keys; every split writes a partial (o, lse) into
 *     `workspace` (>= attn_decode_workspace_size bytes, 256-byte aligned, caller-owned),
 *     and the last split of each (sequence, kv head) to finish combines them exactly, in
 *     the same launch.  Each split marks itself done with a flag word holding a 64-bit
 *     tag of the call, so the workspace needs no initialisation (leftover contents count
 *     as another call's, except with probability 2^-64 per word), and a call leaves its
 *     flags cleared.  Two calls whose work overlaps on the GPU must not share a
 *     workspace.
 *   - D in {64, 128}; Hq a multiple of Hkv with Hq/Hkv <= 128; B*Lmax and B*Hq < 2^31.
 *   - Pointers as in every entry point (16-byte aligned tensors, 4-byte lse/cache_len).
 *   - Deterministic. */
attn_status attn_decode(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* cache_len, void* o, float* lse, int B, int Hq, int Hkv,
                        int Lmax, int D, float scale, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Largest number of partial results one attn_merge call combines. */
#define ATTN_MERGE_MAX_PARTS 16

/* Exact merge of partial attention results for the same queries over disjoint key sets
 * (page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠 FlashAttention
 * 不够？那就加上序列并行", subsection "Ring-Attention": K/V chunks travel around a ring of
 * devices and each device accumulates the partial attention of its own queries; page
 * "ms-swift支持GPU显存碎片整理提升利用率" describes the same scheme).  Each partial is the
 * (o, lse) pair attn_fwd returns for one key chunk; per query row
 *     lse = ln sum_p exp(lse_p),   o = sum_p exp(lse_p - lse) * o_p   (fp32, o rounded to bf16),
 * which is the attention over the union of the chunks.  Partials with lse_p = -inf carry
 * no weight; a row whose partials are all -inf gets o = 0, lse = -inf.
 *   - o_parts, lse_parts: HOST arrays of nparts DEVICE pointers (1 <= nparts <=
 *     ATTN_MERGE_MAX_PARTS); o_parts[p] is bf16 [B][S][H][D], lse_parts[p] fp32 [B][H][S]
 *     (the dense layouts of attn_fwd; for a packed batch pass B = 1 and S = T, which is
 *     the packed [T][H][D] / [H][T] layout).
 *   - o, lse: outputs in the same layouts.  o may be o_parts[0] and lse may be
 *     lse_parts[0] (in-place accumulation); any other overlap is undefined.
 *   - D in {64, 128}; B * S * H < 2^31.  Pointers as in every entry point (o 16-byte,
 *     lse 4-byte aligned).  The host arrays are read during the call only. */
attn_status attn_merge(const void* const* o_parts, const float* const* lse_parts, int nparts,
                       void* o, float* lse, int B, int H, int S, int D, void* stream);

/* Accumulation of block gradients for the Ring-Attention backward (page
 * "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠 FlashAttention 不够？
 * 那就加上序列并行", subsection "Ring-Attention": each device computes the share of the
 * result its queries and the passing key/value block contribute; in the backward, the
 * shares -- bf16 outputs of attn_bwd on each block pair -- are summed in fp32):
 *     acc[i] = (init ? 0 : acc[i]) + x[i]        acc fp32, x bf16, i < n
 * DEVICE pointers, 16-byte aligned; n >= 1 and a multiple of 8. */
attn_status attn_accumulate_bf16(float* acc, const void* x, long long n, int init, void* stream);

/* out[i] = bf16(in[i]) (round to nearest even): the final rounding of an fp32 accumulator
 * (same pointer and size rules as attn_accumulate_bf16). */
attn_status attn_convert_f32_bf16(void* out, const float* in, long long n, void* stream);

/* Block transpose for the layout changes around the all-to-alls of Ulysses sequence
 * parallelism (page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠
 * FlashAttention 不够？那就加上序列并行", Ulysses subsection: split the sequence across
 * devices, all-to-all, attention on every device, all-to-all back to restore the order;
 * also page "ms-swift长文本训练秘诀：Ulysses并行技术解析", section 1).  An all-to-all sends
 * contiguous chunk p to rank p, so data bound for one rank is gathered into one chunk
 * before the exchange and interleaved back after it:
 *     `in` is a grid [n_outer][n_inner] of blocks of block_bytes bytes,
 *     `out` is the grid [n_inner][n_outer]:  out[j][i] = in[i][j].
 * Example: q of one rank, [B*C][Hq][D] bf16, seen as [B*C][N][Hq/N * D * 2 bytes] becomes
 * the send buffer [N][B*C][Hq/N][D] (chunk p = the heads of rank p).
 *   - in, out: DEVICE pointers, 16-byte aligned, not overlapping (INVALID_ARG if they do);
 *     block_bytes a multiple of 16 (MISALIGNED otherwise) and >= 16;
 *     n_outer * n_inner * block_bytes / 16 < 2^31.
 *   - A pure copy: bit-exact, no arithmetic. */
attn_status attn_transpose_blocks(const void* in, void* out, long long n_outer, long long n_inner,
                                  long long block_bytes, void* stream);

/* Self-test of the e4m3 (fp8) tensor-core operand layouts (no page counterpart), D = 128,
 * one 128 x 128 tile; a, b are DEVICE e4m3 bytes [128][128], pin/pq/c DEVICE fp32:
 *   mode 3: c = a . b^T                          (both K-major)
 *   mode 4: c = e4m3(256 pin) . b, pq = e4m3(256 pin) read back as fp32 (b MN-major) */
attn_status attn_selftest_umma_fp8(int mode, const void* a, const void* b, const float* pin,
                                   float* pq, float* c, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* attn_strerror(attn_status status);

/* Synchronises `stream`, then returns ATTN_ERR_TIMEOUT if any kernel of this library
 * recorded a timed-out wait on the current device since the last call (and clears
 * the record), ATTN_ERR_CUDA if the stream reports a CUDA error, else ATTN_OK.
 * If `site` is not NULL it receives the code of the first wait that timed out. */
attn_status attn_device_status(void* stream, unsigned* site);

/* Sets the limit of every device-side wait, in nanoseconds (default 2e9). */
void attn_set_wait_timeout_ns(unsigned long long ns);

/* Validates a HOST copy of cu_seqlens: B+1 entries, cu[0] = 0, non-decreasing,
 * cu[B] = S.  Returns ATTN_OK or ATTN_ERR_INVALID_ARG. */
attn_status attn_check_cu_seqlens(const int32_t* cu_host, int B, int S);

/* Self-test of the failure path: launches one CTA that waits on a barrier nobody
 * arrives on, with a limit of `timeout_ns`.  The wait must give up and record a
 * timeout; call attn_device_status afterwards to observe it.  No page counterpart:
 * it exists to test the bounded-wait machinery without faulting the GPU. */
attn_status attn_selftest_wait_timeout(unsigned long long timeout_ns, void* stream);

/* Self-test of the tensor-core operand layouts (no page counterpart).  One 128-row
 * tile, D in {64, 128}; a, b, p, at, c are device pointers:
 *   mode 0: c[128][128] = a[128][D] . b[128][D]^T          (a, b bf16)
 *   mode 1: c[128][D]   = bf16(p[128][128]) . b[128][D]    (p fp32, b bf16)
 *   mode 2: c[128][D]   = at[128][128]^T . b[128][D]       (at, b bf16)
 * c is fp32. */
attn_status attn_selftest_umma(int mode, int D, const void* a, const void* b, const float* p,
                               const void* at, float* c, void* stream);

/* Self-test of the exponential the forward kernel computes on the FMA pipe for a share
 * of its probabilities (no page counterpart): y[i] = 2^x[i] by that polynomial route,
 * for n values (x, y DEVICE fp32, 16-byte aligned, n > 0 and even).  Maximum relative
 * error 2^-18 for x in [-125, 64]; below -125 the result is about 2^-125. */
attn_status attn_selftest_exp2(const float* x, float* y, long long n, void* stream);

/* Description of the last failing CUDA call this library made on the calling thread
 * ("" if none): the call's name and the CUDA error string.  Static per-thread
 * storage, valid until the thread's next library call. */
const char* attn_last_error(void);

/* Library ABI version (major*100 + minor). */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
