/*
 * fa.h -- C ABI of the B200 (sm_100a) tiled exact attention library.
 *
 * Exact scaled-dot-product attention
 *     O = softmax(Q K^T * scale + mask) V
 * computed tile by tile with the online softmax (a running row max m and row
 * sum l, the output rescaled by exp(m_old - m_new) when the max grows and
 * divided by l once at the end), so the N x N score matrix never reaches
 * device memory.  Sources, by page title and section:
 *   - "Building Flash Attention from Scratch in Pure NumPy": architecture
 *     overview (per-query-block data flow), Step 2 (online softmax update),
 *     Step 3 (the forward's tile loops and its scale=None default), Step 4
 *     (the backward from the saved row statistics, D = rowsum(dO * O)).
 *   - "Build a FlashAttention-2 Inference Kernel from Scratch in Pure Python":
 *     Steps 2-3 (scale, mask to -inf, causal j <= i, sliding-window skipping);
 *     Extending It (paged KV-cache integration, read as a block pool).
 *   - "Build a FlashAttention Kernel with Online Softmax and KV Cache in Pure
 *     Python": Step 4 (single-query decode against a key/value cache).
 *   - Both pure-Python pages' "Extending It" roadmaps (attention split across
 *     devices, each holding part of the key/value space): the per-shard
 *     forward fa_forward_offset and the partial-result merge fa_merge.
 *
 * Conventions shared by every entry point
 *   - Layout: Q, K, V, O, dO, dQ, dK, dV are contiguous row-major
 *     [B][H][N][d] (d innermost).  lse is float32 [B][H][N].  Decode: q and o
 *     are [B][H][d], the caches [B][H][cap][d], seqlens int32 [B]; paged
 *     decode: pools [num_blocks][H][block_size][d], block table int32
 *     [B][max_blocks].
 *   - Mask: key j is visible to query i iff
 *         (causal == 0 || j <= i) && (window <= 0 || j > i - window),
 *     so a window holds exactly `window` keys including the query itself.
 *   - scale <= 0 selects 1/sqrt(d).
 *   - lse is the natural-log logsumexp of the row's scaled, masked scores.
 *     A row with no visible key gets O = 0 and lse = -inf.
 *   - Pointers are DEVICE pointers unless stated; the caller owns every
 *     buffer, including workspaces.  The library allocates no device memory
 *     and keeps no per-call state.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns without synchronising.
 *   - Argument errors are found on the host before anything is launched:
 *     FA_ERR_INVALID (null pointer, non-positive size, misaligned pointer,
 *     workspace too small, window < 0) or FA_ERR_UNSUPPORTED (a dtype/d
 *     combination with no kernel).  FA_ERR_CUDA reports a failed launch.
 *   - Kernels never trap.  A kernel that waits too long on an internal
 *     barrier records FA_ERR_TIMEOUT in a device status word and returns; a
 *     paged decode that meets a block id outside its pool skips that block and
 *     records FA_ERR_INVALID; fa_get_device_status() reports either.
 */
#ifndef TILED_EXACT_ATTENTION_FA_H_
#define TILED_EXACT_ATTENTION_FA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID = 1,
  FA_ERR_UNSUPPORTED = 2,
  FA_ERR_CUDA = 3,
  FA_ERR_TIMEOUT = 4
} fa_status;

typedef enum {
  FA_BF16 = 0, /* bfloat16 inputs/outputs, float32 accumulation (d = 128)   */
  FA_FP32 = 1, /* float32 inputs/outputs, float32 arithmetic (d = 64 or 128) */
  FA_FP16 = 2  /* float16 inputs/outputs, float32 accumulation (d = 128)    */
} fa_dtype;

/*
 * Forward pass.  "Building Flash Attention from Scratch in Pure NumPy",
 * architecture overview and Steps 2-3; masks from "Build a FlashAttention-2
 * Inference Kernel from Scratch in Pure Python", Step 3.
 *
 *   q, k, v : [B][H][N][d] inputs (dtype), 16-byte aligned.
 *   o       : [B][H][N][d] output (dtype), 16-byte aligned.
 *   lse     : [B][H][N] float32 output (natural-log logsumexp per row); may
 *             be NULL when the caller does not need it.
 *   B, H, N : >= 1.  d: 128 for FA_BF16 and FA_FP16; 64 or 128 for FA_FP32.
 *   causal  : 0 or 1.  window: 0 = none, else > 0 (see Mask above).
 * Key tiles that the mask hides completely are skipped, never computed.
 * FA_BF16 and FA_FP16 run on the tensor cores (tcgen05 kind::f16 with both
 * operands of the inputs' type, TMA, TMEM; P is formed in that type); FA_FP32 on CUDA
 * cores in float32.
 */
FA_API fa_status fa_forward(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int N, int d, float scale, int causal, int window,
                     fa_dtype dtype, void* stream);

/*
 * One key shard's forward, for context-parallel attention: queries against a
 * contiguous run of keys that starts `q_offset` positions before query row 0.
 * Both pure-Python kernel pages' "Extending It" roadmaps (the attention matrix
 * split across devices; each worker holds part of the key/value space).
 *
 *   q, o    : [B][H][Nq][d]; k, v: [B][H][Nk][d] (FA_BF16 or FA_FP16,
 *             d = 128), 16-byte aligned.  lse: [B][H][Nq] float32 or NULL.
 *   q_offset: query row i sits at position i + q_offset of the key sequence,
 *             so the mask is (causal == 0 || j <= i + q_offset) &&
 *             (window <= 0 || j > i + q_offset - window), j in [0, Nk).  0
 *             with Nq == Nk is fa_forward.  |q_offset|, Nq, Nk and window must
 *             not exceed 2^29 (FA_ERR_INVALID otherwise).
 * O and lse are the softmax over this shard's keys only; a row that sees none
 * of them gets O = 0 and lse = -inf (query tiles with no visible key run no
 * MMA at all).  fa_merge combines the shards' results into the full
 * attention.
 */
FA_API fa_status fa_forward_offset(const void* q, const void* k, const void* v, void* o, float* lse,
                                   int B, int H, int Nq, int Nk, int q_offset, int d, float scale,
                                   int causal, int window, fa_dtype dtype, void* stream);

/*
 * Merge of S partial results over disjoint key sets.  "Building Flash
 * Attention from Scratch in Pure NumPy", architecture overview (the merge
 * identity for two partial softmaxes, restated for S parts):
 *     lse = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
 *
 *   o_parts   : [S][B][H][N][d] normalised partial outputs in `dtype`:
 *               FA_BF16, FA_FP16, or FA_FP32 (float32 partials, for callers
 *               that keep their partials unrounded); d = 64 or 128;
 *               16-byte aligned.
 *   lse_parts : [S][B][H][N] float32; -inf marks a part with no visible key
 *               for that row (its O is not read).
 *   o         : [B][H][N][d] output in `dtype`; lse: [B][H][N] float32
 *               output or NULL.
 *   S         : 1 .. 65536.
 * A row whose parts are all empty gets O = 0 and lse = -inf; a NaN lse in any
 * part makes the row NaN.
 */
FA_API fa_status fa_merge(const void* o_parts, const float* lse_parts, int S, void* o, float* lse,
                          int B, int H, int N, int d, fa_dtype dtype, void* stream);

/*
 * Bytes of device workspace fa_decode needs for these sizes (a multiple of
 * 256; 0 for invalid sizes).  The workspace holds one partial (o, lse) per
 * key chunk of each (b, h) between the split and combine kernels.
 */
FA_API size_t fa_decode_workspace_size(int B, int H, int cap, int d);

/*
 * Single-token decode against a padded key/value cache.  "Build a
 * FlashAttention Kernel with Online Softmax and KV Cache in Pure Python",
 * Step 4: the cache already holds the current token, so query (b, h) attends
 * to every cached position j < seqlens[b].  The keys are split into chunks
 * scored in parallel; the chunk results are merged with the two-softmax merge
 * identity from "Building Flash Attention from Scratch in Pure NumPy"
 * (architecture overview): lse = ln sum_s exp(lse_s), O = sum_s
 * exp(lse_s - lse) O_s.
 *
 *   q        : [B][H][d] (dtype FA_BF16 or FA_FP16, d = 128), 16-byte aligned.
 *   kcache,
 *   vcache   : [B][H][cap][d], 16-byte aligned.  Rows at j >= seqlens[b]
 *              are never read.
 *   seqlens  : [B] int32 DEVICE array.  Values are clamped to [0, cap]; a
 *              length of 0 gives o = 0, lse = -inf.
 *   o        : [B][H][d] output (dtype).  lse: [B][H] float32 or NULL.
 *   workspace: >= fa_decode_workspace_size(B, H, cap, d) bytes, 256-byte
 *              aligned, contents ignored on entry.
 */
FA_API fa_status fa_decode(const void* q, const void* kcache, const void* vcache,
                    const int32_t* seqlens, void* o, float* lse,
                    int B, int H, int cap, int d, float scale, fa_dtype dtype,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode against a paged cache.  "Build a FlashAttention-2 Inference Kernel
 * from Scratch in Pure Python", Extending It (paged KV-cache integration),
 * read as the usual block pool: the cached rows of all sequences live in
 * fixed-size blocks of one shared pool, and a per-sequence block table maps
 * logical block t (keys [t * block_size, (t + 1) * block_size)) to a physical
 * block.  Attention itself is exactly fa_decode's: query (b, h) attends to the
 * keys j < seqlens[b] of its sequence.
 *
 *   q           : [B][H][d] (dtype FA_BF16 or FA_FP16, d = 128), 16-byte aligned.
 *   kpool,
 *   vpool       : [num_blocks][H][block_size][d], 16-byte aligned; key j of
 *                 sequence b, head h is row (j mod block_size) of block
 *                 block_table[b][j / block_size], head h.
 *   block_table : [B][max_blocks] int32 DEVICE array.  Entries of blocks that
 *                 hold keys j < seqlens[b] must lie in [0, num_blocks); the
 *                 kernel checks each one it uses, skips an out-of-range block
 *                 (never reads it) and records FA_ERR_INVALID for
 *                 fa_get_device_status.  Other entries are never read.
 *   seqlens     : [B] int32 DEVICE array, clamped to [0, max_blocks * block_size].
 *   block_size  : a power of two in [1, 4096].
 *   o, lse      : as fa_decode.
 *   workspace   : >= fa_decode_workspace_size(B, H, max_blocks * block_size, d)
 *                 bytes, 256-byte aligned, contents ignored on entry.
 */
FA_API fa_status fa_decode_paged(const void* q, const void* kpool, const void* vpool,
                          const int32_t* block_table, const int32_t* seqlens, void* o,
                          float* lse, int B, int H, int num_blocks, int block_size,
                          int max_blocks, int d, float scale, fa_dtype dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode for callers that cannot allocate device memory.  The paper has no
 * counterpart: this exists for deployment, not for the method.  Same arguments,
 * layout and results as fa_decode, minus the workspace: the per-chunk
 * partials go to a fixed array of FA_DECODE_NOALLOC_SCRATCH_BYTES compiled into
 * the library.  Serving runtimes that forbid allocation after start-up and
 * plugin interfaces that pass a kernel only its inputs and outputs are the
 * intended users.
 *   - Size limit: fa_decode_workspace_size(B, H, cap, d) must not exceed
 *     FA_DECODE_NOALLOC_SCRATCH_BYTES (for cap = 8192 that is B*H <= 1016);
 *     larger calls return FA_ERR_INVALID with nothing launched.
 *   - With lazy module loading (the CUDA 12 default) the array is reserved on
 *     a device by the first call made there (at library load instead when
 *     CUDA_MODULE_LOADING=EAGER) and held until the process exits.  That first
 *     call can fail with FA_ERR_CUDA when the device has no memory left, so
 *     make it at start-up, as a warm-up, and before any stream capture.
 *   - Every call looks the array's address up in the current context (the
 *     address is per context: a device reset or another context moves it);
 *     once loaded, the lookup does not synchronise.
 *   - All calls share the array: calls whose kernels overlap on the GPU race.
 *     Nothing needs clearing between calls.
 *   - Calls no cudaMalloc/cudaFree and no allocating library routine.
 */
#define FA_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20)
FA_API fa_status fa_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                   const int32_t* seqlens, void* o, float* lse,
                                   int B, int H, int cap, int d, float scale, fa_dtype dtype,
                                   void* stream);

/*
 * Bytes of device workspace fa_backward needs (a multiple of 256): the
 * float32 row terms D = rowsum(dO * O) and a float32 dQ accumulator.
 */
FA_API size_t fa_backward_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass.  "Building Flash Attention from Scratch in Pure NumPy",
 * Step 4: D = rowsum(dO * O); per key tile, P is recomputed from the saved
 * row statistic (here the single logsumexp lse written by fa_forward) and
 *     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
 *     dQ = scale * dS K,  dK = scale * dS^T Q
 * (that page's own dK/dQ lines are declared simplified; these are the exact
 * gradients of the forward).
 *
 *   q, k, v, o, dout : [B][H][N][d] (dtype FA_BF16 or FA_FP16, d = 128), 16-byte aligned.
 *   lse              : [B][H][N] float32 from fa_forward with the same
 *                      arguments.
 *   dq, dk, dv       : [B][H][N][d] outputs (dtype).
 *   workspace        : >= fa_backward_workspace_size(B, H, N, d) bytes,
 *                      256-byte aligned, contents ignored on entry.
 */
FA_API fa_status fa_backward(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      int B, int H, int N, int d, float scale, int causal, int window,
                      fa_dtype dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, then returns FA_ERR_TIMEOUT if any kernel of this
 * library recorded a barrier timeout since the last call, FA_ERR_INVALID if
 * a paged decode met a block id outside its pool (either record is cleared),
 * FA_ERR_CUDA if the stream reports an error, else FA_OK.
 */
FA_API fa_status fa_get_device_status(void* stream);

/*
 * Failure-path self-test: launches one CTA whose only thread block waits on
 * an internal barrier that nothing ever completes, with a bound of
 * `limit_cycles` SM clock cycles (1 .. 4e9).  The wait gives up, the kernel
 * records FA_ERR_TIMEOUT and returns normally, exactly as every production
 * kernel does when a barrier stalls; the next fa_get_device_status() on
 * `stream` reports it and clears it.  The CUDA context stays usable.
 */
FA_API fa_status fa_selftest_wait_timeout(long long limit_cycles, void* stream);

/*
 * Self-test of the exponential used inside the forward softmax: writes
 * y[i] = exp2_poly(x[i]) for i < n, where exp2_poly is the device function
 * that computes part of "Building Flash Attention from Scratch in Pure NumPy",
 * Step 2's P = exp(S - m_new) (in base 2) on the FMA pipe: a Cody-Waite
 * split x = j + f, j = round(x), and a cubic in f fitted for minimum relative
 * error.  Stated behaviour: relative error <= 7.5e-5 for -125.5 <= x <= 0;
 * a result below 2^-125 for x < -125.5 (inputs are clamped at -126.5).
 *   x, y : DEVICE float32 arrays of n elements (n >= 1), 4-byte aligned.
 * Returns FA_ERR_INVALID for a null or misaligned pointer or n < 1.
 */
FA_API fa_status fa_selftest_exp2_poly(const float* x, float* y, long long n, void* stream);

/* Static, human-readable name of a status code. */
FA_API const char* fa_status_string(fa_status status);

/* Library ABI version (major * 100 + minor). */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TILED_EXACT_ATTENTION_FA_H_ */
