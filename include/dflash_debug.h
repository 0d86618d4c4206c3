/*
 * dflash_debug.h - test hooks into the library's GEMM core.
 *
 * These expose the tcgen05 weight-streaming GEMM on its own so that tests can
 * compare it with a plain matrix product.  Not part of the hot-path API in
 * dflash.h; same conventions (device pointers, void* stream, status codes).
 */
#ifndef DFLASH_DEBUG_H
#define DFLASH_DEBUG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* out[s][m][n] = sum over split s's K range of X[m][k] * W[n][k].
 * W: device [N, K]; X: device [M, K]; both of element type elem (DFLASH_BF16 or
 * DFLASH_F16); K % 64 == 0; 16-byte aligned.  out: device fp32
 * [splits][M][N].  The split count is clamped to [1, K/64] and rounded so that
 * every split but the last has the same number of 64-wide K blocks; the count
 * used is written to *splits_used.  err_ws: a zero-filled 256-byte device
 * block that receives device error bits. */
int dflash_debug_gemm(const void* W, int N, int K, const void* X, int M, int elem, int splits,
                      float* out, int* splits_used, void* err_ws, void* stream);

/* Same product with the weights read from their pre-tiled streaming image
 * (written by dflash_debug_tile_weights) instead of a tensor map over W. */
int dflash_debug_gemm_tiled(const void* W_tiled, int N, int K, const void* X, int M, int elem,
                            int splits, float* out, int* splits_used, void* err_ws, void* stream);

/* Bytes of the pre-tiled streaming image of a [N, K] 16-bit weight, and the
 * call that writes it (128-row x 64-column tiles, each the 128-byte-swizzled
 * shared-memory image of the tile, rows past N zero). */
size_t dflash_debug_tiled_bytes(int N, int K);
int dflash_debug_tile_weights(const void* W, void* W_tiled, int N, int K, void* stream);

/* LM-head epilogue: for every token row m and 128-row weight tile t,
 * stats[m][t] = {max_n logit, argmax n (lowest), sum exp(logit - max), 0}
 * (16 bytes per entry); logits (device fp32 [M, N]) receives the raw products
 * when not NULL. */
int dflash_debug_lmhead(const void* W, int N, int K, const void* X, int M, int elem, void* stats,
                        float* logits, void* err_ws, void* stream);

/* Same as dflash_debug_lmhead with the weights read from their pre-tiled
 * image (the layout the model's LM head uses). */
int dflash_debug_lmhead_tiled(const void* W_tiled, int N, int K, const void* X, int M, int elem,
                              void* stats, float* logits, void* err_ws, void* stream);

/* How the tiled GEMMs are launched from now on, process-wide: 0 = the
 * library's rule, 1 = one CTA per 128-row weight tile, 2 = CTA pairs (cluster
 * of two CTAs on one TPC sharing a 256-row weight tile, M = 256 tcgen05.mma
 * with cta_group::2).  Non-tiled weights always use single CTAs.  Returns
 * DFLASH_EINVAL for any other value.  Not thread-safe; tests only. */
int dflash_debug_gemm_mode(int mode);

/* Y = X W^T through the stream-K schedule of the tcgen05 GEMM, stored as fp32
 * out [M, N] (the fused-store epilogue after the in-kernel fixup of split
 * tiles).  Wt is the pre-tiled image (dflash_debug_tile_weights), X [M, K] of
 * the same 16-bit type; ws a zero-filled, 256-byte aligned workspace of at least
 * dflash_debug_gemm_streamk_ws_bytes(M) bytes (its header holds the error word
 * and the tile counters).  The launch mode (single CTAs or CTA pairs) follows
 * dflash_debug_gemm_mode. */
size_t dflash_debug_gemm_streamk_ws_bytes(int M);
int dflash_debug_gemm_streamk(const void* Wt, int N, int K, const void* X, int M, int elem,
                              float* out, void* ws, size_t ws_bytes, void* stream);

/* Schedule of the draft and injection GEMMs for every later call,
 * process-wide.  Stream-K: every CTA (or CTA pair) streams the same number of
 * k-blocks; a tile split between workers is finished inside the GEMM by its
 * last piece, which then applies the following elementwise step in its
 * epilogue.  Fixed splits: K split a fixed number of ways, the partials summed
 * by separate reduction kernels.  0 (default): stream-K for the LM head,
 * fixed splits for the projections and the injection; 1: fixed splits
 * everywhere; 2: stream-K everywhere.  All compute the same products (up to
 * fp32 summation order).  DFLASH_EINVAL for any other value.  Not
 * thread-safe; tests and tuning only. */
int dflash_debug_gemm_schedule(int sched);

/* Failure-detection check: launches one thread that waits, with the
 * library's bounded pipeline wait, on an mbarrier phase nothing completes.
 * After the wait limit (1 s) the kernel sets DFLASH_DEV_TIMEOUT in the error
 * word of err_ws (a 256-byte aligned workspace) and returns; the context stays
 * usable.  No fault and no trap. */
int dflash_debug_wait_timeout(void* err_ws, void* stream);

/* The K split count the draft and injection paths pick for an M x N x K
 * weight-streaming GEMM (before any workspace limit), or DFLASH_EINVAL. */
int dflash_debug_pick_splits(int M, int N, int K);

/* Weight w of the split partials' traffic in the K-split picker of the draft
 * and injection GEMMs, process-wide (default 4): a split count s scores
 * balance / (1 + w * s * M / K).  Returns DFLASH_EINVAL outside [0, 64].  Not
 * thread-safe; tests and tuning only. */
int dflash_debug_split_weight(float w);

/* Schedule of the draft attention (bf16 models) for every later call,
 * process-wide: 0 (default) the split-KV grid on the mma.sync kernel, its key
 * chunk planned on the device per forward (or forced by dflash_debug_attn_chunk); 1 persistent (mma.sync),
 * two CTAs per SM each streaming the same number of 64-key tiles over the
 * (request, kv head) segments, segments split between CTAs merged by their
 * last piece; 2 the split-KV grid on the tcgen05 kernel where its shapes allow
 * (head dim 128, at most 32 query rows per kv head, contiguous K/V; the
 * mma.sync kernel elsewhere).  All give the same result up to fp32 summation
 * order and the rounding of the probabilities to fp16.  DFLASH_EINVAL for any
 * other value.  Not thread-safe; tests and tuning only. */
int dflash_debug_attn_schedule(int sched);

/* The split-KV planner of the draft attention, run on its own.  For the device
 * arrays ctx_len and req_valid (batch entries; ctx_len + B <= cap wherever
 * req_valid is set) it writes to the device array plan_out (8-byte aligned,
 * plan_cap ints, at least 4 + 2 * batch * n_kv * ceil(cap / chunk_min)) what a
 * forward with block size B, n_kv kv heads, grid chunk chunk_min (a positive
 * multiple of 64) and `slots` resident CTAs would use: {chunk, n_items, -, -},
 * the chunk in keys (a multiple of 64, at least chunk_min), then one pair per
 * (request, kv head, chunk) with keys, {request << 16 | kv head << 8 | chunk
 * index, the request's context length or 0 where req_valid is 0},
 * request-major.  Enqueued on `stream`; DFLASH_EINVAL for null pointers,
 * non-positive sizes, more than 255 kv heads or chunks, a bad chunk_min or a
 * short or misaligned plan_out.  dflash_debug_attn_slots returns the resident CTAs of the
 * grid kernel the draft would run for head_dim and `rows` query rows per kv
 * head (contiguous K/V), or DFLASH_EINVAL.  Tests only. */
int dflash_debug_attn_plan(const int32_t* ctx_len, const int32_t* req_valid, int batch, int B,
                           int n_kv, int cap, int chunk_min, int slots, int32_t* plan_out,
                           long long plan_cap, void* stream);
int dflash_debug_attn_slots(int head_dim, int rows, int B);

/* Split-KV chunk of the draft attention, in keys, for every later
 * dflash_draft_block call, process-wide: 0 = the library's rule (bf16 models
 * on the default schedule: a planning kernel picks each forward's chunk from
 * the actual context lengths, at least the grid chunk of at most 64 chunks per
 * request), else a multiple of 64 that is used, unplanned, whenever it gives
 * at most 64 chunks.  Returns DFLASH_EINVAL for a negative
 * value or one that is not a multiple of 64.  Not thread-safe; tests only. */
int dflash_debug_attn_chunk(int keys);

/* The per-entry sampling arithmetic of the draw kernels, element by element,
 * for accuracy tests.  For i < n: g2[i] = the Gumbel variate of Philox output
 * word w[i] in log2 units, -log2(-ln U') with U' = ((w[i] >> 11) + 1/2) 2^-53;
 * l2[i] = log2(1 - 2^d[i]) for d[i] < 0 (the log2 residual weight of a draw
 * from max(0, p - q) relative to p, with d = log2 q - log2 p).  w, d, g2, l2
 * are device arrays of n entries; the call is asynchronous on `stream`.
 * DFLASH_EINVAL for n < 0 or a null array when n > 0. */
int dflash_debug_sample_math(const uint64_t* w, const float* d, int n, float* g2, float* l2,
                             void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DFLASH_DEBUG_H */
