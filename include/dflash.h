/*
 * dflash.h - C ABI of the DFlash block-diffusion speculative-decoding hot path
 * for NVIDIA B200 (sm_100a).
 *
 * The three hot calls follow the problem statement of the DFlash pages:
 *
 *   dflash_inject_kv    "DFlash: Block Diffusion for Flash Speculative Decoding",
 *                       §1 上下文特征提取 and §2 KV 注入; "DFlash + Spec V2 深度解析",
 *                       §2.2 KV 注入: hidden states of tapped target layers are
 *                       fused into context features and written into every draft
 *                       layer's K/V cache (§Immediate Materialization: one
 *                       layer-batched projection).
 *   dflash_draft_block  "DFlash + Spec V2 深度解析", §2.3 块扩散: a block of
 *                       [anchor, MASK, ..., MASK] is predicted in one forward per
 *                       denoising step, most confident positions first.
 *                       Blog "DFlash：用“块扩散”魔法", §核心创新:
 *                       generate_block(context, block_size).
 *   dflash_verify       Blog "DFlash：用“块扩散”魔法", §2 Flash Verification:
 *                       decide_acceptance(logits, draft_block), read greedily.
 *   dflash_verify_sampled  the same step under temperature sampling
 *                       (speculative sampling; see its declaration).
 *   dflash_draft_block_sampled  drafting under temperature sampling.
 *   dflash_inject_kv_paged, dflash_draft_block_paged  the same calls over a
 *                       paged K/V store with prefix sharing.
 *   dflash_draft_begin .. dflash_draft_end, dflash_verify_shard/_merge
 *                       drafting and verify with the vocabulary split over GPUs.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers marked "device" are CUDA device pointers in the caller's current
 *   device; "host" pointers are read during the call only.  Every device buffer
 *   is owned by the caller, except the model's prepacked weight copies, which
 *   dflash_model_create allocates and dflash_model_destroy frees.  The hot calls
 *   (inject, draft, verify) allocate nothing.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   The hot calls only enqueue work on it: none synchronises with the host.
 * - Matrices are row-major.  Weight matrices are [out_features, in_features].
 * - Return value: DFLASH_OK (0) or a negative DFLASH_E* code.  Host-side
 *   argument checks happen before anything is enqueued; a failing call leaves
 *   every buffer untouched.
 * - Errors that only the device can see (a context too long for the cache, an
 *   output buffer that would overflow, a token id outside [0, V), an expired
 *   bounded wait) set bits in a sticky device error word inside the workspace;
 *   the affected request writes nothing and the kernel never traps.
 *   dflash_get_error reads and clears that word.
 * - Workspace: a caller-allocated device buffer of at least the size the
 *   matching *_workspace_size call returns, 256-byte aligned, zero-filled once
 *   (dflash_workspace_init) before its first use.  Calls leave its counters at
 *   zero.  Two calls that share a workspace must not overlap on the GPU.
 */
#ifndef DFLASH_H
#define DFLASH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define DFLASH_OK            0
#define DFLASH_EINVAL       -1  /* null/misaligned pointer, bad size or shape */
#define DFLASH_EUNSUPPORTED -2  /* dtype or shape the library was not built for */
#define DFLASH_ECUDA        -3  /* a CUDA call or kernel launch failed */
#define DFLASH_ENOMEM       -4  /* model creation could not allocate device memory */
#define DFLASH_EWORKSPACE   -5  /* workspace smaller than the size query returned */
#define DFLASH_ESCRATCH     -6  /* request larger than dflash_verify_noalloc's fixed scratch */

/* ---- device error word bits (dflash_get_error) ------------------------ */
#define DFLASH_DEV_CTX_CAP     1  /* position outside the K/V cache capacity */
#define DFLASH_DEV_OUT_CAP     2  /* verify output would pass out_cap */
#define DFLASH_DEV_TOKEN_RANGE 4  /* token id outside [0, V) */
#define DFLASH_DEV_TIMEOUT     8  /* a bounded device wait expired */
#define DFLASH_DEV_ROWS        16 /* cu_rows not monotone or not ending at n_rows */
#define DFLASH_DEV_PAGE        32 /* a position's page-table entry is unmapped (paged K/V) */
#define DFLASH_DEV_RANGE       64 /* an fp16 activation or cache entry overflowed (bf16 models) */
#define DFLASH_DEV_CHECK      128 /* bounds-checked build only: an index failed its check */

/* ---- element types ---------------------------------------------------- */
#define DFLASH_F32  0
#define DFLASH_BF16 1
#define DFLASH_F16  2  /* operand type of the test hooks in dflash_debug.h only */

typedef struct dflash_model dflash_model; /* opaque */

/* Element types inside a model.  DFLASH_F32 models compute and store in fp32.
 * DFLASH_BF16 models take bf16 weights and bf16 tapped hidden states; the
 * library keeps its GEMM weight copies and GEMM activations in fp16 (every
 * bf16 weight in fp16's normal range converts exactly) and multiplies
 * fp16 x fp16 -> fp32 on the tensor cores, and the K/V cache holds fp16.
 * Same bytes as bf16, three more mantissa bits.
 *
 * Draft model shape.  Constraints: n_q % n_kv == 0; head_dim even and <= 256.
 * For DFLASH_BF16: d, H_t, inter, n_q*head_dim multiples of 64, head_dim 64 or
 * 128.  For DFLASH_F32 (SIMT path, for small correctness models) no further
 * constraint.  vocab >= 2; mask_id in [0, vocab). */
typedef struct {
  int32_t dtype;     /* DFLASH_F32 or DFLASH_BF16: type of the weights and tapped states */
  int32_t H_t;       /* target hidden size of one tapped layer */
  int32_t n_tap;     /* tapped target layers (1..8) */
  int32_t n_layers;  /* draft layers L */
  int32_t d;         /* draft hidden size */
  int32_t n_q;       /* query heads */
  int32_t n_kv;      /* key/value heads */
  int32_t head_dim;  /* per-head size */
  int32_t inter;     /* SwiGLU intermediate size */
  int32_t vocab;     /* V */
  int32_t mask_id;   /* the [MASK] token id */
  int32_t max_pos;   /* positions 0..max_pos-1 get a RoPE table entry */
  float eps;         /* RMSNorm epsilon */
  double rope_base;  /* RoPE base; angle of pair i at position p = p*base^(-2i/head_dim) */
} dflash_config;

/* One draft layer, device pointers in the config's dtype, borrowed during
 * dflash_model_create only. */
typedef struct {
  const void* g_in;   /* [d]              input RMSNorm gain */
  const void* Wq;     /* [n_q*hd, d] */
  const void* Wk;     /* [n_kv*hd, d]     also projects the injected context */
  const void* Wv;     /* [n_kv*hd, d]     also projects the injected context */
  const void* Wo;     /* [d, n_q*hd] */
  const void* g_post; /* [d]              post-attention RMSNorm gain */
  const void* Wg;     /* [inter, d]       SwiGLU gate */
  const void* Wu;     /* [inter, d]       SwiGLU up */
  const void* Wd;     /* [d, inter]       SwiGLU down */
} dflash_layer_weights;

typedef struct {
  const void* emb;      /* [V, d]           token embedding */
  const void* W_fc;     /* [d, n_tap*H_t]   context-feature fc (taps concatenated in order) */
  const void* g_ctx;    /* [d]              context-feature RMSNorm gain */
  const void* g_final;  /* [d]              final RMSNorm gain */
  const void* W_lm;     /* [V, d]           LM head */
  const dflash_layer_weights* layers; /* host array of n_layers entries */
} dflash_weights;

/* Creates a model on the current device: checks the shape, prepacks the
 * weights into library-owned device buffers (layer-batched [Wk;Wv] of every
 * layer for injection, [Wq;Wk;Wv] and [Wg;Wu] per layer) and builds the RoPE
 * cos/sin table in fp64 (stored fp32).  Synchronises the device once.
 * Returns DFLASH_EINVAL / DFLASH_EUNSUPPORTED / DFLASH_ENOMEM / DFLASH_ECUDA. */
int dflash_model_create(const dflash_config* cfg, const dflash_weights* w, dflash_model** out);

/* Frees the model's device buffers (synchronises the device).  NULL is a no-op. */
int dflash_model_destroy(dflash_model* m);

/* Bytes of workspace that inject (up to max_inject_rows rows), draft (up to
 * max_batch requests of block size B) and verify (max_batch x B rows) need. */
size_t dflash_workspace_size(const dflash_model* m, int max_batch, int B, int max_inject_rows);

/* Bytes of workspace that dflash_verify needs without a model. */
size_t dflash_verify_workspace_size(int batch, int B, int V);

/* Zero-fills a workspace (asynchronous on `stream`). */
int dflash_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * KV injection.
 *   taps[t]    host array of n_tap device pointers; taps[t] is [n_rows, H_t]
 *              (hidden states of tapped layer t, ascending tap order), 16-byte aligned.
 *   cu_rows    device int32 [batch+1]: rows cu_rows[r]..cu_rows[r+1]-1 belong to
 *              request r; cu_rows[0] = 0, cu_rows[batch] = n_rows.
 *   start_pos  device int32 [batch]: absolute position of request r's first row.
 *   k_cache, v_cache  device [n_layers][batch][n_kv][cache_cap][head_dim] of the
 *              model's cache type (fp16 for DFLASH_BF16 models, fp32 for
 *              DFLASH_F32), 16-byte aligned; K is stored after RoPE.
 * Computes c = RMSNorm(concat_t(taps[t]) W_fc^T; g_ctx) and, for every layer l,
 * K_l[p] = RoPE(c Wk_l^T, p), V_l[p] = c Wv_l^T at p = start_pos[r] + i.
 * Rows whose position falls outside [0, cache_cap) are skipped and set
 * DFLASH_DEV_CTX_CAP.  n_rows == 0 is a no-op.
 */
int dflash_inject_kv(const dflash_model* m, const void* const* taps, const int32_t* cu_rows,
                     const int32_t* start_pos, int batch, int n_rows, void* k_cache, void* v_cache,
                     int cache_cap, void* ws, size_t ws_bytes, void* stream);

/*
 * Masked-block draft forward with n_steps denoising steps.
 *   anchor     device int32 [batch]: token at block position 0 (position ctx_len[r]).
 *   k_cache, v_cache  the caches dflash_inject_kv fills (same layout and type).
 *   ctx_len    device int32 [batch]: injected context length T_r; the block sits at
 *              positions T_r..T_r+B-1 and attends to cache positions 0..T_r-1 plus
 *              the whole block (no mask inside the block).
 *   draft_tokens  device int32 [batch, B] out: anchor then the B-1 drafted tokens.
 *   commit_step   device int32 [batch, B] out or NULL: denoising step at which each
 *              position was committed (-1 at position 0).
 *   logits_dbg    device fp32 [n_steps, batch, B, V] out or NULL: the LM-head logits
 *              of every still-masked position at each step (other rows untouched).
 * Step t commits the ceil(remaining / (n_steps - t)) masked positions with the
 * highest softmax max-probability (ties to the lower position) to their argmax
 * token (ties to the lower token id).  B in [2, 16], n_steps in [1, B-1].
 * A request with ctx_len + B > cache_cap or an anchor outside [0, V) sets a
 * device error bit and writes nothing.
 * The same inputs give the same bits on every call.  The attention splits each
 * request's context into chunks sized from the whole batch's context lengths
 * (planned on the device for bf16 models), so a request's logits can change at
 * fp32 rounding level, and a near-tie token can flip, when the other requests
 * of its batch change.
 */
int dflash_draft_block(const dflash_model* m, const int32_t* anchor, const int32_t* ctx_len,
                       const void* k_cache, const void* v_cache, int cache_cap, int batch, int B,
                       int n_steps, int32_t* draft_tokens, int32_t* commit_step, float* logits_dbg,
                       void* ws, size_t ws_bytes, void* stream);

/*
 * Paged K/V with prefix sharing.  "DFlash: Block Diffusion for Flash Speculative
 * Decoding", §2 KV 注入: the injected K/V is cached for reuse and supports prefix
 * sharing.  An injected row depends only on the target hidden state at its
 * position and on the position, so requests whose contexts share a prefix can
 * share the pages that hold it.  The pages give no layout; this one is:
 *   k_pool, v_pool  device fp16 [n_layers][n_pages][n_kv][page_size][head_dim]
 *                   (DFLASH_BF16 models only), 16-byte aligned; K after RoPE.
 *   page_table      device int32 [batch][max_pages]: position p of request r is
 *                   at page page_table[r][p / page_size], slot p % page_size.
 *                   An entry of -1, or any id outside [0, n_pages), is unmapped.
 *   page_size       a multiple of 64 (no 64-key attention tile crosses a page).
 * Requests may map the same page; the caller makes sure that no two requests of
 * one injection call write the same (page, slot).
 * dflash_inject_kv_paged: as dflash_inject_kv, writing through the table.  A
 * request whose rows touch an unmapped page writes none of its rows and sets
 * DFLASH_DEV_PAGE; rows past page_size * max_pages set DFLASH_DEV_CTX_CAP.
 * dflash_draft_block_paged: as dflash_draft_block, reading the context through
 * the table.  A request with an unmapped page below ctx_len, or with
 * ctx_len > page_size * max_pages, writes nothing and sets DFLASH_DEV_PAGE or
 * DFLASH_DEV_CTX_CAP.  Workspaces: dflash_workspace_size with the call's batch.
 * L * n_pages * n_kv * page_size must stay below 2^31 (DFLASH_EUNSUPPORTED).
 */
int dflash_inject_kv_paged(const dflash_model* m, const void* const* taps, const int32_t* cu_rows,
                           const int32_t* start_pos, int batch, int n_rows, void* k_pool,
                           void* v_pool, int n_pages, int page_size, const int32_t* page_table,
                           int max_pages, void* ws, size_t ws_bytes, void* stream);
int dflash_draft_block_paged(const dflash_model* m, const int32_t* anchor, const int32_t* ctx_len,
                             const void* k_pool, const void* v_pool, int n_pages, int page_size,
                             const int32_t* page_table, int max_pages, int batch, int B,
                             int n_steps, int32_t* draft_tokens, int32_t* commit_step,
                             float* logits_dbg, void* ws, size_t ws_bytes, void* stream);

/*
 * Sampled (temperature) drafting.  "DFlash + Spec V2 深度解析", §2.3 块扩散 gives
 * the greedy steps; "DFlash: Block Diffusion for Flash Speculative Decoding",
 * §消融实验结论, says drafting holds up under high-temperature sampling; the
 * pages give no sampling rule.  The rule taken is the sampled counterpart of
 * the greedy one.  At step t every still-masked position j of request r draws
 *   x_j = argmax_v (Y_jv / temperature - log(-log U'_v))   (ties to the lower id)
 * from its LM-head logits Y_j, with U'_v = ((w >> 11) + 1/2) 2^-53 and w the
 * 64-bit word n % 4 of Philox4x64-10 (Salmon et al., SC 2011) under key
 * (seed, 0) at counter (offset, r, 2, n / 4), n = (t B + j) V + v.  Its
 * confidence is the untempered probability softmax(Y_j)(x_j).  The
 * ceil(remaining / (n_steps - t)) most confident positions (ties to the lower
 * position) commit their drawn tokens.
 *   draft_logits  device [batch, B, V] out, of draft_logits_dtype (DFLASH_F32 or
 *                 DFLASH_BF16), 16-byte aligned: row j holds the logits of the step
 *                 that committed position j, the draft distribution q_j that
 *                 dflash_verify_sampled takes (row 0 is not written).  The draw
 *                 reads the stored row, so each token is drawn from exactly the
 *                 row the caller receives.
 *   temperature   in [1e-4, 1e4]; equal (seed, offset) repeat the call's draws.
 * Other arguments, errors and limits as dflash_draft_block; batch * B <= 32768
 * (DFLASH_EUNSUPPORTED beyond).  A request that sets a device error bit writes
 * none of its draft_tokens, commit_step or draft_logits.
 */
int dflash_draft_block_sampled(const dflash_model* m, const int32_t* anchor,
                               const int32_t* ctx_len, const void* k_cache, const void* v_cache,
                               int cache_cap, int batch, int B, int n_steps, float temperature,
                               uint64_t seed, uint64_t offset, int32_t* draft_tokens,
                               int32_t* commit_step, void* draft_logits, int draft_logits_dtype,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * Vocabulary-parallel LM head and verify across GPUs ("DFlash + Spec V2 深度解析",
 * §3.3: the engine serves the target with tensor parallelism, --tp-size 8).
 * Each of `world` ranks holds a contiguous shard [vocab_lo, vocab_hi) of the
 * vocabulary, shards in rank order covering [0, V).  Per row, a shard reduces
 * its part of the vocabulary to one 16-byte record; the ranks all-gather the
 * records (the only exchange: 16 bytes per row per rank, e.g. an NCCL
 * all-gather on the same stream) and every rank merges them, shards in order,
 * to the same argmax (lowest global id on ties) and confidence.
 */
typedef struct {
  float max;     /* largest logit of the row in the shard */
  int32_t id;    /* its global vocabulary id (lowest on ties) */
  float sumexp;  /* sum over the shard of exp(logit - max) */
  float pad;
} dflash_lm_stat;

typedef struct {
  float value;   /* largest target logit of the row in the shard */
  int32_t id;    /* its global vocabulary id (lowest on ties) */
} dflash_row_argmax;

/* A model whose LM head holds only rows [vocab_lo, vocab_hi) of W_lm (w->W_lm
 * still points at the whole [V, d] matrix; only the shard is copied).  Every
 * other weight is whole.  DFLASH_BF16 models only.  Such a model drafts only
 * through the step calls below (the one-call drafts return DFLASH_EUNSUPPORTED). */
int dflash_model_create_shard(const dflash_config* cfg, const dflash_weights* w, int vocab_lo,
                              int vocab_hi, dflash_model** out);

/* Masked rows of every request at denoising step `step` (the rows of that
 * step's records: request-major, positions ascending), or DFLASH_EINVAL. */
int dflash_draft_rows(int batch, int B, int n_steps, int step);

/* A greedy draft in steps, on every rank with the same inputs:
 *   dflash_draft_begin          block initialisation and request checks;
 *   for step = 0 .. n_steps-1:
 *     dflash_draft_forward_shard  the step's forward; writes this shard's record
 *                                 of every masked row to shard_stats (device,
 *                                 dflash_draft_rows(...) records, 16-byte aligned);
 *     (the caller all-gathers the records of every rank into `gathered`,
 *      [world][rows] records, rank-major)
 *     dflash_draft_commit_shards  merges them and commits the step;
 *   dflash_draft_end            writes draft_tokens / commit_step as
 *                               dflash_draft_block does.
 * With world = 1 and a whole-vocabulary model the result equals
 * dflash_draft_block.  Arguments and errors as dflash_draft_block; the steps of
 * one draft share the workspace and must not interleave with other calls on it. */
int dflash_draft_begin(const dflash_model* m, const int32_t* anchor, const int32_t* ctx_len,
                       int cache_cap, int batch, int B, int n_steps, void* ws, size_t ws_bytes,
                       void* stream);
int dflash_draft_forward_shard(const dflash_model* m, const int32_t* ctx_len, const void* k_cache,
                               const void* v_cache, int cache_cap, int batch, int B, int n_steps,
                               int step, void* shard_stats, void* ws, size_t ws_bytes,
                               void* stream);
int dflash_draft_commit_shards(const dflash_model* m, const void* gathered, int world, int batch,
                               int B, int n_steps, int step, void* ws, size_t ws_bytes,
                               void* stream);
int dflash_draft_end(const dflash_model* m, int batch, int B, int n_steps, int32_t* draft_tokens,
                     int32_t* commit_step, void* ws, size_t ws_bytes, void* stream);

/* Verify across vocabulary shards.  dflash_verify_shard: logits_shard is
 * [batch, B, Vs] (this rank's columns, global ids vocab_offset ..
 * vocab_offset + Vs - 1), row_argmax receives batch * B dflash_row_argmax
 * records; workspace dflash_verify_workspace_size(batch, B, Vs).
 * dflash_verify_merge: gathered holds [world][batch * B] records (rank-major,
 * 16-byte aligned); it takes g_i as the merged argmax and then does exactly
 * what dflash_verify does (same outputs and device errors; workspace: the
 * header, dflash_verify_workspace_size(0, B, V) bytes). */
int dflash_verify_shard(const void* logits_shard, int logits_dtype, int batch, int B, int Vs,
                        int vocab_offset, void* row_argmax, void* ws, size_t ws_bytes,
                        void* stream);
int dflash_verify_merge(const void* gathered, int world, const int32_t* draft_tokens, int batch,
                        int B, int V, int32_t* out_tokens, int32_t* out_len, int out_cap,
                        int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * Greedy verify.
 *   target_logits  device [batch, B, V] of logits_dtype (DFLASH_BF16 or DFLASH_F32),
 *                  16-byte aligned; row i of request r scores the token after block
 *                  position i.
 *   draft_tokens   device int32 [batch, B] (position 0 = anchor).
 *   out_tokens     device int32 [batch, out_cap]; out_len device int32 [batch] in/out.
 *   seq_lens       device int32 [batch] in/out; accept_len, next_anchor device int32
 *                  [batch] out.
 * g_i = argmax_v logits[r, i] (lowest v on ties); a = longest prefix with
 * g_i == draft[r, i+1], a <= B-1; emits draft[r, 1..a] then g_a at
 * out_tokens[r, out_len[r]...]; out_len += a+1; seq_lens += a+1;
 * accept_len = a; next_anchor = g_a.  A request whose draft holds an id outside
 * [0, V) or whose emission would pass out_cap writes nothing and sets a device
 * error bit.  B in [2, 32]; batch == 0 is a no-op.
 */
int dflash_verify(const void* target_logits, int logits_dtype, const int32_t* draft_tokens,
                  int batch, int B, int V, int32_t* out_tokens, int32_t* out_len, int out_cap,
                  int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor, void* ws,
                  size_t ws_bytes, void* stream);

/*
 * Sampled (temperature) verify.  The pages fix no acceptance rule for sampling
 * ("DFlash: Block Diffusion for Flash Speculative Decoding", §消融实验结论: drafting
 * holds up under high-temperature sampling; §与 Speculative Decoding 系列的关系:
 * the speculative-decoding line of Leviathan et al., 2023; blog "DFlash：用“块
 * 扩散”魔法", §2 Flash Verification: the target's probabilities are compared
 * with the draft's).  The rule is standard speculative sampling:
 *   p_i = softmax(target_logits[r, i] / temperature)  (token after position i),
 *   q_j = softmax(draft_logits[r, j] / temperature)   (draft at position j);
 *   for i = 0..B-2 in order d_{i+1} is accepted while
 *   log U_i < log p_i(d_{i+1}) - log q_{i+1}(d_{i+1}); at the first rejection
 *   (a = i) the last token is drawn from max(0, p_i - q_{i+1}); with none
 *   (a = B-1) it is drawn from p_{B-1}.  Emits d_1..d_a and the drawn token as
 *   dflash_verify does; next_anchor = the drawn token.
 * Draws are Gumbel-max, argmax_v (log w_v - log(-log U'_v)), ties to the lower
 * id; if fp32 rounding leaves max(0, p_i - q_{i+1}) empty, the draw uses p_i.
 * Uniforms: Philox4x64-10 (Salmon et al., SC 2011) under key (seed, 0),
 * counter (offset, r, stream, n / 4), 64-bit word n % 4; stream 0 gives U_i
 * (n = i) as (w >> 11) 2^-53, stream 1 gives U'_v (n = v) as
 * ((w >> 11) + 1/2) 2^-53.  Equal (seed, offset) repeat the call's draws;
 * advance offset between calls.  Arithmetic is fp32.
 *   target_logits, draft_logits  device [batch, B, V] of logits_dtype
 *                  (DFLASH_BF16 or DFLASH_F32), 16-byte aligned; row 0 of
 *                  draft_logits is not read.
 *   draft_tokens   device int32 [batch, B] (position 0 = anchor).
 *   temperature    in [1e-4, 1e4].
 *   out_tokens .. next_anchor  as in dflash_verify.
 *   ws             workspace of at least
 *                  dflash_verify_sampled_workspace_size(batch, B, V) bytes.
 * Errors as in dflash_verify; B in [2, 32]; 2 * batch * B <= 65535
 * (DFLASH_EUNSUPPORTED beyond); batch == 0 is a no-op.
 */
size_t dflash_verify_sampled_workspace_size(int batch, int B, int V);
int dflash_verify_sampled(const void* target_logits, const void* draft_logits, int logits_dtype,
                          const int32_t* draft_tokens, int batch, int B, int V, float temperature,
                          uint64_t seed, uint64_t offset, int32_t* out_tokens, int32_t* out_len,
                          int out_cap, int32_t* seq_lens, int32_t* accept_len,
                          int32_t* next_anchor, void* ws, size_t ws_bytes, void* stream);

/*
 * Greedy verify without any workspace or allocation.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory -- an inference server that reserves all of its device memory
 * in its own pool at start-up and allows no allocation afterwards, a plugin
 * that runs inside another framework's allocator, or a latency-critical loop
 * that avoids cudaMalloc because it may synchronise the device.
 *
 * Same arguments, semantics and results as dflash_verify, without ws /
 * ws_bytes.  Its scratch (argmax partials, per-request completion counters
 * and the device error word) is a fixed array of 320 KiB + 256 bytes in the
 * library's device memory, present on every GPU that loads the library until
 * the process exits.  That bounds a call
 * to batch * B <= 32768 rows (8 bytes of partials per row chunk; rows are split
 * into chunks only while batch * B < ~600); larger calls return DFLASH_ESCRATCH
 * before anything is enqueued.
 *   error_bits  device int32 out or NULL: the call's device error bits
 *               (DFLASH_DEV_*), written on `stream` at the end of the call.
 * The first call on a device looks up the scratch array's device address and
 * caches it; make that first call before any stream capture.  Every call
 * shares the array and clears its error word at the start: calls that overlap
 * on the GPU (different streams, or different host threads) race on it.
 * Allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 */
int dflash_verify_noalloc(const void* target_logits, int logits_dtype,
                          const int32_t* draft_tokens, int batch, int B, int V,
                          int32_t* out_tokens, int32_t* out_len, int out_cap, int32_t* seq_lens,
                          int32_t* accept_len, int32_t* next_anchor, int32_t* error_bits,
                          void* stream);

/* Waits for `stream`, copies the workspace's device error word to *bits and
 * clears it.  The only call that synchronises with the host. */
int dflash_get_error(void* ws, void* stream, int32_t* bits);

/* Static description of a status code. */
const char* dflash_status_str(int status);

/* Per-kernel-class device timing (CUDA events on the launching stream).  While
 * enabled, every hot call records an event pair around each kernel it launches
 * and adds the elapsed time to the class's total when dflash_timing_read is
 * called.  Classes: 0 GEMM (tcgen05), 1 attention, 2 row/elementwise,
 * 3 verify, 4 LM head.  read() synchronises on the recorded events. */
int dflash_timing_enable(int on);
int dflash_timing_read(double* ms_per_class, int64_t* launches_per_class, int n_classes);

#ifdef __cplusplus
}
#endif
#endif /* DFLASH_H */
