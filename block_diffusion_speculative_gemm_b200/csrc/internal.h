// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>
#include <vector>

#include "../../include/dflash.h"

namespace dflash {

// ---------------------------------------------------------------- launches
// Hot-path launch with programmatic stream serialization (the kernel starts
// while its predecessor finishes; it must begin with pdl_trigger/pdl_wait as
// common.cuh describes).  `cluster` > 1 also groups CTAs into clusters of
// that many along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

// ---------------------------------------------------------------- timing
enum TimingClass { TC_GEMM = 0, TC_ATTN = 1, TC_ROW = 2, TC_VERIFY = 3, TC_LMHEAD = 4, TC_N = 5 };
void timing_begin(cudaStream_t s, int cls);
void timing_end(cudaStream_t s, int cls);
struct TimedScope {
  cudaStream_t s;
  int cls;
  TimedScope(cudaStream_t s_, int c) : s(s_), cls(c) { timing_begin(s, cls); }
  ~TimedScope() { timing_end(s, cls); }
};

// ---------------------------------------------------------------- tcgen05 GEMM
constexpr int kTileN = 128;    // weight rows per CTA tile (UMMA M)
constexpr int kTileK = 64;     // K elements per pipeline stage
constexpr int kMaxSeg = 8;     // K segments of the activation operand
constexpr int kMaxBN = 256;    // largest token tile (UMMA N)

struct LmStat {                // per (token row, 128-wide vocab tile)
  float max;                   // largest logit in the tile
  int32_t idx;                 // its vocabulary id (lowest on ties)
  float sumexp;                // sum over the tile of exp(logit - max)
  float pad;
};

enum GemmEpi { EPI_PARTIAL = 0, EPI_LMHEAD = 1 };

// Where injected K/V rows live.  table == nullptr: the contiguous cache
// [L][batch][nkv][cap][hd].  Otherwise paged pools [L][n_pages][nkv][page][hd]
// (prefix sharing): position p of request r is at page table[r * max_pages +
// p / page], slot p % page; `page` is a multiple of 64 so that no 64-key
// attention tile crosses a page.
struct KvPages {
  const int32_t* table = nullptr;
  const int32_t* req_ok = nullptr;  // injection: 1 when every page a request's rows touch is mapped
  int max_pages = 0, page = 0, n_pages = 0;
};

// Row (in units of hd elements) of (layer, request, position, head) in the K/V
// store of `batch` requests and capacity `cap`, for a mapped position.
__host__ __device__ inline int64_t kv_row(const KvPages& pg, int layer, int batch, int req,
                                          int nkv, int head, int cap, int pos) {
  if (pg.table == nullptr) return (((int64_t)layer * batch + req) * nkv + head) * cap + pos;
  const int page = pg.table[(int64_t)req * pg.max_pages + pos / pg.page];
  return (((int64_t)layer * pg.n_pages + page) * nkv + head) * pg.page + pos % pg.page;
}

// What the EPI_PARTIAL kernel does with the product Y[m][n] = sum_k X[m][k] W[n][k].
// OP_PARTIAL writes each K split's share (fp32, for a reduction kernel); the
// other ops need an unsplit GEMM and apply the step that follows the
// projection on the hot path straight from the accumulator.
enum GemmOp {
  OP_PARTIAL = 0,  // part[split][m][n] = split's share                         (fp32)
  OP_STORE = 1,    // f32[m][n] = Y                                             (fp32)
  OP_RESID = 2,    // f32[m][n] += Y   (the residual stream)                    (fp32)
  OP_QKV = 3,      // Y = [q heads | k heads | v heads]: RoPE on q and k at position
                   // ctx_len[m / B] + m % B; h1 = q [M][nq][hd], h2 = k [M][nkv][hd],
                   // h3 = v [M][nkv][hd]                                       (fp16)
  OP_SWIGLU = 4,   // weight rows interleaved in 64-row blocks (64 gate rows, then the
                   // 64 up rows of the same features): h1 = act [M][I] = silu(g) * u
  OP_KV = 5,       // Y = per layer [K heads | V heads] of injected rows row0 + m:
                   // RoPE on K at start_pos[r] + row - cu_rows[r]; h1/h2 = K/V cache
                   // [L][batch][nkv][cap][hd] (fp16); bad positions set err, skip
};

struct GemmOut {
  int op = OP_PARTIAL;
  float* part = nullptr;          // OP_PARTIAL: [splits][M][N] fp32
  LmStat* stats = nullptr;        // EPI_LMHEAD: [M][ceil(N/128)]
  int vocab_offset = 0;           // EPI_LMHEAD: global id of weight row 0 (a vocabulary shard)
  void* dbg = nullptr;            // EPI_LMHEAD, optional: logits rows
  const int32_t* dbg_rows = nullptr;  // token row -> dbg row
  int64_t dbg_ld = 0;             // dbg row stride (elements)
  int dbg_bf16 = 0;               // dbg rows stored as bf16 (else fp32)
  const int32_t* dbg_valid = nullptr;  // optional: skip dbg row d when !dbg_valid[d / B]
  // fused ops
  float* f32 = nullptr;           // OP_STORE / OP_RESID: [M][N]
  __half* h1 = nullptr;
  __half* h2 = nullptr;
  __half* h3 = nullptr;
  const float* cos_t = nullptr;   // RoPE tables [max_pos][hd/2]
  const float* sin_t = nullptr;
  const int32_t* ctx_len = nullptr;    // OP_QKV
  const int32_t* req_valid = nullptr;  // OP_QKV
  const int32_t* cu_rows = nullptr;    // OP_KV
  const int32_t* start_pos = nullptr;  // OP_KV
  KvPages pages;                       // OP_KV: the K/V store (contiguous when no table)
  // stream-K schedule (gemm_tc with splits == 0): fixup shares and per-tile
  // counters (2 per tile, zero before and after the call)
  float* sk_slots = nullptr;           // gemm_sk_slot_bytes(M) bytes
  unsigned* sk_cnt = nullptr;
  int sk_cnt_cap = 0;                  // counters available
  int64_t kv_ls = 0, kv_hs = 0;        // OP_KV: rows between layers / between heads
  int B = 0, nq = 0, nkv = 0, hd = 0, I = 0;
  int row0 = 0, batch = 0, cap = 0, max_pos = 0;
};


// A weight operand prepared once: tensor map over [N, K] rows of 16-bit
// elements (elem = DFLASH_BF16 or DFLASH_F16).  The activation operand of a
// GEMM against it must have the same element type.
//
// `tiled`, when set, holds the same weights pre-tiled for streaming: tile
// (n-tile t, k-block kb) is 16 KB at ((t * K/64) + kb) * 16384, already in the
// 128-byte-swizzled shared-memory image of a [128 x 64] K-major tile, so the
// GEMM fetches it with one bulk copy instead of a 128-row tensor box.
struct WeightMap {
  CUtensorMap map;         // row-major weights, 128-byte swizzle (when ptr is set)
  CUtensorMap tmap;        // pre-tiled weights as rows of 128 bytes, no swizzle
  const void* ptr = nullptr;
  const void* tiled = nullptr;
  int N = 0, K = 0;
  int elem = DFLASH_BF16;
};

bool encode_weight_map(WeightMap& w, const void* ptr, int N, int K, int elem);
// Sets w.tiled and the tensor map the CTA-pair GEMM streams it through.
bool set_tiled_weights(WeightMap& w, const void* tiled);

// CTA-pair GEMM choice for M token rows and N weight rows; a debug override
// (0 automatic, 1 single CTAs, 2 pairs) replaces the rule when non-zero.
bool gemm_use_pair(int M, int N);
void gemm_set_mode(int mode);
// Weight of the split partials' traffic in the split picker (default 4).
void gemm_set_split_weight(float w);

// Writes the pre-tiled streaming image of a row-major 16-bit W [N, K] (K % 64
// == 0) into dst (ceil(N/128) * K/64 * 16384 bytes; rows past N are zero).
void tile_weights(const void* src, void* dst, int N, int K, cudaStream_t s);
size_t tiled_bytes(int N, int K);

// 2D tensor map over `rows` rows of `cols` 16-bit elements (row stride `ld`
// elements) with a box of 64 columns x box_rows rows, 128-byte swizzle, zero
// fill outside the tensor.
bool encode_2d(CUtensorMap* m, const void* ptr, int64_t rows, int cols, int ld, int box_rows,
               int elem);

// Y = X * W^T for X [M, K] of W's element type (given as n_seg K-segments of
// seg_k columns, each [M, seg_k] with row stride ld_seg elements) and W [N, K].
// splits >= 1: fixed K splits (OP_PARTIAL writes each split's share; a fused
// op needs splits == 1).  splits == 0: stream-K, every worker the same number
// of k-blocks, tiles split between workers finished in the kernel (any op,
// and the LM-head epilogue), with out.sk_slots / out.sk_cnt as scratch.
int gemm_tc(const WeightMap& W, const void* const* xseg, int n_seg, int seg_k, int ld_seg, int M,
            int splits, int epi, const GemmOut& out, int32_t* err, cudaStream_t s);

// Number of K splits for an M x N x K weight-streaming GEMM; always a count
// that gemm_tc uses unchanged (see gemm_effective_splits).
int gemm_pick_splits(int M, int N, int K, int max_splits);
// Fixup scratch of a stream-K GEMM of M token rows (an upper bound for any N, K).
size_t gemm_sk_slot_bytes(int M);
// The split count gemm_tc actually runs for a requested count: every split
// gets ceil(k-blocks / splits) k-blocks, the last one possibly fewer.
int gemm_effective_splits(int K, int splits);

// ---------------------------------------------------------------- fp32 SIMT GEMM
void gemm_simt_f32(const float* W, int N, int K, const float* const* xseg, int n_seg, int seg_k,
                   int M, float* out, cudaStream_t s);

// ---------------------------------------------------------------- row kernels
// The row kernels that store fp16 set DFLASH_DEV_RANGE in err when a value
// overflows fp16 (see narrow_bad).
template <typename TE, typename T>
void launch_embed_norm(const int32_t* tokens, const TE* emb, const float* g, float* x, T* h, int M,
                       int d, float eps, int32_t* err, cudaStream_t s);
template <typename T>
void launch_residual_norm(const float* part, int splits, int M, int d, float* x, const float* g,
                          T* h, const int32_t* out_row, float eps, int32_t* err, cudaStream_t s);
template <typename T>
void launch_ctx_norm(const float* part, int splits, int n, int d, const float* g, T* c, float eps,
                     int32_t* err, cudaStream_t s);
template <typename T>
void launch_qkv_post(const float* part, int splits, int M, int B, const int32_t* ctx_len,
                     const int32_t* req_valid, int nq, int nkv, int hd, const float* cos_t,
                     const float* sin_t, T* q, T* kb, T* vb, int32_t* err, cudaStream_t s);
template <typename T>
void launch_swiglu(const float* part, int splits, int M, int I, T* act, int32_t* err,
                   cudaStream_t s);
// cap: positions per request (max_pages * page when paged).
template <typename T>
void launch_kv_scatter(const float* part, int splits, int n_rows, int row0, int L, int nkv, int hd,
                       const int32_t* cu_rows, const int32_t* start_pos, int batch, int cap,
                       const KvPages& pages, const float* cos_t, const float* sin_t, int max_pos,
                       T* kc, T* vc, int32_t* err, cudaStream_t s);
// One warp per request: req_ok[r] = 1 when every page holding positions
// start_pos[r] .. start_pos[r] + rows - 1 is mapped, else 0 and DFLASH_DEV_PAGE.
void launch_inject_page_check(const int32_t* cu_rows, const int32_t* start_pos, int batch,
                              const KvPages& pages, int32_t* req_ok, int32_t* err, cudaStream_t s);

// ---------------------------------------------------------------- attention
constexpr int kAttnMaxRows = 64;  // B * (n_q / n_kv) query rows per (request, kv head)

// Tensor-core block attention (fp16 rows and fp16 cache) with its chunk
// combine: split-KV partials part_o [batch][nkv][n_chunks][kAttnMaxRows][hd]
// fp32 and part_ml [...][2] (max, sum); the last chunk CTA of each (request,
// kv head), found with cnt[request * nkv + head] (zero before and after the
// call), merges them into o [batch * B][nq][hd].  The cache is
// [L][batch][nkv][cap][hd]; `layer` selects the layer.
// Persistent schedule: seg_start (from launch_attn_plan, once per forward)
// non-null; partials part_o [(2 * SMs + batch * nkv) * 64][hd] and part_ml
// [...][2]; cnt one zeroed counter per (request, kv head).  seg_start null: the
// split-KV grid of `chunk`-key chunks.
int launch_attn_plan(const int32_t* ctx_len, const int32_t* req_valid, int batch, int nkv,
                     int32_t* seg_start, cudaStream_t s);
// Split-KV grid: the plan of every attention launch of one forward, made on
// the device from the requests' actual context lengths.  plan receives {chunk,
// n_items, -, -, items}: the chunk in keys, a multiple of 64 and at least
// chunk_min (so a grid sized for chunk_min always covers the list), chosen to
// minimise an estimate of the grid's time (waves of CTAs over `slots` resident
// CTAs times the tiles plus a fixed cost of one chunk, plus the merge of a mean
// request's chunks); plan[2..3] unused; then from int 4 one pair per (request,
// kv head, chunk) with keys, {request << 16 | kv head << 8 | chunk index, the
// request's context length (0 when it is not valid)}, request-major.  plan
// holds 4 + 2 * batch * nkv * ceil((cap + B) / chunk_min) ints, 8-byte aligned.
// slots: attn_grid_slots for the kernel the grid runs.
int launch_attn_chunk_plan(const int32_t* ctx_len, const int32_t* req_valid, int batch, int B,
                           int nkv, int chunk_min, int32_t* chunk_out, int slots,
                           cudaStream_t s);
// CTAs of the split-KV grid kernel (head dim hd, R = B * n_q / n_kv query rows
// per kv head, contiguous or paged K/V) that are resident at once on the GPU.
int attn_grid_slots(int hd, int R, int B, bool paged);
// The tcgen05 attention kernel (head dim 128, at most 32 query rows per kv
// head, contiguous K/V, the grid schedule): used by launch_attn_tc while
// g_attn_umma is set (dflash_debug_attn_schedule(2)); tk/tv are tensor maps of
// 64-row, 64-column boxes (the mma.sync kernel's).  DFLASH_EUNSUPPORTED
// outside its shapes (and for a chunk that is not a multiple of 64 keys).
extern int g_attn_umma;
int attn_umma_ctas_per_sm();  // resident CTAs per SM of the tcgen05 attention kernel
int launch_attn_umma(const CUtensorMap& tk, const CUtensorMap& tv, const __half* q,
                     const __half* kb, const __half* vb, const KvPages& pg, long long kv_rows,
                     int layer, int batch, int cap, const int32_t* ctx_len,
                     const int32_t* req_valid, int B, int nq, int nkv, int chunk,
                     const int32_t* plan_dev, int n_chunks, float* part_o, float* part_ml,
                     unsigned* cnt, __half* o, int32_t* err, cudaStream_t s);
int launch_attn_tc(const __half* q, const __half* kb, const __half* vb, const __half* kc,
                   const __half* vc, const KvPages& pages, int layer, int batch, int cap,
                   const int32_t* ctx_len, const int32_t* req_valid, int B, int nq, int nkv,
                   int hd, int L, int chunk, const int32_t* plan_dev, int n_chunks,
                   const int32_t* seg_start, float* part_o, float* part_ml, unsigned* cnt,
                   __half* o, int32_t* err, cudaStream_t s);

// T: type of q, the block's k/v and the output o; TC: K/V cache type.
// Paged K/V (pages.table set) and the persistent schedule (seg_start set) are
// the tensor-core kernel's only.
template <typename T, typename TC>
int launch_block_attention(const T* q, const T* kb, const T* vb, const TC* kc, const TC* vc,
                           const KvPages& pages, int layer, int L, int batch, int cap,
                           const int32_t* ctx_len, const int32_t* req_valid, int B, int nq,
                           int nkv, int hd, float* part_o, float* part_ml, int n_chunks, int chunk,
                           const int32_t* plan_dev, const int32_t* seg_start, T* o,
                           unsigned* cnt, int32_t* err, cudaStream_t s);

// ---------------------------------------------------------------- draft bookkeeping
// cap bounds ctx_len + B; with paged K/V every page below ctx_len must also be
// mapped (else the request is invalid and DFLASH_DEV_PAGE is set).
void launch_draft_init(const int32_t* anchor, const int32_t* ctx_len, int batch, int B, int V,
                       int mask_id, int cap, const KvPages& pages, int32_t* tokens, int32_t* zrow,
                       int32_t* lm_rows, int32_t* cstep, int32_t* req_valid, int32_t* err,
                       cudaStream_t s);
// Per row q: merges the n_tiles statistics stats[q * row_stride + t * tile_stride]
// (t ascending) into the row's argmax token and max-probability confidence,
// and, when out_stat is given, the merged (max, id, sum) itself.
void launch_lm_reduce(const LmStat* stats, int n_tiles, int rows, int64_t row_stride,
                      int64_t tile_stride, int32_t* tok, float* conf, LmStat* out_stat,
                      cudaStream_t s);
// dbg (optional): logits rows copied to dbg[dbg_rows[q] * dbg_ld ...] as fp32, or
// as bf16 when dbg_bf16; rows of requests with !dbg_valid[dbg_rows[q] / B] are
// skipped when dbg_valid is given.
void launch_lm_stats_from_logits(const float* logits, int rows, int V, LmStat* stats,
                                 void* dbg, const int32_t* dbg_rows, int64_t dbg_ld,
                                 int dbg_bf16, const int32_t* dbg_valid, int B, cudaStream_t s);

// ---------------------------------------------------------------- sampled drafting
// Draw of every still-masked row at denoising step `step` from its logits row
// q[lm_rows[row]] (fp32, or bf16 when q_bf16): Gumbel-max at temperature tau with
// Philox4x64-10 stream 2 noise, and the untempered probability of the drawn
// token.  part: [rows][chunks] partials; cnt: one zeroed counter per row.
int sampled_draw_chunks(int rows, int V);
size_t sampled_draw_part_bytes(int rows, int chunks);
// Rows of requests with !req_valid[r] (req_valid nullable) read nothing and draw
// token 0 with confidence 0.
int launch_sampled_draw(const void* q, int q_bf16, const int32_t* lm_rows,
                        const int32_t* req_valid, int rows, int B, int V, int step, float tau,
                        uint64_t seed, uint64_t offset, int32_t* tok, float* conf, void* part,
                        int chunks, unsigned* cnt, cudaStream_t s);
void launch_commit(const int32_t* tok, const float* conf, int batch, int B, int rem, int k,
                   int step, int32_t* tokens, int32_t* zrow, int32_t* lm_rows, int32_t* cstep,
                   int32_t* err, cudaStream_t s);
void launch_draft_finish(const int32_t* tokens, const int32_t* cstep, const int32_t* req_valid,
                         int batch, int B, int32_t* draft_out, int32_t* cstep_out,
                         cudaStream_t s);

// ---------------------------------------------------------------- verify
int launch_verify(const void* logits, int dtype, const int32_t* draft, int batch, int B, int V,
                  int32_t* out_tokens, int32_t* out_len, int out_cap, int32_t* seq_lens,
                  int32_t* accept_len, int32_t* next_anchor, void* part, int chunks,
                  unsigned* cnt, int32_t* err, cudaStream_t s);
int verify_chunks(int rows, int V);
// Vocabulary shard of verify: per row, the (largest logit, lowest global id)
// over the shard's columns (global id = vocab_offset + column).
struct ArgPart {
  float v;
  int32_t i;
};
int launch_verify_shard(const void* logits, int dtype, int batch, int B, int Vs, int vocab_offset,
                        ArgPart* out, void* part, int chunks, unsigned* cnt, cudaStream_t s);
// Accept step from per-shard row argmaxes parts[w * batch * B + row], w < world
// (shards in ascending vocabulary order).
int launch_verify_merge(const ArgPart* parts, int world, const int32_t* draft, int batch, int B,
                        int V, int32_t* out_tokens, int32_t* out_len, int out_cap,
                        int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor,
                        int32_t* err, cudaStream_t s);

// ---------------------------------------------------------------- sampled verify
// Scratch bytes of one sampled-verify call (placed after the workspace header).
size_t sampled_verify_bytes(int batch, int B, int V);
int launch_sample_math(const uint64_t* w, const float* d, int n, float* g2, float* l2,
                       cudaStream_t s);
int launch_sampled_verify(const void* target, const void* drafted, int dtype, const int32_t* draft,
                          int batch, int B, int V, float tau, uint64_t seed, uint64_t offset,
                          int32_t* out_tokens, int32_t* out_len, int out_cap, int32_t* seq_lens,
                          int32_t* accept_len, int32_t* next_anchor, void* scratch,
                          unsigned* cnt, int32_t* err, cudaStream_t s);

}  // namespace dflash
