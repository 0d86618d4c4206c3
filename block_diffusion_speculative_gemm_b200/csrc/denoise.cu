// Draft-block bookkeeping: block initialisation, reduction of the LM-head tile
// statistics to (token, confidence) per masked row, and the confidence-ordered
// commit of each denoising step ("DFlash + Spec V2 深度解析", §2.3: start from an
// all-[MASK] block behind the anchor, predict every position in one forward,
// fix positions over 2-3 rounds).
//
// Device state per request r and block position j (row m = r*B + j):
//   tokens[m]   current token (anchor, committed token or mask id)
//   zrow[m]     compact LM-head row of a still-masked position, -1 otherwise
//   lm_rows[q]  inverse map: compact row q -> m
//   cstep[m]    step at which position j was committed (-1 for the anchor)
// Compact rows are request-major with positions ascending; every request has
// the same number of masked positions at a given step, so row q belongs to
// request q / rem.
#include "common.cuh"
#include "internal.h"

namespace dflash {

// One warp per request (lane j = block position j; blockDim.x == 32).  With
// paged K/V the warp also checks that every page holding a context position
// is mapped; a request with an unmapped one is invalid (DFLASH_DEV_PAGE).
__global__ void draft_init_kernel(const int32_t* __restrict__ anchor,
                                  const int32_t* __restrict__ ctx_len, int batch, int B, int V,
                                  int mask_id, int cap, const KvPages pg, int32_t* tokens,
                                  int32_t* zrow, int32_t* lm_rows, int32_t* cstep,
                                  int32_t* req_valid, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * blockDim.y + threadIdx.y;
  const int j = threadIdx.x;
  if (r >= batch) return;  // the whole warp
  const int a = anchor[r];
  const int T = ctx_len[r];
  const bool ok_tok = a >= 0 && a < V;
  const bool ok_ctx = T >= 0 && (long long)T + B <= cap;
  bool ok_page = true;
  if (pg.table != nullptr && ok_ctx) {
    bool bad = false;
    const int n_pg = (T + pg.page - 1) / pg.page;
    for (int k = j; k < n_pg; k += 32) {
      const int e = k < pg.max_pages ? pg.table[(long long)r * pg.max_pages + k] : -1;
      bad |= e < 0 || e >= pg.n_pages;
    }
    ok_page = !__any_sync(0xffffffffu, bad);
  }
  if (j >= B) return;
  if (j == 0) {
    req_valid[r] = (ok_tok && ok_ctx && ok_page) ? 1 : 0;
    if (!ok_tok) set_error(err, DFLASH_DEV_TOKEN_RANGE);
    if (!ok_ctx) set_error(err, DFLASH_DEV_CTX_CAP);
    if (!ok_page) set_error(err, DFLASH_DEV_PAGE);
  }
  const int m = r * B + j;
  tokens[m] = j == 0 ? (ok_tok ? a : 0) : mask_id;
  cstep[m] = -1;
  if (j == 0) {
    zrow[m] = -1;
  } else {
    const int qrow = r * (B - 1) + (j - 1);
    zrow[m] = qrow;
    lm_rows[qrow] = m;
  }
}

void launch_draft_init(const int32_t* anchor, const int32_t* ctx_len, int batch, int B, int V,
                       int mask_id, int cap, const KvPages& pages, int32_t* tokens, int32_t* zrow,
                       int32_t* lm_rows, int32_t* cstep, int32_t* req_valid, int32_t* err,
                       cudaStream_t s) {
  dim3 block(32, 8);
  TimedScope ts(s, TC_ROW);
  launch_pdl(draft_init_kernel, dim3((batch + 7) / 8), dim3(block), 0, s, 1, anchor, ctx_len, batch,
      B, V, mask_id, cap, pages, tokens, zrow, lm_rows, cstep, req_valid, err);
}

// Merge of two tile statistics: the larger maximum wins (lower id on equal
// maxima); the exp-sums are rescaled to the winning maximum.
__device__ __forceinline__ void stat_merge(float& mx, int& id, float& se, float m2, int i2,
                                           float s2) {
  if (m2 > mx || (m2 == mx && i2 < id)) {
    se = se * expf(mx - m2) + s2;
    mx = m2;
    id = i2;
  } else {
    se = se + s2 * expf(m2 - mx);
  }
}

__global__ void lm_reduce_kernel(const LmStat* __restrict__ stats, int n_vtiles,
                                 int64_t row_stride, int64_t tile_stride,
                                 int32_t* __restrict__ tok, float* __restrict__ conf,
                                 LmStat* __restrict__ out_stat) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_m[32], s_s[32];
  __shared__ int s_i[32];
  const int q = blockIdx.x;
  const LmStat* st = stats + (int64_t)q * row_stride;
  float mx = -INFINITY, se = 0.f;
  int id = 0x7fffffff;
  for (int t = threadIdx.x; t < n_vtiles; t += blockDim.x) {
    const LmStat v = st[(int64_t)t * tile_stride];
    if (v.max == -INFINITY) continue;  // an empty tile (a shard with no columns)
    if (mx == -INFINITY) { mx = v.max; id = v.idx; se = v.sumexp; continue; }
    stat_merge(mx, id, se, v.max, v.idx, v.sumexp);
  }
  // tree merge inside the warp, then across warps
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, mx, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, id, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, se, o);
    if (m2 == -INFINITY) continue;
    if (mx == -INFINITY) { mx = m2; id = i2; se = s2; continue; }
    stat_merge(mx, id, se, m2, i2, s2);
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) { s_m[w] = mx; s_i[w] = id; s_s[w] = se; }
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = s_m[0], S = s_s[0];
    int I = s_i[0];
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k) {
      if (s_m[k] == -INFINITY) continue;
      if (M == -INFINITY) { M = s_m[k]; I = s_i[k]; S = s_s[k]; continue; }
      stat_merge(M, I, S, s_m[k], s_i[k], s_s[k]);
    }
    if (tok) tok[q] = I;
    if (conf) conf[q] = 1.f / S;
    if (out_stat) out_stat[q] = LmStat{M, I, S, 0.f};
  }
}

void launch_lm_reduce(const LmStat* stats, int n_tiles, int rows, int64_t row_stride,
                      int64_t tile_stride, int32_t* tok, float* conf, LmStat* out_stat,
                      cudaStream_t s) {
  if (rows <= 0) return;
  TimedScope ts(s, TC_ROW);
  launch_pdl(lm_reduce_kernel, dim3(rows), dim3(256), 0, s, 1, stats, n_tiles, row_stride,
             tile_stride, tok, conf, out_stat);
}

// fp32 model type: tile statistics from a full logits matrix [rows, V].
__global__ void lm_stats_from_logits_kernel(const float* __restrict__ logits, int V,
                                            LmStat* __restrict__ stats, void* dbg,
                                            const int32_t* dbg_rows, int64_t dbg_ld,
                                            int dbg_bf16, const int32_t* dbg_valid, int B) {
  pdl_trigger();
  pdl_wait();
  const int q = blockIdx.y, t = blockIdx.x;
  const int n_vtiles = gridDim.x;
  const int v = t * kTileN + threadIdx.x;
  const float x = v < V ? logits[(size_t)q * V + v] : -INFINITY;
  if (dbg && v < V) {
    const int64_t d = dbg_rows[q];
    if (!dbg_valid || dbg_valid[d / B]) {
      if (dbg_bf16)
        static_cast<__nv_bfloat16*>(dbg)[d * dbg_ld + v] = __float2bfloat16_rn(x);
      else
        static_cast<float*>(dbg)[d * dbg_ld + v] = x;
    }
  }
  __shared__ float xs[kTileN];
  xs[threadIdx.x] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mx = xs[0];
    int bi = 0;
    for (int i = 1; i < kTileN; ++i)
      if (xs[i] > mx) { mx = xs[i]; bi = i; }
    float se = 0.f;
    for (int i = 0; i < kTileN; ++i) se += expf(xs[i] - mx);
    LmStat st;
    st.max = mx;
    st.idx = t * kTileN + bi;
    st.sumexp = se;
    st.pad = 0.f;
    stats[(size_t)q * n_vtiles + t] = st;
  }
}

void launch_lm_stats_from_logits(const float* logits, int rows, int V, LmStat* stats,
                                 void* dbg, const int32_t* dbg_rows, int64_t dbg_ld,
                                 int dbg_bf16, const int32_t* dbg_valid, int B, cudaStream_t s) {
  if (rows <= 0) return;
  dim3 grid((V + kTileN - 1) / kTileN, rows);
  TimedScope ts(s, TC_LMHEAD);
  launch_pdl(lm_stats_from_logits_kernel, dim3(grid), dim3(kTileN), 0, s, 1, logits, V, stats, dbg,
      dbg_rows, dbg_ld, dbg_bf16, dbg_valid, B);
}

// One warp per request, lane j = block position j.  The k most confident
// still-masked positions (ties to the lower position) take their argmax token;
// the others get new compact rows for the next step.  A warp touches only its
// own request's rows of zrow/tokens/cstep and its own compact range of lm_rows.
__global__ void commit_kernel(const int32_t* __restrict__ tok, const float* __restrict__ conf,
                              int batch, int B, int rem, int k, int step, int32_t* tokens,
                              int32_t* zrow, int32_t* lm_rows, int32_t* cstep, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= batch) return;
  const int m = r * B + lane;
  int q = lane < B ? zrow[m] : -1;
  if (q >= 0 && !DFLASH_CHECK(q < batch * rem, err)) q = -1;
  const bool live = q >= 0;
  const float c = live ? conf[q] : -INFINITY;
  const int t = live ? tok[q] : 0;
  bool chosen = false;
  for (int it = 0; it < k; ++it) {
    float bc = (live && !chosen) ? c : -INFINITY;
    int bp = (live && !chosen) ? lane : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float c2 = __shfl_xor_sync(0xffffffffu, bc, o);
      const int p2 = __shfl_xor_sync(0xffffffffu, bp, o);
      if (c2 > bc || (c2 == bc && p2 < bp)) { bc = c2; bp = p2; }
    }
    if (live && lane == bp) chosen = true;
  }
  const unsigned keep = __ballot_sync(0xffffffffu, live && !chosen);
  const int new_rem = rem - k;
  if (live) {
    if (chosen) {
      tokens[m] = t;
      cstep[m] = step;
      zrow[m] = -1;
    } else {
      const int nq = r * new_rem + __popc(keep & ((1u << lane) - 1u));
      zrow[m] = nq;
      lm_rows[nq] = m;
    }
  }
}

void launch_commit(const int32_t* tok, const float* conf, int batch, int B, int rem, int k,
                   int step, int32_t* tokens, int32_t* zrow, int32_t* lm_rows, int32_t* cstep,
                   int32_t* err, cudaStream_t s) {
  TimedScope ts(s, TC_ROW);
  const int wpb = 4;
  launch_pdl(commit_kernel, dim3((batch + wpb - 1) / wpb), dim3(32 * wpb), 0, s, 1, tok, conf,
      batch, B, rem, k, step, tokens, zrow, lm_rows, cstep, err);
}

__global__ void draft_finish_kernel(const int32_t* __restrict__ tokens,
                                    const int32_t* __restrict__ cstep,
                                    const int32_t* __restrict__ req_valid, int batch, int B,
                                    int32_t* draft_out, int32_t* cstep_out) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= batch * B) return;
  if (!req_valid[m / B]) return;
  draft_out[m] = tokens[m];
  if (cstep_out) cstep_out[m] = cstep[m];
}

void launch_draft_finish(const int32_t* tokens, const int32_t* cstep, const int32_t* req_valid,
                         int batch, int B, int32_t* draft_out, int32_t* cstep_out,
                         cudaStream_t s) {
  TimedScope ts(s, TC_ROW);
  const int n = batch * B;
  launch_pdl(draft_finish_kernel, dim3((n + 255) / 256), dim3(256), 0, s, 1, tokens, cstep,
      req_valid, batch, B, draft_out, cstep_out);
}

}  // namespace dflash
