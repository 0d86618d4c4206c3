// Persistent tcgen05 weight-streaming GEMM for sm_100a.
//
// Every dense contraction of the draft hot path multiplies a small set of
// token rows X [M, K] (M <= 256 per tile) by a large weight W [N, K]:
// context-feature fc, the layer-batched K/V injection projection, the QKV,
// output and SwiGLU projections, and the LM head.  A tile therefore puts 128
// weight rows on the UMMA M axis and up to 256 token rows on the UMMA N axis
// ("swap-AB"): each weight tile streams from HBM once, the token tile is
// re-read from L2.
//
// Work units are (token tile, weight tile, K split), ordered split-major so
// that CTAs running at the same time share the K range of X.  One CTA per SM
// walks units u = blockIdx.x, + gridDim.x, ... with warp-specialised roles:
//   warp 0 (one lane)  TMA producer: per 64-wide k-block, the weight tile
//                      [128 x 64] and the token tile [BN x 64], 128-byte
//                      swizzled, through a ring of `stages` smem stages that
//                      runs on across unit boundaries.
//   warp 1 (one lane)  MMA issuer: 4 x tcgen05.mma (K = 16) per stage into one
//                      of two TMEM accumulators (128 lanes x BN fp32 columns),
//                      alternating per unit; tcgen05.commit releases the stage.
//   warps 2..5         epilogue: drain the accumulator of unit j while the
//                      MMA warp fills the other one for unit j + 1, then give it
//                      back.  PARTIAL: coalesced fp32 store of the split's
//                      partial product (kept in L2 for the reduction kernel),
//                      or, for an unsplit GEMM, a fused step (residual add,
//                      RoPE + q/k/v split, SwiGLU, K/V cache scatter).  LMHEAD: per token and 128-row
//                      vocabulary tile, the maximum, its lowest index and the
//                      sum of exp(logit - max), through per-warp 32 x 33 shared
//                      transposes (no fp32 logits leave the SM).
// Every mbarrier wait is bounded (1 s) and reports DFLASH_DEV_TIMEOUT.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dflash {

struct BMaps {
  CUtensorMap m[kMaxSeg];
};

struct GemmArgs {
  int N, M;
  int seg_k;          // K columns per activation segment
  int BN;             // token tile (multiple of 32)
  int stages;
  int kb_per_split;   // 64-wide k-blocks per split
  int n_kb;           // total k-blocks
  int tiles_n;        // weight tiles
  int tiles_m;        // token tiles
  int units;          // tiles_n * tiles_m * splits
  int splits;
  int tile_rows;      // weight rows per unit: 128, or 256 for a CTA pair
  int n_vtiles;       // LM head: number of 128-row vocabulary tiles
  int epi_bytes;      // shared bytes of the epilogue region
  uint32_t idesc;     // tcgen05 instruction descriptor (operand type, tile_rows x BN)
  const uint8_t* a_tiled;  // pre-tiled weights (bulk copies) or null (tensor map)
  // stream-K schedule (sk = 1): workers (CTAs, or pairs) take equal shares of
  // the sk_W = tiles * n_kb (tile, k-block) iterations, tiles in order; a tile
  // split between workers is finished by whichever of its pieces arrives last
  int sk;
  int sk_P;
  long long sk_W;
  GemmOut out;
  int32_t* err;
};

constexpr int kGemmThreads = 192;
constexpr int kMaxStages = 8;   // smem ring depth cap
constexpr int kEpiWarp0 = 2;  // first epilogue warp
constexpr int kLmTr = 32 * 33;  // floats of one warp's transpose buffer
constexpr int kStLd = kTileN + 1; // row stride of the fused-op staging tile [32 tokens][128 rows]
// staging tile + token maps (request, position: int; row base: int64) + flag
constexpr int kFusedSmem = 32 * kStLd * 4 + 64 * 4 + 32 * 8 + 16;
constexpr int kLmSmem = 4 * kLmTr * 4 + 4 * kMaxBN * (int)sizeof(LmStat);

// Applies the fused op to one 32-token chunk of a finished output tile.
// st[j * kStLd + r] = Y[m_base + j][n0 + r]; t = epilogue thread (0..127).
// For OP_KV, tok_req/tok_pos hold each token's request and position (request
// -1: skip) and tok_base the token's row in the K/V store at layer 0, head 0.
// fp16 results that overflow set DFLASH_DEV_RANGE in err.
//
// Every op issues all of a chunk's global loads (the residual stream, the RoPE
// table entries) before its first store: a load placed after a store the
// compiler cannot prove disjoint would wait for it, and 32 tokens of
// dependent round trips per chunk would stall the epilogue.
__device__ __forceinline__ void apply_op(const GemmOut& o, int M, int N, const float* st,
                                         const int* tok_req, const int* tok_pos,
                                         const long long* tok_base, int m_base, int n0, int t,
                                         int32_t* err) {
  bool bad = false;
  const int jn = min(32, M - m_base);  // tokens of this chunk
  switch (o.op) {
    case OP_STORE:
    case OP_RESID: {
      const int n = n0 + t;
      if (n >= N) break;
      float* base = o.f32 + (size_t)m_base * N + n;
      float old[32];
#pragma unroll
      for (int j = 0; j < 32; ++j)
        old[j] = (o.op == OP_RESID && j < jn) ? base[(size_t)j * N] : 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < jn) base[(size_t)j * N] = old[j] + st[j * kStLd + t];
    } break;
    case OP_SWIGLU: {
      const int p = t & 63, par = t >> 6;
      const int i = (n0 >> 1) + p;
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        const int j = par + 2 * jj;
        if (j >= jn) break;
        const float g = st[j * kStLd + p], u = st[j * kStLd + p + 64];
        const float y = g / (1.f + expf(-g)) * u;
        o.h1[(size_t)(m_base + j) * o.I + i] = __float2half_rn(y);
        bad |= narrow_bad<__half>(y);
      }
    } break;
    case OP_QKV: {
      const int hd = o.hd, half = hd >> 1;
      const int p = t & 63, par = t >> 6;
      const int hl = p / half, i = p % half;
      const int ra = hl * hd + i;
      const int head = (n0 + hl * hd) / hd;
      const bool rope = head < o.nq + o.nkv;
      float cs[16], sn[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        const int j = par + 2 * jj;
        cs[jj] = 1.f;
        sn[jj] = 0.f;
        if (rope && j < jn) {
          const size_t e = (size_t)tok_pos[j] * half + i;
          cs[jj] = o.cos_t[e];
          sn[jj] = o.sin_t[e];
        }
      }
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        const int j = par + 2 * jj;
        if (j >= jn) break;
        const int m = m_base + j;
        const float x1 = st[j * kStLd + ra], x2 = st[j * kStLd + ra + half];
        const float y1 = x1 * cs[jj] - x2 * sn[jj], y2 = x2 * cs[jj] + x1 * sn[jj];
        __half* dst = head < o.nq    ? o.h1 + ((size_t)m * o.nq + head) * hd
                      : rope         ? o.h2 + ((size_t)m * o.nkv + head - o.nq) * hd
                                     : o.h3 + ((size_t)m * o.nkv + head - o.nq - o.nkv) * hd;
        dst[i] = __float2half_rn(y1);
        dst[i + half] = __float2half_rn(y2);
        bad |= narrow_bad<__half>(y1) || narrow_bad<__half>(y2);
      }
    } break;
    case OP_KV: {
      const int hd = o.hd, half = hd >> 1;
      const int p = t & 63, par = t >> 6;
      const int hl = p / half, i = p % half;
      const int ra = hl * hd + i;
      const int per_layer = 2 * o.nkv * hd;
      const int nl = n0 + hl * hd;
      const int layer = nl / per_layer, wl = nl % per_layer;
      const bool is_v = wl >= o.nkv * hd;
      const int head = (wl % (o.nkv * hd)) / hd;
      float cs[16], sn[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        const int j = par + 2 * jj;
        cs[jj] = 1.f;
        sn[jj] = 0.f;
        if (!is_v && j < jn && tok_req[j] >= 0) {
          const size_t e = (size_t)tok_pos[j] * half + i;
          cs[jj] = o.cos_t[e];
          sn[jj] = o.sin_t[e];
        }
      }
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        const int j = par + 2 * jj;
        if (j >= jn) break;
        if (tok_req[j] < 0) continue;
        const float x1 = st[j * kStLd + ra], x2 = st[j * kStLd + ra + half];
        const float y1 = x1 * cs[jj] - x2 * sn[jj], y2 = x2 * cs[jj] + x1 * sn[jj];
        const long long drow = layer * o.kv_ls + tok_base[j] + head * o.kv_hs;
        if (!DFLASH_CHECK(drow >= 0 && tok_base[j] + head * o.kv_hs < o.kv_ls &&
                              layer < N / per_layer,
                          err))
          continue;
        __half* dst = (is_v ? o.h2 : o.h1) + (size_t)drow * hd;
        dst[i] = __float2half_rn(y1);
        dst[i + half] = __float2half_rn(y2);
        bad |= narrow_bad<__half>(y1) || narrow_bad<__half>(y2);
      }
    } break;
    default:
      break;
  }
  if (bad) set_error(err, DFLASH_DEV_RANGE);
}

__host__ __device__ inline int tmem_cols_for(int bn) {
  int c = 32;
  while (c < bn) c <<= 1;
  return c;
}

struct Unit {
  int n0, m0, split, kb0, nk, tile;
};

// Stream-K: start of worker c's iteration range, and the worker whose range
// holds iteration g (ranges are [c W / P, (c + 1) W / P), W >= P).
__device__ __forceinline__ long long sk_g0(const GemmArgs& a, int c) {
  return (long long)c * a.sk_W / a.sk_P;
}
__device__ __forceinline__ int sk_worker_of(const GemmArgs& a, long long g) {
  return (int)(((g + 1) * a.sk_P + a.sk_W - 1) / a.sk_W) - 1;
}
// Fixup slot of worker c's piece of the tile starting at iteration tg: each
// worker has at most two pieces that are not whole tiles, its first and last.
__device__ __forceinline__ int sk_slot(const GemmArgs& a, int c, long long tg) {
  return 2 * c + (sk_g0(a, c) >= tg ? 0 : 1);
}

// The work items of one worker in order: split units u = cid, cid + ncl, ...,
// or the stream-K pieces of the worker's range.
struct WorkIter {
  long long g, g1;
  int u;
};
__device__ __forceinline__ WorkIter work_begin(const GemmArgs& a, int cid) {
  WorkIter it;
  it.u = cid;
  it.g = a.sk ? sk_g0(a, cid) : 0;
  it.g1 = a.sk ? sk_g0(a, cid + 1) : 0;
  return it;
}

// Unit u of the CTA with pair rank `rank` (0 outside pairs): its 128 weight
// rows start at n0.
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, int u, int rank) {
  Unit w;
  const int per = a.tiles_n * a.tiles_m;
  w.split = u / per;
  const int rem = u % per;
  w.tile = rem;
  w.m0 = (rem / a.tiles_n) * a.BN;
  w.n0 = (rem % a.tiles_n) * a.tile_rows + rank * kTileN;
  w.kb0 = w.split * a.kb_per_split;
  w.nk = min(a.n_kb, w.kb0 + a.kb_per_split) - w.kb0;
  return w;
}

// Next work item of a worker; false when its work is done.
__device__ __forceinline__ bool work_next(const GemmArgs& a, int ncl, int rank, WorkIter& it,
                                          Unit& w) {
  if (!a.sk) {
    if (it.u >= a.units) return false;
    w = decode_unit(a, it.u, rank);
    it.u += ncl;
    return true;
  }
  if (it.g >= it.g1) return false;
  const int t = (int)(it.g / a.n_kb);
  w.tile = t;
  w.split = 0;
  w.kb0 = (int)(it.g - (long long)t * a.n_kb);
  w.nk = (int)min((long long)(a.n_kb - w.kb0), it.g1 - it.g);
  w.m0 = (t / a.tiles_n) * a.BN;
  w.n0 = (t % a.tiles_n) * a.tile_rows + rank * kTileN;
  it.g += w.nk;
  return true;
}

// Contiguous global -> shared bulk copy completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void st_keep(float* p, float v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kGemmThreads - kEpiWarp0 * 32) : "memory");
}
// AND of `v` over the epilogue warps (named barrier 1)
__device__ __forceinline__ bool epi_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kGemmThreads - kEpiWarp0 * 32)
      : "memory");
  return r != 0;
}

// PAIR: launched as clusters of two CTAs sharing each 256-row weight tile
// (see the CTA-pair notes in common.cuh).  Both CTAs stream their own weight
// rows and half of the token tile; their loads complete on rank 0's `full`
// barriers, rank 0 issues the M = 256 MMAs and its commits release the stages
// and accumulators of both CTAs; both CTAs' epilogue warps hand the
// accumulator back to rank 0.  tmA is then the pre-tiled weight map.
template <int EPI, bool PAIR>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BMaps tmB,
                   const GemmArgs a) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int bn_cta = PAIR ? a.BN / 2 : a.BN;  // token rows this CTA stages per k-block
  const int stage_bytes = kTileN * 128 + bn_cta * 128;
  // [stages][A | B] | epilogue region (LM-head transposes + partials, or the
  // fused-op staging tile + token maps + flag) | barriers
  uint8_t* epi_smem = smem + a.stages * stage_bytes;
  float* lm_tr = reinterpret_cast<float*>(epi_smem);
  LmStat* lm_part = reinterpret_cast<LmStat*>(lm_tr + 4 * kLmTr);
  float* st = reinterpret_cast<float*>(epi_smem);
  int* tok_req = reinterpret_cast<int*>(st + 32 * kStLd);
  int* tok_pos = tok_req + 32;
  long long* tok_base = reinterpret_cast<long long*>(tok_pos + 32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_smem + a.epi_bytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * a.stages + 4);
  volatile uint32_t* sk_flag = tmem_slot + 1;  // stream-K: this piece finishes its tile
  const uint32_t smem0 = smem_u32(smem);
  auto sA = [&](int s) { return smem0 + s * stage_bytes; };
  auto sB = [&](int s) { return smem0 + s * stage_bytes + kTileN * 128; };
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + a.stages + s); };
  auto acc_full = [&](int b) { return smem_u32(bars + 2 * a.stages + b); };
  auto acc_empty = [&](int b) { return smem_u32(bars + 2 * a.stages + 2 + b); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = tmem_cols_for(a.BN);
  // pair rank, and the index / count of the CTAs (or pairs) walking the units
  const int rank = PAIR ? (int)cluster_rank() : 0;
  const int cid = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int ncl = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      // one elected lane per epilogue warp (of both CTAs for a pair)
      mbar_init(acc_empty(b), PAIR ? 8 : 4);
    }
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmA);
  if (warp == kEpiWarp0) {
    if (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), 2 * ncols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), 2 * ncols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (PAIR)
    cluster_sync_all();  // the peer's barriers are initialised before any remote use
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      // k-block i of unit w: the rotated index (each CTA or pair starts its K
      // walk at its own offset so that the SMs do not all request the same
      // activation rows of L2 at the same moment)
      auto kx_of = [&](const Unit& w, int i) {
        // stream-K pieces keep the natural order: the fixup sums pieces in order
        int ki = i + (a.sk ? 0 : (int)((cid * 7u) % (unsigned)w.nk));
        if (ki >= w.nk) ki -= w.nk;
        return (w.kb0 + ki) * kTileK;
      };
      auto expect = [&](int s) {
        if (!PAIR)
          mbar_arrive_expect_tx(full(s), stage_bytes);
        else if (rank == 0)  // rank 0 expects both CTAs' bytes; the peer's may land first
          mbar_arrive_expect_tx(full(s), 2 * stage_bytes);
      };
      auto load_w = [&](int s, const Unit& w, int kx) {
        if (PAIR)  // weight tile n0/128, k-block kx/64 of the tiled image; rows past
                   // the last tile read as zeros
          tma_load_2d_pair(sA(s), &tmA, mapa_shared(full(s), 0), 0,
                           ((w.n0 / kTileN) * a.n_kb + kx / kTileK) * kTileN, pol_w);
        else if (a.a_tiled != nullptr)
          bulk_load(sA(s), a.a_tiled + ((size_t)(w.n0 / kTileN) * a.n_kb + kx / kTileK) * 16384,
                    16384, full(s), pol_w);
        else
          tma_load_2d(sA(s), &tmA, full(s), kx, w.n0, pol_w);
      };
      auto load_x = [&](int s, const Unit& w, int kx) {
        const int seg = kx / a.seg_k;
        if (PAIR)
          tma_load_2d_pair(sB(s), &tmB.m[seg], mapa_shared(full(s), 0), kx - seg * a.seg_k,
                           w.m0 + rank * bn_cta, pol_x);
        else
          tma_load_2d(sB(s), &tmB.m[seg], full(s), kx - seg * a.seg_k, w.m0, pol_x);
      };
      // The weights are never written by another kernel: the first stages of
      // the first unit are requested before the predecessor kernel has
      // finished (their empty barriers are fresh), the activations after it.
      int pre = 0;
      {
        WorkIter wi = work_begin(a, cid);
        Unit w;
        if (work_next(a, ncl, rank, wi, w)) {
          pre = min(a.stages, w.nk);
          for (int i = 0; i < pre; ++i) {
            expect(i);
            load_w(i, w, kx_of(w, i));
          }
        }
      }
      pdl_wait();
      uint32_t it = 0;
      WorkIter wi = work_begin(a, cid);
      Unit w;
      while (ok && work_next(a, ncl, rank, wi, w)) {
        for (int i = 0; i < w.nk; ++i, ++it) {
          const int s = it % a.stages;
          const uint32_t ph = (it / a.stages) & 1;
          const int kx = kx_of(w, i);
          if ((int)it < pre) {  // weights already requested
            load_x(s, w, kx);
            continue;
          }
          if (!mbar_wait(empty(s), ph ^ 1)) { ok = false; break; }
          expect(s);
          load_w(s, w, kx);
          load_x(s, w, kx);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      uint32_t it = 0;
      int j = 0;
      WorkIter wi = work_begin(a, cid);
      Unit w;
      for (; ok && work_next(a, ncl, 0, wi, w); ++j) {
        const int b = j & 1;
        if (!mbar_wait(acc_empty(b), ((j >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + b * ncols;
        for (int i = 0; i < w.nk; ++i, ++it) {
          const int s = it % a.stages;
          const uint32_t ph = (it / a.stages) & 1;
          if (!mbar_wait(full(s), ph)) { ok = false; break; }
          tc_fence_after();
          if (PAIR) {
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk)
              umma_f16_pair(d, smem_desc_sw128(sA(s) + kk * 32), smem_desc_sw128(sB(s) + kk * 32),
                            a.idesc, (i | kk) != 0 ? 1u : 0u);
            umma_commit_pair(empty(s));
            umma_commit_pair(mapa_shared(empty(s), 1));
          } else {
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk)
              umma_f16(d, smem_desc_sw128(sA(s) + kk * 32), smem_desc_sw128(sB(s) + kk * 32),
                       a.idesc, (i | kk) != 0 ? 1u : 0u);
            umma_commit(empty(s));
          }
        }
        if (PAIR) {
          umma_commit_pair(acc_full(b));
          umma_commit_pair(mapa_shared(acc_full(b), 1));
        } else {
          umma_commit(acc_full(b));
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane group of this warp
    const int row = q * 32 + lane;       // weight row inside the tile
    const int nchunk = a.BN / 32;
    pdl_wait();  // the epilogue reads and writes other kernels' buffers
    int j = 0;
    WorkIter wi = work_begin(a, cid);
    Unit w;
    for (; work_next(a, ncl, rank, wi, w); ++j) {
      const int b = j & 1;
      // the second half of a pair's last tile can lie past the weights
      const bool live = w.n0 < a.N;
      bool got = mbar_wait(acc_full(b), (j >> 1) & 1);
      got = epi_bar_and(got);  // the epilogue warps leave together
      __syncwarp();
      if (!got) { ok = false; break; }
      tc_fence_after();
      const uint32_t tb = tmem + b * ncols + ((uint32_t)(q * 32) << 16);
      const int n = w.n0 + row;
      const int et = threadIdx.x - kEpiWarp0 * 32;
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR)
            mbar_arrive_cluster(mapa_shared(acc_empty(b), 0));
          else
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acc_empty(b)) : "memory");
        }
      };
      if (!live) {
        release();
        continue;
      }
      // Stream-K: a piece that is not a whole tile stores its share in its
      // fixup slot ([token][128 rows] fp32) and counts itself on the tile's
      // counter; the last piece to arrive sums every piece's share in worker
      // order (its own from TMEM), so the result does not depend on the order
      // of arrival, and applies the epilogue.  Nobody waits for anybody.
      bool fix = false;
      int c_lo = 0, c_hi = -1;
      long long tg = 0;
      auto slot_ptr = [&](int worker) {
        return a.out.sk_slots +
               ((size_t)sk_slot(a, worker, tg) * (PAIR ? 2 : 1) + rank) * kTileN * a.BN;
      };
      if (a.sk && !(w.kb0 == 0 && w.nk == a.n_kb)) {
        tg = (long long)w.tile * a.n_kb;
        c_lo = sk_worker_of(a, tg);
        c_hi = sk_worker_of(a, tg + a.n_kb - 1);
        float* my = slot_ptr(cid);
        const uint64_t keep = policy_evict_last();
        for (int c = 0; c < nchunk; ++c) {
          if (w.m0 + c * 32 >= a.M) break;  // uniform across the CTA
          float v[32];
          tmem_ld32(tb + c * 32, v);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) st_keep(my + (size_t)(c * 32 + jj) * kTileN + row, v[jj], keep);
        }
        __threadfence();  // this share is visible before the piece is counted
        epi_bar_sync();
        if (et == 0) {
          unsigned* cnt = a.out.sk_cnt + (size_t)w.tile * 2 + rank;
          const bool last = atomicAdd(cnt, 1u) == (unsigned)(c_hi - c_lo);
          if (last) *cnt = 0;  // ready for the next launch
          *sk_flag = last ? 1u : 0u;
        }
        epi_bar_sync();
        if (*sk_flag == 0u) {
          release();
          continue;
        }
        __threadfence();  // every counted share is visible to the reads below
        fix = true;
      }
      // the whole tile's value of chunk c: this piece's accumulator, or (fixup)
      // the shares of every piece in worker order
      auto load_chunk = [&](int c, float (&v)[32]) {
        tmem_ld32(tb + c * 32, v);
        if (!fix) return;
        float acc[32];
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) acc[jj] = 0.f;
        for (int cw = c_lo; cw <= c_hi; ++cw) {
          if (cw == cid) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) acc[jj] += v[jj];
          } else {
            const float* o = slot_ptr(cw) + (size_t)(c * 32) * kTileN + row;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) acc[jj] += __ldcg(o + (size_t)jj * kTileN);
          }
        }
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) v[jj] = acc[jj];
      };
      // token -> (request, cache position) for OP_KV, and the block position's
      // RoPE position for OP_QKV; one thread per token of the chunk
      auto token_maps = [&](int m_base) {
        if (et >= 32) return;
        if (a.out.op == OP_QKV) {
          const int m = m_base + et;
          int pos = 0;
          if (m < a.M) {
            const int r = m / a.out.B;
            pos = (a.out.req_valid[r] ? a.out.ctx_len[r] : 0) + m % a.out.B;
          }
          tok_pos[et] = pos;
          return;
        }
        if (a.out.op != OP_KV) return;
        const int m = m_base + et;
        int req = -1, pos = 0;
        long long base = 0;
        if (m < a.M) {
          const int nrow = a.out.row0 + m;
          int lo = 0, hi = a.out.batch - 1;
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a.out.cu_rows[mid] <= nrow) lo = mid; else hi = mid - 1;
          }
          if (nrow < a.out.cu_rows[lo] || nrow >= a.out.cu_rows[lo + 1]) {
            set_error(a.err, DFLASH_DEV_ROWS);
          } else {
            pos = a.out.start_pos[lo] + (nrow - a.out.cu_rows[lo]);
            const KvPages& pg = a.out.pages;
            if (pg.table != nullptr && !pg.req_ok[lo]) {
              // the page check reported the request: it writes nothing
            } else if (pos < 0 || pos >= a.out.cap || pos >= a.out.max_pos) {
              set_error(a.err, DFLASH_DEV_CTX_CAP);
            } else if (pg.table == nullptr) {
              req = lo;
              base = (long long)lo * a.out.nkv * a.out.cap + pos;
            } else {
              req = lo;
              const int page = pg.table[(long long)lo * pg.max_pages + pos / pg.page];
              base = (long long)page * a.out.nkv * pg.page + pos % pg.page;
            }
          }
        }
        tok_req[et] = req;
        tok_pos[et] = pos;
        tok_base[et] = base;
      };
      if (EPI == EPI_PARTIAL && a.out.op == OP_PARTIAL) {
        // partials are read back right away by the reduction kernel: keep them in L2
        const uint64_t keep = policy_evict_last();
        float* out = a.out.part + (size_t)w.split * a.M * a.N;
        for (int c = 0; c < nchunk; ++c) {
          if (w.m0 + c * 32 >= a.M) break;  // uniform across the CTA
          float v[32];
          tmem_ld32(tb + c * 32, v);
          if (n < a.N) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              const int m = w.m0 + c * 32 + jj;
              if (m < a.M) st_keep(out + (size_t)m * a.N + n, v[jj], keep);
            }
          }
        }
        release();
      } else if (EPI == EPI_PARTIAL && a.splits == 1) {
        // the whole K range is in TMEM (or in the pieces' shares): apply the op
        // chunk by chunk
        for (int c = 0; c < nchunk; ++c) {
          if (w.m0 + c * 32 >= a.M) break;
          float v[32];
          load_chunk(c, v);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) st[jj * kStLd + row] = v[jj];
          token_maps(w.m0 + c * 32);
          epi_bar_sync();
          apply_op(a.out, a.M, a.N, st, tok_req, tok_pos, tok_base, w.m0 + c * 32, w.n0, et,
                   a.err);
          epi_bar_sync();
        }
        release();
      } else {
        float* tr = lm_tr + q * kLmTr;
        for (int c = 0; c < nchunk; ++c) {
          float v[32];
          if (fix && w.m0 + c * 32 >= a.M) {  // no shares stored past the last token
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) v[jj] = 0.f;
          } else {
            load_chunk(c, v);
          }
          // transpose through shared memory: lane jj then owns token column jj
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) tr[jj * 33 + lane] = (n < a.N) ? v[jj] : -INFINITY;
          __syncwarp();
          const float* col = tr + lane * 33;
          if (a.out.dbg != nullptr) {
            // the logits rows: this lane's token, 32 consecutive vocabulary
            // entries (64 or 128 contiguous bytes), one row lookup per lane
            const int m = w.m0 + c * 32 + lane;
            const int n0 = w.n0 + q * 32;
            if (m < a.M) {
              const int64_t d = a.out.dbg_rows ? (int64_t)a.out.dbg_rows[m] : (int64_t)m;
              if (!a.out.dbg_valid || a.out.dbg_valid[d / a.out.B]) {
                const int nv = min(32, a.N - n0);
                if (a.out.dbg_bf16) {
                  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.out.dbg) + d * a.out.dbg_ld + n0;
                  if (nv == 32 && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                      uint4 u;
                      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                      for (int k = 0; k < 4; ++k)
                        h[k] = __floats2bfloat162_rn(col[i + 2 * k], col[i + 2 * k + 1]);
                      *reinterpret_cast<uint4*>(o + i) = u;
                    }
                  } else {
                    for (int i = 0; i < nv; ++i) o[i] = __float2bfloat16_rn(col[i]);
                  }
                } else {
                  float* o = static_cast<float*>(a.out.dbg) + d * a.out.dbg_ld + n0;
                  if (nv == 32 && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                      *reinterpret_cast<float4*>(o + i) =
                          make_float4(col[i], col[i + 1], col[i + 2], col[i + 3]);
                  } else {
                    for (int i = 0; i < nv; ++i) o[i] = col[i];
                  }
                }
              }
            }
          }
          float mx = col[0];
          int bi = 0;
#pragma unroll 8
          for (int i = 1; i < 32; ++i)
            if (col[i] > mx) { mx = col[i]; bi = i; }
          float se = 0.f;
          if (mx != -INFINITY) {
#pragma unroll 8
            for (int i = 0; i < 32; ++i) se += expf(col[i] - mx);
          }
          LmStat st;
          st.max = mx;
          st.idx = a.out.vocab_offset + w.n0 + q * 32 + bi;
          st.sumexp = se;
          st.pad = 0.f;
          lm_part[q * kMaxBN + c * 32 + lane] = st;
          __syncwarp();
        }
        epi_bar_sync();
        // merge the four row groups (ascending vocabulary order) per token column
        for (int col = threadIdx.x - kEpiWarp0 * 32; col < a.BN; col += 128) {
          const int m = w.m0 + col;
          if (m >= a.M) continue;
          LmStat r = lm_part[col];
          for (int g = 1; g < 4; ++g) {
            const LmStat p = lm_part[g * kMaxBN + col];
            if (p.max > r.max) {
              r.sumexp = r.sumexp * expf(r.max - p.max) + p.sumexp;
              r.max = p.max;
              r.idx = p.idx;
            } else {
              r.sumexp += (p.max == -INFINITY) ? 0.f : p.sumexp * expf(p.max - r.max);
            }
          }
          a.out.stats[(size_t)m * a.n_vtiles + w.n0 / kTileN] = r;
        }
        epi_bar_sync();
      }
      if (EPI == EPI_LMHEAD) release();
    }
  }
  if (!ok) set_error(a.err, DFLASH_DEV_TIMEOUT);
  tc_fence_before();
  if (PAIR) {
    // neither CTA leaves while the other may still touch its barriers, shared
    // memory or TMEM
    cluster_sync_all();
    tc_fence_after();
    if (warp == kEpiWarp0) tmem_dealloc_pair(tmem, 2 * ncols);
  } else {
    __syncthreads();
    if (warp == kEpiWarp0) tmem_dealloc(tmem, 2 * ncols);
  }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D 16-bit tensor map (bf16 or fp16): `rows` rows of `cols` elements, row
// stride `ld` elements, box = 64 columns x box_rows rows, 128-byte swizzle,
// zero fill outside.
bool encode_2d(CUtensorMap* m, const void* ptr, int64_t rows, int cols, int ld, int box_rows,
               int elem) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      elem == DFLASH_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool set_tiled_weights(WeightMap& w, const void* tiled) {
  auto enc = get_encode();
  if (!enc || !tiled || (reinterpret_cast<uintptr_t>(tiled) & 15) != 0) return false;
  if (w.elem != DFLASH_BF16 && w.elem != DFLASH_F16) return false;
  // the tiled image viewed as rows of 64 elements (128 bytes): tile t, k-block
  // kb is rows [(t * K/64 + kb) * 128, + 128), already in the swizzled order
  const cuuint64_t rows = (cuuint64_t)((w.N + kTileN - 1) / kTileN) * (w.K / kTileK) * kTileN;
  cuuint64_t dims[2] = {(cuuint64_t)kTileK, rows};
  cuuint64_t strides[1] = {(cuuint64_t)kTileK * 2};
  cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)kTileN};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      w.elem == DFLASH_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(&w.tmap, dt, 2, const_cast<void*>(tiled), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  w.tiled = tiled;
  return true;
}

bool encode_weight_map(WeightMap& w, const void* ptr, int N, int K, int elem) {
  if (elem != DFLASH_BF16 && elem != DFLASH_F16) return false;
  w.ptr = ptr;
  w.N = N;
  w.K = K;
  w.elem = elem;
  return encode_2d(&w.map, ptr, N, K, K, kTileN, elem);
}

int gemm_effective_splits(int K, int splits) {
  const int nkb = K / kTileK;
  if (splits < 1) splits = 1;
  if (splits > nkb) splits = nkb;
  const int per = (nkb + splits - 1) / splits;
  return (nkb + per - 1) / per;
}

int num_sms() {
  static int sms[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (sms[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    sms[dev] = v > 0 ? v : 148;
  }
  return sms[dev];
}

static int g_gemm_mode = 0;
static float g_split_weight = 4.0f;

void gemm_set_mode(int mode) { g_gemm_mode = mode; }
void gemm_set_split_weight(float w) { g_split_weight = w; }

bool gemm_use_pair(int M, int N) {
  if (g_gemm_mode == 1) return false;
  if (g_gemm_mode == 2) return true;
  // a pair halves the token bytes each SM stages and reads per weight byte;
  // measured on B200 it pays for a large token tile against a wide weight
  // (SwiGLU gate/up and LM head at 224-256 tokens), where the coarser 256-row
  // work units still balance across the SM pairs, and for the tensor-bound
  // GEMMs of thousands of token rows (prefill injection: 66% of the sustained
  // bf16 peak with pairs, 63% without)
  return (M > 160 && N >= 16384) || M >= 1024;
}

int gemm_pick_splits(int M, int N, int K, int max_splits) {
  const bool pair = gemm_use_pair(M, N);
  const int rows = pair ? 2 * kTileN : kTileN;
  const int tiles = ((N + rows - 1) / rows) * ((M + kMaxBN - 1) / kMaxBN);
  const int nkb = K / kTileK;
  const int sms = pair ? num_sms() / 2 : num_sms();
  int best = 1;
  double best_score = -1.0;
  // at least 4 k-blocks (256 of K) per split keeps the TMA pipeline busy
  const int smax = std::max(1, std::min(max_splits, nkb / 4));
  for (int s = 1; s <= smax; ++s) {
    const int se = gemm_effective_splits(K, s);
    const int units = tiles * se;
    // persistent CTAs (pairs): the busiest one runs ceil(units / sms) units
    const int per_sm = (units + sms - 1) / sms;
    const double eff = (double)units / ((double)per_sm * sms);
    // each split writes (and its consumer reads) one fp32 partial of the
    // output: M*N*4*2 bytes next to the N*K*2 bytes of weights
    const double score = eff / (1.0 + g_split_weight * se * (double)M / K);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = se;
    }
  }
  return best;
}

// ---------------------------------------------------------------- weight tiling

__global__ void tile_weights_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int N,
                                    int K) {
  // one 16-byte chunk (8 elements) per thread: tile (t, kb), row r, chunk j
  const int nkb = K / kTileK;
  const size_t total = (size_t)((N + kTileN - 1) / kTileN) * nkb * kTileN * 8;
  for (size_t c = (size_t)blockIdx.x * blockDim.x + threadIdx.x; c < total;
       c += (size_t)gridDim.x * blockDim.x) {
    const int j = (int)(c & 7);
    const int r = (int)((c >> 3) & (kTileN - 1));
    const size_t tk = c >> 10;  // tile index t * nkb + kb
    const int kb = (int)(tk % nkb);
    const int t = (int)(tk / nkb);
    const int n = t * kTileN + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < N) v = src[((size_t)n * K + (size_t)kb * kTileK) / 8 + j];
    dst[tk * 1024 + (size_t)r * 8 + (j ^ (r & 7))] = v;
  }
}

size_t tiled_bytes(int N, int K) {
  return (size_t)((N + kTileN - 1) / kTileN) * (K / kTileK) * 16384;
}

void tile_weights(const void* src, void* dst, int N, int K, cudaStream_t s) {
  const size_t chunks = tiled_bytes(N, K) / 16;
  const unsigned blocks = (unsigned)std::min<size_t>((chunks + 255) / 256, 148 * 32);
  tile_weights_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(src),
                                             static_cast<uint4*>(dst), N, K);
}


static int token_tile(int M) {
  if (M >= kMaxBN) return kMaxBN;
  return (M + 31) / 32 * 32;
}

size_t gemm_sk_slot_bytes(int M) {
  // two shares per worker (its first and last pieces), 128 weight rows x the token tile each
  return (size_t)2 * num_sms() * kTileN * token_tile(std::max(M, 1)) * sizeof(float);
}

int gemm_tc(const WeightMap& W, const void* const* xseg, int n_seg, int seg_k, int ld_seg, int M,
            int splits, int epi, const GemmOut& out, int32_t* err, cudaStream_t s) {
  if (M <= 0) return DFLASH_OK;
  if (n_seg < 1 || n_seg > kMaxSeg || seg_k % kTileK != 0 || W.K != n_seg * seg_k)
    return DFLASH_EINVAL;
  const bool sk = splits == 0;
  const int BN = token_tile(M);
  const bool pair = W.tiled != nullptr && gemm_use_pair(M, W.N);
  const int bn_cta = pair ? BN / 2 : BN;
  BMaps maps;
  memset(&maps, 0, sizeof(maps));
  for (int i = 0; i < n_seg; ++i)
    if (!encode_2d(&maps.m[i], xseg[i], M, seg_k, ld_seg, bn_cta, W.elem)) return DFLASH_ECUDA;

  GemmArgs a;
  a.N = W.N;
  a.M = M;
  a.seg_k = seg_k;
  a.BN = BN;
  const int stage_bytes = kTileN * 128 + bn_cta * 128;
  a.n_kb = W.K / kTileK;
  if (epi == EPI_LMHEAD || sk) splits = 1;
  splits = gemm_effective_splits(W.K, splits);
  a.kb_per_split = (a.n_kb + splits - 1) / splits;
  a.tile_rows = pair ? 2 * kTileN : kTileN;
  a.tiles_n = (W.N + a.tile_rows - 1) / a.tile_rows;
  a.tiles_m = (M + BN - 1) / BN;
  a.units = a.tiles_n * a.tiles_m * splits;
  a.splits = splits;
  a.sk = 0;
  a.sk_P = 1;
  a.sk_W = 1;
  if (sk) {
    const long long tiles = (long long)a.tiles_n * a.tiles_m;
    if (!out.sk_slots || !out.sk_cnt || tiles * 2 > out.sk_cnt_cap) return DFLASH_EINVAL;
    a.sk = 1;
    a.sk_W = tiles * a.n_kb;
    const int workers = pair ? num_sms() / 2 : num_sms();
    a.sk_P = (int)std::min<long long>(workers, a.sk_W);
  }
  // fused ops need the whole K range in one unit
  if (epi == EPI_PARTIAL && out.op != OP_PARTIAL && splits > 1) return DFLASH_EINVAL;
  a.n_vtiles = (W.N + kTileN - 1) / kTileN;
  a.idesc = idesc_f16kind(a.tile_rows, BN, W.elem == DFLASH_BF16);
  a.a_tiled = static_cast<const uint8_t*>(W.tiled);
  a.out = out;
  a.err = err;

  // plain partial stores need no epilogue staging: the space goes to stages
  a.epi_bytes = epi == EPI_LMHEAD ? kLmSmem : (out.op == OP_PARTIAL ? 0 : kFusedSmem);
  const size_t fixed = 1024 + a.epi_bytes + 8 * (2 * kMaxStages + 4) + 16;
  const size_t cap = 227 * 1024;
  a.stages = (int)std::min<size_t>(kMaxStages, (cap - fixed) / stage_bytes);
  if (a.stages < 2) return DFLASH_EUNSUPPORTED;
  const size_t smem = fixed + (size_t)a.stages * stage_bytes;
  const int sms = num_sms();
  TimedScope ts(s, epi == EPI_LMHEAD ? TC_LMHEAD : TC_GEMM);
  if (!pair) {
    const int grid = sk ? a.sk_P : std::min(a.units, sms);
    auto k = epi == EPI_PARTIAL ? gemm_tc_kernel<EPI_PARTIAL, false>
                                : gemm_tc_kernel<EPI_LMHEAD, false>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const cudaError_t e =
        launch_pdl(k, dim3(grid), dim3(kGemmThreads), smem, s, 1, W.map, maps, a);
    return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
  }
  auto k =
      epi == EPI_PARTIAL ? gemm_tc_kernel<EPI_PARTIAL, true> : gemm_tc_kernel<EPI_LMHEAD, true>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const cudaError_t e = launch_pdl(k, dim3(2 * (sk ? a.sk_P : std::min(a.units, sms / 2))),
                                   dim3(kGemmThreads), smem, s, 2, W.tmap, maps, a);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace dflash
