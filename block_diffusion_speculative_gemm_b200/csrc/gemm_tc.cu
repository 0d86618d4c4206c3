// tcgen05 weight-streaming GEMM for sm_100a.
//
// Every dense contraction of the draft hot path multiplies a small set of
// token rows X [M, K] (M <= 256 per tile) by a large weight W [N, K]:
// context-feature fc, the layer-batched K/V injection projection, the QKV,
// output and SwiGLU projections, and the LM head.  The CTA tile therefore puts
// 128 weight rows on the UMMA M axis and the token rows on the UMMA N axis
// ("swap-AB"): one weight tile is streamed from HBM exactly once, the token
// tile is re-read from L2.
//
// Structure of one CTA (128 threads, one output tile, one K range):
//   warp 0 lane 0  TMA producer: weight tile [128 x 64] + token tile [BN x 64]
//                  per stage, 128-byte swizzled, completion on a full barrier.
//   warp 1 lane 0  MMA issuer: 4 x tcgen05.mma (K = 16 each) per stage into a
//                  TMEM accumulator of 128 lanes x BN fp32 columns; a
//                  tcgen05.commit per stage releases the stage to the producer.
//   warp 2         allocates and frees the TMEM columns.
//   all warps      epilogue: tcgen05.ld of the accumulator (lane = weight row)
//                  and either a coalesced fp32 partial store (split-K) or the
//                  LM-head reduction (per token: max, argmax, sum of exp).
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
  int n_vtiles;       // LM head: number of 128-row vocabulary tiles
  uint32_t idesc;     // tcgen05 instruction descriptor (operand type, 128 x BN)
  GemmOut out;
  int32_t* err;
};

__host__ __device__ inline int tmem_cols_for(int bn) {
  int c = 32;
  while (c < bn) c <<= 1;
  return c;
}

template <int EPI>
__global__ void __launch_bounds__(128, 2)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BMaps tmB,
                   const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int stage_bytes = kTileN * 128 + a.BN * 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.stages * stage_bytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * a.stages + 1);
  const uint32_t smem0 = smem_u32(smem);
  auto sA = [&](int s) { return smem0 + s * stage_bytes; };
  auto sB = [&](int s) { return smem0 + s * stage_bytes + kTileN * 128; };
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + a.stages + s); };
  const uint32_t accum = smem_u32(bars + 2 * a.stages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kTileN;
  const int m0 = blockIdx.y * a.BN;
  const int split = blockIdx.z;
  const int kb0 = split * a.kb_per_split;
  const int kb1 = min(a.n_kb, kb0 + a.kb_per_split);
  const int nk = kb1 - kb0;
  const uint32_t ncols = tmem_cols_for(a.BN);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(accum, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  if (warp == 0) {
    if (lane == 0 && nk > 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      for (int i = 0; i < nk; ++i) {
        const int s = i % a.stages;
        const uint32_t ph = (i / a.stages) & 1;
        if (!mbar_wait(empty(s), ph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(full(s), stage_bytes);
        const int kx = (kb0 + i) * kTileK;
        tma_load_2d(sA(s), &tmA, full(s), kx, n0, pol_w);
        const int seg = kx / a.seg_k;
        tma_load_2d(sB(s), &tmB.m[seg], full(s), kx - seg * a.seg_k, m0, pol_x);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = a.idesc;
      for (int i = 0; i < nk; ++i) {
        const int s = i % a.stages;
        const uint32_t ph = (i / a.stages) & 1;
        if (!mbar_wait(full(s), ph)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk) {
          umma_f16(tmem, smem_desc_sw128(sA(s) + kk * 32), smem_desc_sw128(sB(s) + kk * 32),
                    idesc, (i | kk) != 0 ? 1u : 0u);
        }
        umma_commit(empty(s));
      }
      umma_commit(accum);
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- epilogue
  const bool acc_ok = (nk > 0) ? mbar_wait(accum, 0) : true;
  __syncwarp();
  tc_fence_after();
  if ((!ok || !acc_ok) && lane == 0) set_error(a.err, DFLASH_DEV_TIMEOUT);

  const int row = warp * 32 + lane;  // TMEM lane = weight row inside the tile
  const int n = n0 + row;
  const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16);
  const int nchunk = a.BN / 32;

  if (EPI == EPI_PARTIAL) {
    float* out = a.out.part + (size_t)split * a.M * a.N;
    for (int c = 0; c < nchunk; ++c) {
      if (m0 + c * 32 >= a.M) break;  // uniform across the CTA
      float v[32];
      if (nk > 0) {
        tmem_ld32(tbase + c * 32, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      if (n < a.N) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int m = m0 + c * 32 + j;
          if (m < a.M) out[(size_t)m * a.N + n] = v[j];
        }
      }
    }
  } else {
    // LM head: stage the tile as [token][weight row] in shared memory, then one
    // thread per token reduces its 128 logits (max, lowest argmax, sum exp).
    float* tile = reinterpret_cast<float*>(smem);  // stages are idle once accum completed
    const int ld = kTileN + 1;
    for (int c = 0; c < nchunk; ++c) {
      float v[32];
      tmem_ld32(tbase + c * 32, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) tile[(c * 32 + j) * ld + row] = (n < a.N) ? v[j] : -INFINITY;
      if (a.out.dbg != nullptr && n < a.N) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int m = m0 + c * 32 + j;
          if (m < a.M)
            a.out.dbg[(a.out.dbg_rows ? (int64_t)a.out.dbg_rows[m] : (int64_t)m) * a.out.dbg_ld + n] = v[j];
        }
      }
    }
    __syncthreads();
    for (int col = threadIdx.x; col < a.BN; col += blockDim.x) {
      const int m = m0 + col;
      if (m >= a.M) continue;
      const float* t = tile + col * ld;
      float mx = t[0];
      int bi = 0;
      for (int i = 1; i < kTileN; ++i) {
        const float x = t[i];
        if (x > mx) { mx = x; bi = i; }
      }
      float se = 0.f;
      for (int i = 0; i < kTileN; ++i) se += expf(t[i] - mx);
      LmStat st;
      st.max = mx;
      st.idx = n0 + bi;
      st.sumexp = se;
      st.pad = 0.f;
      a.out.stats[(size_t)m * a.n_vtiles + blockIdx.x] = st;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) tmem_dealloc(tmem, ncols);
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
  CUresult r = enc(m, dt, 2, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
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

int gemm_pick_splits(int M, int N, int K, int max_splits) {
  const int tiles = ((N + kTileN - 1) / kTileN) * ((M + kMaxBN - 1) / kMaxBN);
  const int nkb = K / kTileK;
  const int sms = 148;
  int best = 1;
  double best_score = -1.0;
  // at least 4 k-blocks (256 of K) per split keeps the TMA pipeline busy
  const int smax = std::max(1, std::min(max_splits, nkb / 4));
  for (int s = 1; s <= smax; ++s) {
    const int se = gemm_effective_splits(K, s);
    const int ctas = tiles * se;
    const int waves = (ctas + sms - 1) / sms;
    const double eff = (double)ctas / (waves * sms);
    // each split writes (and its consumer reads) one fp32 partial of the
    // output: M*N*4*2 bytes next to the N*K*2 bytes of weights
    const double score = eff / (1.0 + 4.0 * se * (double)M / K);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = se;
    }
  }
  return best;
}

static int token_tile(int M) {
  if (M >= kMaxBN) return kMaxBN;
  return (M + 31) / 32 * 32;
}

int gemm_tc(const WeightMap& W, const void* const* xseg, int n_seg, int seg_k, int ld_seg, int M,
            int splits, int epi, const GemmOut& out, int32_t* err, cudaStream_t s) {
  if (M <= 0) return DFLASH_OK;
  if (n_seg < 1 || n_seg > kMaxSeg || seg_k % kTileK != 0 || W.K != n_seg * seg_k)
    return DFLASH_EINVAL;
  const int BN = token_tile(M);
  BMaps maps;
  memset(&maps, 0, sizeof(maps));
  for (int i = 0; i < n_seg; ++i)
    if (!encode_2d(&maps.m[i], xseg[i], M, seg_k, ld_seg, BN, W.elem)) return DFLASH_ECUDA;

  GemmArgs a;
  a.N = W.N;
  a.M = M;
  a.seg_k = seg_k;
  a.BN = BN;
  const int stage_bytes = kTileN * 128 + BN * 128;
  a.n_kb = W.K / kTileK;
  if (epi == EPI_LMHEAD) splits = 1;
  splits = gemm_effective_splits(W.K, splits);
  const long ctas = (long)((W.N + kTileN - 1) / kTileN) * ((M + BN - 1) / BN) * splits;
  // More than one wave: ~100 KB per CTA so that two CTAs share an SM and one's
  // prologue/epilogue overlaps the other's weight stream; otherwise one deep
  // pipeline per SM.
  int budget = ctas > 148 ? 100 * 1024 : 200 * 1024;
  // the LM-head epilogue stages the BN x 128 fp32 tile (padded rows) in the stage buffers
  const int lm_tile = BN * (kTileN + 1) * 4;
  if (epi == EPI_LMHEAD && budget < lm_tile) budget = lm_tile;
  a.stages = (budget + stage_bytes - 1) / stage_bytes;
  if (a.stages > 8) a.stages = 8;
  if (a.stages < 2) a.stages = 2;
  if (epi == EPI_LMHEAD && a.stages * stage_bytes < lm_tile) return DFLASH_EUNSUPPORTED;
  if (a.stages * stage_bytes > 210 * 1024) a.stages = 210 * 1024 / stage_bytes;
  a.kb_per_split = (a.n_kb + splits - 1) / splits;
  a.n_vtiles = (W.N + kTileN - 1) / kTileN;
  a.idesc = idesc_f16kind(kTileN, BN, W.elem == DFLASH_BF16);
  a.out = out;
  a.err = err;

  const size_t smem = (size_t)a.stages * stage_bytes + 1024 + 8 * (2 * a.stages + 2) + 64;
  dim3 grid((W.N + kTileN - 1) / kTileN, (M + BN - 1) / BN, splits);
  TimedScope ts(s, epi == EPI_LMHEAD ? TC_LMHEAD : TC_GEMM);
  if (epi == EPI_PARTIAL) {
    cudaFuncSetAttribute(gemm_tc_kernel<EPI_PARTIAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    gemm_tc_kernel<EPI_PARTIAL><<<grid, 128, smem, s>>>(W.map, maps, a);
  } else {
    cudaFuncSetAttribute(gemm_tc_kernel<EPI_LMHEAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    gemm_tc_kernel<EPI_LMHEAD><<<grid, 128, smem, s>>>(W.map, maps, a);
  }
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace dflash
