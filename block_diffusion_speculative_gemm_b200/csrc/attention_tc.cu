// Tensor-core block-vs-context attention (split-KV partials), fp16 rows over
// an fp16 K/V cache.
//
// A CTA handles (key chunk, kv head, request) with 4 warps.  Context keys of
// the chunk (cache positions below T_r) arrive in 64-key tiles by TMA: per
// tile two 64-column boxes of K and of V (128-byte swizzled), completing on a
// per-stage mbarrier, issued one thread ahead of the consumers through a
// 3-stage ring.  The block's own keys (at most 16) come last, as a small tile
// copied with cp.async into the query area once the query fragments are in
// registers.  Warp (mt, kg) owns query rows [16 mt, 16 mt + 16) and key group
// kg of every tile: S = Q K^T and O += P V run as fp16 mma.sync.m16n8k16 with
// fp32 accumulation; the online softmax (row max m, row sum l) is updated once
// per tile.  Key groups are merged through shared memory and one (m, l, O)
// partial per query row and chunk is written; the last chunk CTA of each
// (request, kv head) -- counted on a per-(request, head) counter that it sets
// back to zero -- merges the chunks into the output rows.
//
// Memory-bound: 4 * B * G flop per cache byte read, every cache byte read once.
#include <algorithm>

#include "attn_combine.cuh"
#include "common.cuh"
#include "internal.h"

namespace dflash {

int g_attn_umma = 0;

namespace {

constexpr int kComputeWarps = 4;
constexpr int kThreads = 32 * kComputeWarps + 32;  // + one producer warp
constexpr int kKeys = 64;    // keys per context tile
constexpr int kMaxChunksTc = 64;  // split-KV chunks per request
constexpr int kBlkKeys = 16; // rows of the block tile

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8, fp32) += A (16x16, fp16, row) * B (16x8, fp16, col)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// A tile of `rows` key rows of HD fp16 is stored as HD/64 column halves; each
// half is [rows][128 bytes] with 16-byte chunk j of row r at chunk j ^ (r & 7)
// (the 128-byte TMA swizzle).  Chunk c of a row (8 elements) is in half c / 8.
__device__ __forceinline__ uint32_t toff(int rows, int row, int c) {
  return (uint32_t)((c >> 3) * rows * 128 + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// Shared memory of one CTA: the TMA stage ring, then the query rows (later
// reused for the block tile), then the stage barriers (full, then empty).
// Sized so that two CTAs fit on an SM: 3 stages for up to 32 query rows, 2
// stages for 64.
template <int HD, int MT>
struct Layout {
  static constexpr int kStages = MT <= 2 ? 3 : 2;
  static constexpr int kTile = kKeys * HD * 2;       // K or V of one context tile
  static constexpr int kStage = 2 * kTile;
  static constexpr int kQRows = MT * 16;
  static constexpr int kQ = (kQRows > 2 * kBlkKeys ? kQRows : 2 * kBlkKeys) * HD * 2;
  static constexpr int kBars = 2 * kStages * 8;
  static constexpr int kSmem = kStages * kStage + kQ + kBars + 1024;  // + alignment slack
  static_assert(2 * kBlkKeys * HD * 2 <= kQ, "block tile fits the query area");
};

template <int HD, int MT>
struct Warp {
  static constexpr int KG = MT == 1 ? 4 : (MT == 2 ? 2 : 1);  // key groups
  static constexpr int KPW = kKeys / KG;                      // keys per warp per tile
  static constexpr int NT = HD / 8;
  static constexpr int KS = HD / 16;
};

// Byte offsets of this lane's ldmatrix rows inside a swizzled tile: every row
// a lane addresses has row & 7 == lane & 7, so the swizzle term of 16-byte
// chunk j is (j ^ (lane & 7)) << 4.  K fragments (non-transposed) take chunk
// 2 q + (mi & 1) of column half q / 4; V fragments (transposed) take chunk
// 2 q + (mi >> 1).
struct LdsmOff {
  uint32_t rk, rv;        // row offset of the lane's K / V row inside a 16-row group
  uint32_t xk[4], xv[4];  // swizzled chunk offsets for q = 0..3
};
__device__ __forceinline__ LdsmOff ldsm_offsets(int lane) {
  const int mi = lane >> 3, li = lane & 7;
  LdsmOff o;
  o.rk = (uint32_t)(((mi >> 1) * 8 + li) * 128);
  o.rv = (uint32_t)(((mi & 1) * 8 + li) * 128);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    o.xk[q] = (uint32_t)(((2 * q + (mi & 1)) ^ li) << 4);
    o.xv[q] = (uint32_t)(((2 * q + (mi >> 1)) ^ li) << 4);
  }
  return o;
}

// One tile's worth of keys for one warp: keys [kbeg, kbeg + NKEYS) of a tile
// stored with `rows` rows; keys at tile-local index >= nvalid are masked.
// The running row maxima m0/m1 are kept in log2 units of the scaled score
// (score * sl2, sl2 = log2(e) / sqrt(hd)), so that every exponential is one
// FMA and one exp2.
template <int HD, int NKEYS>
__device__ __forceinline__ void attend(uint32_t sK, uint32_t sV, int rows, int kbeg, int nvalid,
                                       const uint32_t (&qa)[HD / 16][4], float (&o)[HD / 8][4],
                                       float& m0, float& m1, float& l0, float& l1, float sl2,
                                       const LdsmOff& lo, int lane) {
  constexpr int NS = NKEYS / 8;
  const int tq = lane & 3;
  float s[NS][4];
#pragma unroll
  for (int n = 0; n < NS; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < HD / 16; ++ks) {
#pragma unroll
    for (int np = 0; np < NKEYS / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sK + (ks >> 2) * rows * 128 + (kbeg + np * 16) * 128 + lo.rk + lo.xk[ks & 3], b0,
              b1, b2, b3);
      mma16816(s[2 * np], qa[ks], b0, b1);
      mma16816(s[2 * np + 1], qa[ks], b2, b3);
    }
  }
  if (kbeg + NKEYS > nvalid) {  // keys past the context in this warp's range
#pragma unroll
    for (int n = 0; n < NS; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (kbeg + n * 8 + 2 * tq + (e & 1) >= nvalid) s[n][e] = -INFINITY;
  }
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int n = 0; n < NS; ++n) {
    mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
    mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float n0 = fmaxf(m0, mx0 * sl2), n1 = fmaxf(m1, mx1 * sl2);
  // every key masked (the same for all rows): nothing to add
  if (kbeg + NKEYS > nvalid && __all_sync(0xffffffffu, n0 == -INFINITY && n1 == -INFINITY))
    return;
  const float c0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - n0);
  const float c1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - n1);
  float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
  for (int n = 0; n < NS; ++n) {
    // a masked score is -inf and gives exp2(-inf) = 0 (n0, n1 are finite here)
    s[n][0] = exp2f(fmaf(s[n][0], sl2, -n0));
    s[n][1] = exp2f(fmaf(s[n][1], sl2, -n0));
    s[n][2] = exp2f(fmaf(s[n][2], sl2, -n1));
    s[n][3] = exp2f(fmaf(s[n][3], sl2, -n1));
    ps0 += s[n][0] + s[n][1];
    ps1 += s[n][2] + s[n][3];
  }
  l0 = l0 * c0 + ps0;
  l1 = l1 * c1 + ps1;
  // the output only needs rescaling when some row's maximum moved
  if (__any_sync(0xffffffffu, n0 != m0 || n1 != m1)) {
#pragma unroll
    for (int n = 0; n < HD / 8; ++n) {
      o[n][0] *= c0;
      o[n][1] *= c0;
      o[n][2] *= c1;
      o[n][3] *= c1;
    }
  }
  m0 = n0;
  m1 = n1;
#pragma unroll
  for (int kb = 0; kb < NKEYS / 16; ++kb) {
    const uint32_t pa[4] = {pack_h2(s[2 * kb][0], s[2 * kb][1]),
                            pack_h2(s[2 * kb][2], s[2 * kb][3]),
                            pack_h2(s[2 * kb + 1][0], s[2 * kb + 1][1]),
                            pack_h2(s[2 * kb + 1][2], s[2 * kb + 1][3])};
#pragma unroll
    for (int nd = 0; nd < HD / 8; nd += 2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sV + (nd >> 3) * rows * 128 + (kbeg + kb * 16) * 128 + lo.rv +
                    lo.xv[(nd & 7) >> 1],
                b0, b1, b2, b3);
      mma16816(o[nd], pa, b0, b1);
      mma16816(o[nd + 1], pa, b2, b3);
    }
  }
}

// Warps 0-3 compute (warp (mt, kg) = (warp % MT, warp / MT)); warp 4 lane 0
// streams the context tiles: it refills a stage once the four compute warps
// have released it on the stage's `empty` barrier, so the warps never wait
// for one another inside the tile loop.
template <int HD, int MT>
__global__ void __launch_bounds__(kThreads)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __half* __restrict__ q, const __half* __restrict__ kb,
                   const __half* __restrict__ vb, const KvPages pg, long long kv_rows, int layer,
                   int batch, int cap,
                   const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ req_valid,
                   int B, int nq, int nkv, int chunk_host, const int32_t* plan_dev, int n_chunks,
                   float* __restrict__ part_o, float* __restrict__ part_ml,
                   unsigned* __restrict__ cnt, __half* __restrict__ out, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  // A planned forward runs a 1-D grid over the planning kernel's work list
  // ({chunk, items, -, -, then per item: request << 16 | kv head << 8 |
  // chunk index and the request's context length}, in the 3-D grid's order);
  // CTAs past the list exit.  Otherwise the grid is (chunk, kv head, request)
  // with the host's chunk.
  int c = blockIdx.x, g = blockIdx.y, r = blockIdx.z, chunk = chunk_host, Tc;
  if (plan_dev != nullptr) {
    const int n_items = plan_dev[1];
    const int2 it = reinterpret_cast<const int2*>(plan_dev)[2 + blockIdx.x];
    chunk = plan_dev[0];
    if ((int)blockIdx.x >= n_items) return;
    r = it.x >> 16;
    g = (it.x >> 8) & 255;
    c = it.x & 255;
    Tc = it.y;
  } else {
    Tc = req_valid[r] ? ctx_len[r] : 0;
  }
  using LY = Layout<HD, MT>;
  using WP = Warp<HD, MT>;
  constexpr int kStages = LY::kStages;
  constexpr int NT = WP::NT, KS = WP::KS, KG = WP::KG, KPW = WP::KPW;
  constexpr int HALVES = HD / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base + kStages * LY::kStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * LY::kStage + LY::kQ);
  auto full = [&](int st) { return smem_u32(bars + st); };
  auto empty = [&](int st) { return smem_u32(bars + kStages + st); };

  const int G = nq / nkv;
  const int R = B * G;
  const int k0 = c * chunk;
  if (k0 >= Tc + B) return;
  const int k1 = min(Tc + B, k0 + chunk);
  const int kc_end = min(k1, Tc);                       // context keys [k0, kc_end)
  const int nt = kc_end > k0 ? (kc_end - k0 + kKeys - 1) / kKeys : 0;
  const int kb_lo = max(k0, Tc), kb_hi = min(k1, Tc + B);  // block keys [kb_lo, kb_hi)
  const int row_base = pg.table == nullptr ? ((layer * batch + r) * nkv + g) * cap : 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt = warp % MT, kg = warp / MT;
  const bool computes = warp < kComputeWarps;

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), kComputeWarps);
    }
    fence_barrier_init();
  }
  // query rows of this kv head: row i = (block position i / G, head g*G + i % G)
  for (int idx = tid; idx < MT * 16 * (HD / 8); idx += kThreads) {
    const int row = idx / (HD / 8), ch = idx % (HD / 8);
    const void* src = q;
    int bytes = 0;
    if (row < R) {
      src = q + ((size_t)(r * B + row / G) * nq + g * G + row % G) * HD + ch * 8;
      bytes = 16;
    }
    cp_async16(s_q + toff(LY::kQRows, row, ch), src, bytes);
  }
  cp_async_commit();
  __syncthreads();  // barrier init visible before any wait

  auto issue = [&](int t) {  // one thread: TMA of context tile t into its stage
    const int st = t % kStages;
    const uint32_t sK = s_base + st * LY::kStage, sV = sK + LY::kTile;
    mbar_arrive_expect_tx(full(st), 2 * LY::kTile);
    // the tile's first key position; a paged store finds its row through the
    // request's page table (a tile never crosses a page)
    const int p0 = k0 + t * kKeys;
    int y = pg.table == nullptr ? row_base + p0
                                : (int)kv_row(pg, layer, batch, r, nkv, g, cap, p0);
    if (!DFLASH_CHECK(y >= 0 && y < kv_rows, err)) y = 0;  // a tile inside the store
#pragma unroll
    for (int h = 0; h < HALVES; ++h) {
      tma_load_2d(sK + h * kKeys * 128, &tmK, full(st), h * 64, y, policy_evict_first());
      tma_load_2d(sV + h * kKeys * 128, &tmV, full(st), h * 64, y, policy_evict_first());
    }
  };
  const bool producer = warp == kComputeWarps && lane == 0;
  if (producer)
    for (int t = 0; t < kStages && t < nt; ++t) issue(t);  // fresh stages

  uint32_t qa[KS][4];
  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = rsqrtf((float)HD) * 1.4426950408889634f;  // log2(e) / sqrt(hd)
  const int mi = lane >> 3, li = lane & 7;
  const LdsmOff lo = ldsm_offsets(lane);

  cp_async_wait_all();
  __syncthreads();
  if (computes) {
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int row = mt * 16 + (mi & 1) * 8 + li;
      ldsm_x4(s_q + toff(LY::kQRows, row, ks * 2 + (mi >> 1)), qa[ks][0], qa[ks][1], qa[ks][2],
              qa[ks][3]);
    }
  }
  __syncthreads();  // the query area now holds the block tile
  const bool has_blk = kb_hi > kb_lo;
  if (has_blk) {
    for (int idx = tid; idx < 2 * kBlkKeys * (HD / 8); idx += kThreads) {
      const int mat = idx / (kBlkKeys * (HD / 8));
      const int rem = idx % (kBlkKeys * (HD / 8));
      const int row = rem / (HD / 8), ch = rem % (HD / 8);
      const int key = kb_lo + row;
      const void* src = kb;
      int bytes = 0;
      if (key < kb_hi) {
        src = (mat ? vb : kb) + ((size_t)(r * B + key - Tc) * nkv + g) * HD + ch * 8;
        bytes = 16;
      }
      cp_async16(s_q + mat * (kBlkKeys * HD * 2) + toff(kBlkKeys, row, ch), src, bytes);
    }
    cp_async_commit();
  }

  bool ok = true;
  if (producer) {
    for (int t = kStages; t < nt; ++t) {
      const int st = t % kStages;
      if (!mbar_wait(empty(st), ((t / kStages) + 1) & 1)) { ok = false; break; }
      issue(t);
    }
  } else if (computes) {
    for (int t = 0; t < nt; ++t) {
      const int st = t % kStages;
      if (!mbar_wait(full(st), (t / kStages) & 1)) ok = false;
      const int nvalid = min(kKeys, kc_end - (k0 + t * kKeys));
      const uint32_t sK = s_base + st * LY::kStage, sV = sK + LY::kTile;
      const int kbeg = kg * KPW;
      if (nvalid < kbeg + KPW) {
        // rows past the context hold other cache positions: zero this warp's V
        // rows there so that masked keys contribute exactly nothing (the other
        // warp of the same key group writes the same zeros)
        uint8_t* v = smem + st * LY::kStage + LY::kTile;
        const int z0 = max(nvalid, kbeg);
        for (int idx = lane; idx < (kbeg + KPW - z0) * (HD / 8); idx += 32) {
          const int row = z0 + idx / (HD / 8), ch = idx % (HD / 8);
          *reinterpret_cast<uint4*>(v + toff(kKeys, row, ch)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();  // before the stage goes back to the TMA
        __syncwarp();
      }
      attend<HD, KPW>(sK, sV, kKeys, kbeg, nvalid, qa, o, m0, m1, l0, l1, sl2, lo, lane);
      __syncwarp();
      if (lane == 0)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty(st)) : "memory");
    }
  }
  if (!ok) set_error(err, DFLASH_DEV_TIMEOUT);
  if (has_blk) {
    cp_async_wait_all();
    __syncthreads();
    if (computes && kg == 0)
      attend<HD, kBlkKeys>(s_q, s_q + kBlkKeys * HD * 2, kBlkKeys, 0, kb_hi - kb_lo, qa, o, m0, m1,
                           l0, l1, sl2, lo, lane);
  }

  // row sums over the quad, then merge the key groups of each row tile
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  constexpr int kSlot = NT * 4 + 4;
  static_assert(4 * 32 * kSlot * 4 <= kStages * LY::kStage, "merge scratch");
  float* scratch = reinterpret_cast<float*>(smem);
  __syncthreads();  // every tile consumed: the stage ring becomes merge scratch
  if (KG > 1 && computes && kg > 0) {
    float* sl = scratch + ((size_t)warp * 32 + lane) * kSlot;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sl[n * 4 + e] = o[n][e];
    sl[NT * 4 + 0] = m0;
    sl[NT * 4 + 1] = m1;
    sl[NT * 4 + 2] = l0;
    sl[NT * 4 + 3] = l1;
  }
  __syncthreads();
  const size_t pbase = (((size_t)r * nkv + g) * n_chunks + c) * kAttnMaxRows;
  if (computes && kg == 0) {
#pragma unroll
    for (int k = 1; k < KG; ++k) {
      const float* sl = scratch + ((size_t)(k * MT + mt) * 32 + lane) * kSlot;
      const float pm0 = sl[NT * 4 + 0], pm1 = sl[NT * 4 + 1];
      const float nm0 = fmaxf(m0, pm0), nm1 = fmaxf(m1, pm1);
      const float a0 = m0 == -INFINITY ? 0.f : exp2f(m0 - nm0);
      const float a1 = m1 == -INFINITY ? 0.f : exp2f(m1 - nm1);
      const float b0 = pm0 == -INFINITY ? 0.f : exp2f(pm0 - nm0);
      const float b1 = pm1 == -INFINITY ? 0.f : exp2f(pm1 - nm1);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] = o[n][0] * a0 + sl[n * 4 + 0] * b0;
        o[n][1] = o[n][1] * a0 + sl[n * 4 + 1] * b0;
        o[n][2] = o[n][2] * a1 + sl[n * 4 + 2] * b1;
        o[n][3] = o[n][3] * a1 + sl[n * 4 + 3] * b1;
      }
      l0 = l0 * a0 + sl[NT * 4 + 2] * b0;
      l1 = l1 * a1 + sl[NT * 4 + 3] * b1;
      m0 = nm0;
      m1 = nm1;
    }
    // partial maxima leave in natural-log units of the scaled score
    const float ln2 = 0.6931471805599453f;
    m0 *= ln2;
    m1 *= ln2;
    const int tq = lane & 3;
    const int row0 = mt * 16 + (lane >> 2), row1 = row0 + 8;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int col = n * 8 + 2 * tq;
      if (row0 < R)
        *reinterpret_cast<float2*>(part_o + (pbase + row0) * HD + col) =
            make_float2(o[n][0], o[n][1]);
      if (row1 < R)
        *reinterpret_cast<float2*>(part_o + (pbase + row1) * HD + col) =
            make_float2(o[n][2], o[n][3]);
    }
    if (tq == 0) {
      if (row0 < R) *reinterpret_cast<float2*>(part_ml + (pbase + row0) * 2) = make_float2(m0, l0);
      if (row1 < R) *reinterpret_cast<float2*>(part_ml + (pbase + row1) * 2) = make_float2(m1, l1);
    }
    __threadfence();  // this chunk's partial is visible before the chunk is counted
  }

  // ---- chunk combine: the last chunk CTA of (request, kv head) merges every
  // chunk's (m, l, O) into the output rows
  static_assert(2 * kMaxChunksTc * kAttnMaxRows * 4 <= kStages * LY::kStage, "combine scratch");
  attn_chunk_combine<HD, kThreads>(reinterpret_cast<float*>(smem), r, g, R, B, G, nq, nkv, Tc,
                                   chunk, n_chunks, part_o, part_ml, cnt, out);
}

// ---------------------------------------------------------------- persistent schedule
// Segment s = r * nkv + g (request r, kv head g) holds units 0 .. n_s - 1: its
// ceil(T_r / 64) context tiles, then one unit for the block's own keys.
// seg_start[s] = units before segment s, seg_start[S] = W.  CTA c of the P
// CTAs with work takes units [c W / P, (c + 1) W / P): every CTA streams the
// same number of tiles through one TMA ring that runs on across segments, and
// sets up once.  A piece (the units of one segment inside one CTA's range)
// publishes one (m, l, O) partial per warp; the piece that counts itself last
// on the segment's counter merges every piece's partials, CTAs in order, into
// the output rows and sets the counter back to zero.

// One CTA of 1024 threads: exclusive scan of the segments' unit counts.
__global__ void __launch_bounds__(1024)
    attn_plan_kernel(const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ req_valid,
                     int batch, int nkv, int32_t* __restrict__ seg_start) {
  pdl_trigger();
  pdl_wait();
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int S = batch * nkv;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + threadIdx.x;
    int n = 0;
    if (s < S) {
      const int r = s / nkv;
      const int T = req_valid[r] ? ctx_len[r] : 0;
      n = (T + kKeys - 1) / kKeys + 1;
    }
    int x = n;  // inclusive scan inside the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
      int t = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    const int excl = carry + (w > 0 ? warp_tot[w - 1] : 0) + x - n;
    if (s < S) seg_start[s] = excl;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = excl + n;
    __syncthreads();
  }
  if (threadIdx.x == 0) seg_start[S] = carry;
}

// named barrier 1 among the 128 threads of the compute warps
__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int HD, int MT>
__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_persistent(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __half* __restrict__ q,
                       const __half* __restrict__ kb, const __half* __restrict__ vb,
                       const KvPages pg, long long kv_rows, int layer, int batch, int cap,
                       const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ req_valid,
                       int B, int nq, int nkv, const int32_t* __restrict__ seg_start,
                       float* __restrict__ part_o, float* __restrict__ part_ml,
                       unsigned* __restrict__ cnt, __half* __restrict__ out, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  using LY = Layout<HD, MT>;
  using WP = Warp<HD, MT>;
  constexpr int kStages = LY::kStages;
  constexpr int NT = WP::NT, KS = WP::KS, KG = WP::KG, KPW = WP::KPW;
  constexpr int HALVES = HD / 64;
  constexpr int kRows = MT * 16;           // rows of one warp partial
  constexpr int kAcc = (kRows * HD / 4 + 127) / 128;  // float4 outputs per thread in a merge
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base + kStages * LY::kStage;
  float* scratch = reinterpret_cast<float*>(smem + kStages * LY::kStage);  // the query area
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * LY::kStage + LY::kQ);
  auto full = [&](int st) { return smem_u32(bars + st); };
  auto empty = [&](int st) { return smem_u32(bars + kStages + st); };
  __shared__ int s_last;

  const int S = batch * nkv;
  const long long W = seg_start[S];
  const int P = (int)min((long long)gridDim.x, W);
  const int c = blockIdx.x;
  if (c >= P) return;  // the whole CTA, before any barrier is initialised
  const long long g0 = (long long)c * W / P, g1 = (long long)(c + 1) * W / P;
  const int G = nq / nkv;
  const int R = B * G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt = warp % MT, kg = warp / MT;

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), kComputeWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();  // the last block-wide barrier: the producer warp runs on alone

  // segment of unit gq: the last s with seg_start[s] <= gq
  auto seg_of = [&](long long gq) {
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (seg_start[mid] <= gq) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  auto ctx_of = [&](int r) { return req_valid[r] ? ctx_len[r] : 0; };

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int it = 0;
      for (long long gq = g0; gq < g1 && ok;) {
        const int sg = seg_of(gq);
        const long long st0 = seg_start[sg], en = seg_start[sg + 1];
        const int a = (int)(gq - st0), b = (int)(min(en, g1) - st0);
        const int r = sg / nkv, gh = sg % nkv;
        const int nctx = (ctx_of(r) + kKeys - 1) / kKeys;
        const int row_base = pg.table == nullptr ? ((layer * batch + r) * nkv + gh) * cap : 0;
        for (int t = a; t < min(b, nctx); ++t, ++it) {
          const int stg = it % kStages;
          if (it >= kStages && !mbar_wait(empty(stg), ((it / kStages) + 1) & 1)) {
            ok = false;
            break;
          }
          const uint32_t sK = s_base + stg * LY::kStage, sV = sK + LY::kTile;
          mbar_arrive_expect_tx(full(stg), 2 * LY::kTile);
          const int p0 = t * kKeys;
          int y = pg.table == nullptr ? row_base + p0
                                      : (int)kv_row(pg, layer, batch, r, nkv, gh, cap, p0);
          if (!DFLASH_CHECK(y >= 0 && y < kv_rows, err)) y = 0;
#pragma unroll
          for (int h = 0; h < HALVES; ++h) {
            tma_load_2d(sK + h * kKeys * 128, &tmK, full(stg), h * 64, y, policy_evict_first());
            tma_load_2d(sV + h * kKeys * 128, &tmV, full(stg), h * 64, y, policy_evict_first());
          }
        }
        gq = st0 + b;
      }
      if (!ok) set_error(err, DFLASH_DEV_TIMEOUT);
    }
    return;
  }

  // -------------------------------------------------------------- compute warps
  const float sl2 = rsqrtf((float)HD) * 1.4426950408889634f;  // log2(e) / sqrt(hd)
  const int mi = lane >> 3, li = lane & 7;
  const LdsmOff lo = ldsm_offsets(lane);
  bool ok = true;
  int it = 0;
  for (long long gq = g0; gq < g1;) {
    const int sg = seg_of(gq);
    const long long st0 = seg_start[sg], en = seg_start[sg + 1];
    const int a = (int)(gq - st0), b = (int)(min(en, g1) - st0);
    const int r = sg / nkv, gh = sg % nkv;
    const int Tc = ctx_of(r);
    const int nctx = (Tc + kKeys - 1) / kKeys;
    const bool has_blk = b == (int)(en - st0);  // the segment's last unit: the block's keys

    // query rows of this (request, kv head): row i = (position i / G, head gh*G + i % G)
    for (int idx = tid; idx < kRows * (HD / 8); idx += 128) {
      const int row = idx / (HD / 8), ch = idx % (HD / 8);
      const void* src = q;
      int bytes = 0;
      if (row < R) {
        src = q + ((size_t)(r * B + row / G) * nq + gh * G + row % G) * HD + ch * 8;
        bytes = 16;
      }
      cp_async16(s_q + toff(LY::kQRows, row, ch), src, bytes);
    }
    cp_async_commit();
    cp_async_wait_all();
    compute_bar();
    uint32_t qa[KS][4];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int row = mt * 16 + (mi & 1) * 8 + li;
      ldsm_x4(s_q + toff(LY::kQRows, row, ks * 2 + (mi >> 1)), qa[ks][0], qa[ks][1], qa[ks][2],
              qa[ks][3]);
    }
    compute_bar();  // the query area now takes the block tile
    if (has_blk) {
      for (int idx = tid; idx < 2 * kBlkKeys * (HD / 8); idx += 128) {
        const int mat = idx / (kBlkKeys * (HD / 8));
        const int rem = idx % (kBlkKeys * (HD / 8));
        const int row = rem / (HD / 8), ch = rem % (HD / 8);
        const void* src = kb;
        int bytes = 0;
        if (row < B) {
          src = (mat ? vb : kb) + ((size_t)(r * B + row) * nkv + gh) * HD + ch * 8;
          bytes = 16;
        }
        cp_async16(s_q + mat * (kBlkKeys * HD * 2) + toff(kBlkKeys, row, ch), src, bytes);
      }
      cp_async_commit();
    }

    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    for (int t = a; t < min(b, nctx); ++t, ++it) {
      const int stg = it % kStages;
      if (!mbar_wait(full(stg), (it / kStages) & 1)) ok = false;
      const int nvalid = min(kKeys, Tc - t * kKeys);
      const uint32_t sK = s_base + stg * LY::kStage, sV = sK + LY::kTile;
      const int kbeg = kg * KPW;
      if (nvalid < kbeg + KPW) {
        // rows past the context hold other positions: zero this warp's V rows
        // there so that masked keys contribute exactly nothing
        uint8_t* v = smem + stg * LY::kStage + LY::kTile;
        const int z0 = max(nvalid, kbeg);
        for (int idx = lane; idx < (kbeg + KPW - z0) * (HD / 8); idx += 32) {
          const int row = z0 + idx / (HD / 8), ch = idx % (HD / 8);
          *reinterpret_cast<uint4*>(v + toff(kKeys, row, ch)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();  // before the stage goes back to the TMA
        __syncwarp();
      }
      attend<HD, KPW>(sK, sV, kKeys, kbeg, nvalid, qa, o, m0, m1, l0, l1, sl2, lo, lane);
      __syncwarp();
      if (lane == 0)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty(stg)) : "memory");
    }
    if (has_blk) {
      cp_async_wait_all();
      compute_bar();
      if (kg == 0)
        attend<HD, kBlkKeys>(s_q, s_q + kBlkKeys * HD * 2, kBlkKeys, 0, B, qa, o, m0, m1, l0, l1,
                             sl2, lo, lane);
    }

    // this warp's partial: slot (c + sg) * KG + kg, rows of its row tile
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    {
      const float ln2 = 0.6931471805599453f;  // partial maxima in natural-log units
      const size_t pbase = ((size_t)(c + sg) * KG + kg) * kRows;
      const int tq = lane & 3;
      const int row0 = mt * 16 + (lane >> 2), row1 = row0 + 8;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int col = n * 8 + 2 * tq;
        if (row0 < R)
          *reinterpret_cast<float2*>(part_o + (pbase + row0) * HD + col) =
              make_float2(o[n][0], o[n][1]);
        if (row1 < R)
          *reinterpret_cast<float2*>(part_o + (pbase + row1) * HD + col) =
              make_float2(o[n][2], o[n][3]);
      }
      if (tq == 0) {
        if (row0 < R)
          *reinterpret_cast<float2*>(part_ml + (pbase + row0) * 2) = make_float2(m0 * ln2, l0);
        if (row1 < R)
          *reinterpret_cast<float2*>(part_ml + (pbase + row1) * 2) = make_float2(m1 * ln2, l1);
      }
    }
    __threadfence();  // this piece's partials are visible before it is counted
    compute_bar();
    // pieces of this segment: the CTAs whose ranges meet it
    const int c_lo = (int)(((st0 + 1) * P + W - 1) / W) - 1;
    const int c_hi = (int)((en * P + W - 1) / W) - 1;
    if (tid == 0) {
      const bool last = atomicAdd(&cnt[sg], 1u) == (unsigned)(c_hi - c_lo);
      if (last) cnt[sg] = 0;  // ready for the next launch
      s_last = last ? 1 : 0;
    }
    compute_bar();
    if (s_last) {
      __threadfence();  // every counted partial is visible to the reads below
      // merge: weights exp(m - M) / L per (partial, row), CTAs in order
      const int NP = (c_hi - c_lo + 1) * KG;
      auto slot_of = [&](int e) { return (size_t)(c_lo + e / KG + sg) * KG + e % KG; };
      float* sM = scratch;
      float* sIL = scratch + kRows;
      float* sw = scratch + 2 * kRows;
      const int CH = (LY::kQ / 4 - 2 * kRows) / kRows;  // partials per weight chunk
      if (tid < R) {
        float M = -INFINITY, L = 0.f;
        for (int e = 0; e < NP; ++e) {
          const float2 ml =
              __ldcg(reinterpret_cast<const float2*>(part_ml + (slot_of(e) * kRows + tid) * 2));
          if (ml.x == -INFINITY) continue;
          if (ml.x > M) {
            L = (M == -INFINITY ? 0.f : L * expf(M - ml.x)) + ml.y;
            M = ml.x;
          } else {
            L += ml.y * expf(ml.x - M);
          }
        }
        sM[tid] = M;
        sIL[tid] = L > 0.f ? 1.f / L : 0.f;
      }
      compute_bar();
      float4 acc[kAcc];
#pragma unroll
      for (int k = 0; k < kAcc; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int e0 = 0; e0 < NP; e0 += CH) {
        const int ne = min(CH, NP - e0);
        for (int idx = tid; idx < ne * kRows; idx += 128) {
          const int e = e0 + idx / kRows, row = idx % kRows;
          float wgt = 0.f;
          if (row < R) {
            const float mm = __ldcg(part_ml + (slot_of(e) * kRows + row) * 2);
            wgt = mm == -INFINITY ? 0.f : expf(mm - sM[row]) * sIL[row];
          }
          sw[idx] = wgt;
        }
        compute_bar();
#pragma unroll
        for (int k = 0; k < kAcc; ++k) {
          const int i4 = tid + k * 128;
          if (i4 >= R * HD / 4) break;
          const int row = (i4 * 4) / HD, col = (i4 * 4) % HD;
          for (int e = e0; e < e0 + ne; ++e) {
            const float wgt = sw[(e - e0) * kRows + row];
            const float4 v =
                __ldcg(reinterpret_cast<const float4*>(part_o + (slot_of(e) * kRows + row) * HD + col));
            acc[k].x += wgt * v.x;
            acc[k].y += wgt * v.y;
            acc[k].z += wgt * v.z;
            acc[k].w += wgt * v.w;
          }
        }
        compute_bar();
      }
#pragma unroll
      for (int k = 0; k < kAcc; ++k) {
        const int i4 = tid + k * 128;
        if (i4 >= R * HD / 4) break;
        const int row = (i4 * 4) / HD, col = (i4 * 4) % HD;
        __half* dst = out + ((size_t)(r * B + row / G) * nq + gh * G + row % G) * HD + col;
        *reinterpret_cast<__half2*>(dst) = __floats2half2_rn(acc[k].x, acc[k].y);
        *reinterpret_cast<__half2*>(dst + 2) = __floats2half2_rn(acc[k].z, acc[k].w);
      }
    }
    compute_bar();  // the query area is free for the next piece
    gq = st0 + b;
  }
  if (!ok) set_error(err, DFLASH_DEV_TIMEOUT);
}

template <int HD, int MT>
int launch_persistent(const CUtensorMap& tk, const CUtensorMap& tv, const __half* q,
                      const __half* kb, const __half* vb, const KvPages& pg, long long kv_rows,
                      int layer, int batch, int cap, const int32_t* ctx_len,
                      const int32_t* req_valid, int B, int nq, int nkv, const int32_t* seg_start,
                      float* part_o, float* part_ml, unsigned* cnt, __half* o, int32_t* err,
                      cudaStream_t s) {
  const int smem = Layout<HD, MT>::kSmem;
  if (cudaFuncSetAttribute(attn_tc_persistent<HD, MT>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DFLASH_ECUDA;
  const cudaError_t e = launch_pdl(attn_tc_persistent<HD, MT>, dim3(2 * num_sms()),
                                   dim3(kThreads), smem, s, 1, tk, tv, q, kb, vb, pg, kv_rows,
                                   layer, batch, cap, ctx_len, req_valid, B, nq, nkv, seg_start,
                                   part_o, part_ml, cnt, o, err);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

// Chunk of the split-KV grid for one forward, from the actual context
// lengths.  The estimate follows how the grid behaves on B200: every CTA pays
// a fixed cost (set-up, the partial's write and fence: about kPlanFixed 64-key
// tiles' worth), CTAs run in waves over the resident slots, and the chunks of
// a request are merged by its last CTA (about kPlanMerge tiles per chunk).
// With L the mean keys of a request (context plus block), candidate q cuts L
// into q chunks, scaled by kPlanScale so that requests a little longer than
// the mean still take one chunk, rounded up to 64 keys and at least
// chunk_min.  One thread per candidate q = 1..64; ties go to the larger chunk.
// It then writes the forward's work list (see attn_tc_kernel).
constexpr float kPlanFixed = 8.f;
constexpr float kPlanMerge = 0.5f;
constexpr float kPlanScale = 1.06f;
constexpr int kPlanThreads = 64;

__global__ void __launch_bounds__(kPlanThreads)
    attn_chunk_plan_kernel(const int32_t* ctx_len, const int32_t* req_valid, int batch, int B,
                           int nkv, int chunk_min, int slots, int32_t* plan) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_sum[kPlanThreads / 32];
  __shared__ float s_est[kPlanThreads];
  __shared__ int s_chunk[kPlanThreads];
  __shared__ int s_tot[kPlanThreads / 32];
  __shared__ int s_carry;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  auto keys = [&](int r) { return (req_valid[r] ? ctx_len[r] : 0) + B; };  // context + block
  float acc = 0.f;
  for (int r = threadIdx.x; r < batch; r += kPlanThreads) acc += (float)keys(r);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) s_sum[w] = acc;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kPlanThreads / 32; ++i) tot += s_sum[i];
  const float L = fmaxf(tot / (float)max(batch, 1), 1.f);
  const int q = threadIdx.x + 1;
  int C = (int)ceilf(kPlanScale * L / (float)q);
  C = max(chunk_min, (C + kKeys - 1) / kKeys * kKeys);
  const float qe = ceilf(L / (float)C);  // chunks of a mean request
  const float waves = ceilf((float)batch * (float)nkv * qe / (float)max(slots, 1));
  s_est[threadIdx.x] = waves * ((float)((C + kKeys - 1) / kKeys) + kPlanFixed) + kPlanMerge * qe;
  s_chunk[threadIdx.x] = C;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  int best = 0;
  for (int i = 1; i < kPlanThreads; ++i)
    if (s_est[i] < s_est[best]) best = i;
  const int chunk = s_chunk[best];
  // the work list: every request's kv heads and chunks, in the order of the
  // (chunk, kv head, request) grid, request-major
  for (int base = 0; base < batch; base += kPlanThreads) {
    const int r = base + threadIdx.x;
    const int qr = r < batch ? (keys(r) + chunk - 1) / chunk : 0;
    const int n = nkv * qr;
    int x = n;  // inclusive scan inside the warp, then across the two warps
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_tot[w] = x;
    __syncthreads();
    const int start = s_carry + (w > 0 ? s_tot[0] : 0) + x - n;
    const int Tr = r < batch && req_valid[r] ? ctx_len[r] : 0;
    int2* items = reinterpret_cast<int2*>(plan) + 2;
    for (int j = 0; j < n; ++j) items[start + j] = make_int2((r << 16) | ((j / qr) << 8) | (j % qr), Tr);
    __syncthreads();
    if (threadIdx.x == kPlanThreads - 1) s_carry = start + n;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    plan[0] = chunk;
    plan[1] = s_carry;
  }
}

// Resident CTAs per SM of the split-KV grid kernel.
template <int HD, int MT>
int grid_ctas_per_sm() {
  static const int n = [] {  // thread-safe one-time initialisation
    const int smem = Layout<HD, MT>::kSmem;
    int v = 0;
    if (cudaFuncSetAttribute(attn_tc_kernel<HD, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, attn_tc_kernel<HD, MT>, kThreads,
                                                      smem) != cudaSuccess)
      v = 1;
    return std::max(1, v);
  }();
  return n;
}

template <int HD, int MT>
int launch_cfg(const CUtensorMap& tk, const CUtensorMap& tv, const __half* q, const __half* kb,
               const __half* vb, const KvPages& pg, long long kv_rows, int layer, int batch, int cap,
               const int32_t* ctx_len,
               const int32_t* req_valid, int B, int nq, int nkv, int chunk,
               const int32_t* plan_dev, int n_chunks, float* part_o, float* part_ml,
               unsigned* cnt, __half* o, int32_t* err, cudaStream_t s) {
  const int smem = Layout<HD, MT>::kSmem;
  if (cudaFuncSetAttribute(attn_tc_kernel<HD, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return DFLASH_ECUDA;
  // a planned forward runs a 1-D grid sized for the smallest chunk the plan may pick
  const dim3 grid = plan_dev != nullptr ? dim3(n_chunks * nkv * batch) : dim3(n_chunks, nkv, batch);
  const cudaError_t e =
      launch_pdl(attn_tc_kernel<HD, MT>, grid, dim3(kThreads), smem, s, 1, tk, tv, q, kb, vb, pg,
                 kv_rows, layer, batch, cap, ctx_len, req_valid, B, nq, nkv, chunk, plan_dev,
                 n_chunks, part_o, part_ml, cnt, o, err);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

template <int HD>
int launch_hd(const __half* q, const __half* kb, const __half* vb, const __half* kc,
              const __half* vc, const KvPages& pg, int layer, int batch, int cap,
              const int32_t* ctx_len, const int32_t* req_valid, int B, int nq, int nkv, int L,
              int chunk, const int32_t* plan_dev, int n_chunks, const int32_t* seg_start,
              float* part_o, float* part_ml,
              unsigned* cnt, __half* o, int32_t* err, cudaStream_t s) {
  CUtensorMap tk, tv;
  const int64_t rows = pg.table == nullptr ? (int64_t)L * batch * nkv * cap
                                           : (int64_t)L * pg.n_pages * nkv * pg.page;
  if (!encode_2d(&tk, kc, rows, HD, HD, kKeys, DFLASH_F16) ||
      !encode_2d(&tv, vc, rows, HD, HD, kKeys, DFLASH_F16))
    return DFLASH_ECUDA;
  const int R = B * (nq / nkv);
  if (seg_start != nullptr) {
    if (R <= 16)
      return launch_persistent<HD, 1>(tk, tv, q, kb, vb, pg, rows, layer, batch, cap, ctx_len,
                                      req_valid, B, nq, nkv, seg_start, part_o, part_ml, cnt, o,
                                      err, s);
    if (R <= 32)
      return launch_persistent<HD, 2>(tk, tv, q, kb, vb, pg, rows, layer, batch, cap, ctx_len,
                                      req_valid, B, nq, nkv, seg_start, part_o, part_ml, cnt, o,
                                      err, s);
    return launch_persistent<HD, 4>(tk, tv, q, kb, vb, pg, rows, layer, batch, cap, ctx_len,
                                    req_valid, B, nq, nkv, seg_start, part_o, part_ml, cnt, o, err,
                                    s);
  }
  if (HD == 128 && R <= 32 && B <= 16 && pg.table == nullptr && g_attn_umma) {
    return launch_attn_umma(tk, tv, q, kb, vb, pg, rows, layer, batch, cap, ctx_len,
                            req_valid, B, nq, nkv, chunk, plan_dev, n_chunks, part_o, part_ml, cnt,
                            o, err, s);
  }
  if (R <= 16)
    return launch_cfg<HD, 1>(tk, tv, q, kb, vb, pg, rows, layer, batch, cap, ctx_len, req_valid, B, nq, nkv,
                             chunk, plan_dev, n_chunks, part_o, part_ml, cnt, o, err, s);
  if (R <= 32)
    return launch_cfg<HD, 2>(tk, tv, q, kb, vb, pg, rows, layer, batch, cap, ctx_len, req_valid, B, nq, nkv,
                             chunk, plan_dev, n_chunks, part_o, part_ml, cnt, o, err, s);
  return launch_cfg<HD, 4>(tk, tv, q, kb, vb, pg, rows, layer, batch, cap, ctx_len, req_valid, B, nq, nkv,
                           chunk, plan_dev, n_chunks, part_o, part_ml, cnt, o, err, s);
}

}  // namespace

int launch_attn_plan(const int32_t* ctx_len, const int32_t* req_valid, int batch, int nkv,
                     int32_t* seg_start, cudaStream_t s) {
  TimedScope ts(s, TC_ATTN);
  const cudaError_t e = launch_pdl(attn_plan_kernel, dim3(1), dim3(1024), 0, s, 1, ctx_len,
                                   req_valid, batch, nkv, seg_start);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

int launch_attn_chunk_plan(const int32_t* ctx_len, const int32_t* req_valid, int batch, int B,
                           int nkv, int chunk_min, int32_t* chunk_out, int slots,
                           cudaStream_t s) {
  if (chunk_min <= 0 || chunk_min % kKeys != 0) return DFLASH_EINVAL;
  TimedScope ts(s, TC_ATTN);
  const cudaError_t e = launch_pdl(attn_chunk_plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, 1,
                                   ctx_len, req_valid, batch, B, nkv, chunk_min, slots, chunk_out);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

int attn_grid_slots(int hd, int R, int B, bool paged) {
  int per = 1;
  if (hd == 128 && R <= 32 && B <= 16 && !paged && g_attn_umma)
    per = attn_umma_ctas_per_sm();
  else if (hd == 128)
    per = R <= 16 ? grid_ctas_per_sm<128, 1>()
                  : (R <= 32 ? grid_ctas_per_sm<128, 2>() : grid_ctas_per_sm<128, 4>());
  else if (hd == 64)
    per = R <= 16 ? grid_ctas_per_sm<64, 1>()
                  : (R <= 32 ? grid_ctas_per_sm<64, 2>() : grid_ctas_per_sm<64, 4>());
  return per * num_sms();
}

int launch_attn_tc(const __half* q, const __half* kb, const __half* vb, const __half* kc,
                   const __half* vc, const KvPages& pg, int layer, int batch, int cap,
                   const int32_t* ctx_len,
                   const int32_t* req_valid, int B, int nq, int nkv, int hd, int L, int chunk,
                   const int32_t* plan_dev, int n_chunks, const int32_t* seg_start,
                   float* part_o, float* part_ml,
                   unsigned* cnt, __half* o, int32_t* err, cudaStream_t s) {
  if (B * (nq / nkv) > kAttnMaxRows || B > kBlkKeys) return DFLASH_EUNSUPPORTED;
  if (seg_start == nullptr && (chunk % kKeys != 0 || n_chunks > kMaxChunksTc))
    return DFLASH_EUNSUPPORTED;
  if (pg.table == nullptr && (int64_t)L * batch * nkv * cap > 0x7fffffffLL)
    return DFLASH_EUNSUPPORTED;
  if (pg.table != nullptr &&
      (pg.page % kKeys != 0 || (int64_t)L * pg.n_pages * nkv * pg.page > 0x7fffffffLL))
    return DFLASH_EUNSUPPORTED;
  TimedScope ts(s, TC_ATTN);
  if (hd == 128)
    return launch_hd<128>(q, kb, vb, kc, vc, pg, layer, batch, cap, ctx_len, req_valid, B, nq, nkv, L,
                          chunk, plan_dev, n_chunks, seg_start, part_o, part_ml, cnt, o, err, s);
  if (hd == 64)
    return launch_hd<64>(q, kb, vb, kc, vc, pg, layer, batch, cap, ctx_len, req_valid, B, nq, nkv, L,
                         chunk, plan_dev, n_chunks, seg_start, part_o, part_ml, cnt, o, err, s);
  return DFLASH_EUNSUPPORTED;
}

}  // namespace dflash
