// Block-vs-context attention on the 5th-generation tensor cores (tcgen05):
// head dim 128, up to 32 query rows per kv head, fp16 rows over an fp16 K/V
// cache.  Same grid, partials and chunk combine as the mma.sync kernel
// (attention_tc.cu): a CTA handles (key chunk, kv head, request).
//
// Per 48-key context tile (then one tile of the block's own keys, at most 16):
//   S = Q K^T   UMMA M = 128 (query rows; only the first 32 are real), N = 48
//               keys, K = 128; both operands K-major in the 128-byte swizzled
//               layout TMA writes; S lands in one of two TMEM buffers.
//   softmax     warp 0, one thread per query row: reads its S row from TMEM,
//               keeps a reference max (log2 units) and the sum, rescales its
//               O row in TMEM when some row's max grew by more than 2^8, and
//               writes P (fp16) into one of two shared-memory buffers, so it
//               waits for the O += P V two tiles back, not the last one.
//   O += P V    UMMA M = 128, N = 128 (head dim), K = 48 keys; V is the
//               MN-major B operand (its rows are keys, head dim contiguous).
// Warp 1 issues the MMAs (S of tile t + 1 before O += P V of tile t), warp 2
// streams K/V tiles with TMA through a 3-stage ring (48-key tiles keep three
// stages and two CTAs on an SM), warp 3 helps with the loads at setup.  Tiles
// may run past a chunk's end; those keys are masked.  The 96 unused rows of the M = 128 operands (Q and P) are
// never read back: their descriptors run over the neighbouring buffers of
// the same region instead of zero padding, so two CTAs fit on an SM.
//
// Memory-bound: 4 * B * G flop per cache byte read, every cache byte read once.
#include "attn_combine.cuh"
#include "common.cuh"
#include "internal.h"

namespace dflash {

namespace {

constexpr int kHD = 128;
constexpr int kUKeys = kUmmaKeys;                // keys per context tile (48)
constexpr int kUBlk = 16;                        // rows of the block tile
constexpr int kUStages = 3;
constexpr int kUThreads = 128;
constexpr int kUTile = kUKeys * kHD * 2;         // K or V of one tile (12 KB)
constexpr int kUStage = 2 * kUTile;
constexpr int kURegion = 32 * 1024;              // Q, P and the block tile
constexpr int kUSmem = kURegion + kUStages * kUStage + 1024;  // + alignment slack
// region offsets (the region comes first, so the unused rows of the last
// buffers run over the stages, inside the allocation): Q rows 0-31 of column
// half 0, P buffer 0 rows 0-31, block K and V (16 rows x two column halves
// each), Q rows 0-31 of column half 1, P buffer 1 rows 0-31
constexpr int kOffQ0 = 0, kOffP0 = 4096, kOffBK = 8192, kOffBV = 12288, kOffQ1 = 16384,
              kOffP1 = 20480;
constexpr uint32_t kColS = 0;    // two S buffers, 64 columns apart
constexpr uint32_t kColO = 128;  // O: 128 columns
constexpr uint32_t kTmemCols = 256;
constexpr float kLazy = 8.f;  // log2 growth of the row max before O is rescaled

static_assert(kUStages * kUStage >= 2 * kAttnMaxChunks * kAttnMaxRows * 4, "combine scratch");

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzled
// layout (64 MN-contiguous elements per 128-byte row, rows along K): `lbo` is
// the byte distance between 64-element column halves, 8-row (K) groups are
// 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Each thread of the warp writes 32 consecutive fp32 columns of its TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
      "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
      "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void cp_async16_u(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Byte offset of 16-byte chunk `ch` (8 elements) of row `row` in one 64-column
// half of a 128-byte swizzled tile.
__device__ __forceinline__ uint32_t swz(int row, int ch) {
  return (uint32_t)(row * 128 + (((ch & 7) ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kUThreads, 2)
    attn_umma_kernel(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __half* q, const __half* kb,
                     const __half* vb, const KvPages pg, long long kv_rows, int layer, int batch,
                     int cap, const int32_t* ctx_len, const int32_t* req_valid, int B, int nq,
                     int nkv, int chunk, int n_chunks, float* __restrict__ part_o,
                     float* __restrict__ part_ml, unsigned* __restrict__ cnt,
                     __half* __restrict__ out, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[2 * kUStages + 4 + 4];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int c = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int G = nq / nkv;
  const int R = B * G;
  const int Tc = req_valid[r] ? ctx_len[r] : 0;
  const int k0 = c * chunk;
  if (k0 >= Tc + B) return;
  const int k1 = min(Tc + B, k0 + chunk);
  const int kc_end = min(k1, Tc);                          // context keys [k0, kc_end)
  const int nt = kc_end > k0 ? (kc_end - k0 + kUKeys - 1) / kUKeys : 0;
  const int kb_lo = max(k0, Tc), kb_hi = min(k1, Tc + B);  // block keys [kb_lo, kb_hi)
  const bool has_blk = kb_hi > kb_lo;
  const int ntot = nt + (has_blk ? 1 : 0);                 // the block tile comes last
  const int row_base = pg.table == nullptr ? ((layer * batch + r) * nkv + g) * cap : 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_reg = s_base;
  auto sK = [&](int st) { return s_base + kURegion + st * kUStage; };
  auto sV = [&](int st) { return s_base + kURegion + st * kUStage + kUTile; };
  auto pbuf = [&](int t) { return (uint32_t)((t & 1) ? kOffP1 : kOffP0); };
  auto full = [&](int st) { return smem_u32(&bars[st]); };
  auto empty = [&](int st) { return smem_u32(&bars[kUStages + st]); };
  auto s_full = [&](int b) { return smem_u32(&bars[2 * kUStages + b]); };
  auto s_free = [&](int b) { return smem_u32(&bars[2 * kUStages + 2 + b]); };
  const uint32_t p_full = smem_u32(&bars[2 * kUStages + 4]);
  auto p_free = [&](int b) { return smem_u32(&bars[2 * kUStages + 5 + b]); };  // per P buffer
  const uint32_t o_done = smem_u32(&bars[2 * kUStages + 7]);

  if (tid == 0) {
    for (int st = 0; st < kUStages; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), 1);
    }
    mbar_init(p_full, 1);
    mbar_init(p_free(0), 1);
    mbar_init(p_free(1), 1);
    mbar_init(o_done, 1);
    fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), kTmemCols);
    tmem_relinquish();
  }
  // query rows of this kv head (row i = block position i / G, head g G + i % G;
  // rows R..31 zero) and the block's own keys, by cp.async
  for (int idx = tid; idx < 32 * (kHD / 8); idx += kUThreads) {
    const int row = idx / (kHD / 8), ch = idx % (kHD / 8);
    const void* src = q;
    int bytes = 0;
    if (row < R) {
      src = q + ((size_t)(r * B + row / G) * nq + g * G + row % G) * kHD + ch * 8;
      bytes = 16;
    }
    cp_async16_u(s_reg + (ch < 8 ? kOffQ0 : kOffQ1) + swz(row, ch), src, bytes);
  }
  if (has_blk) {
    for (int idx = tid; idx < 2 * kUBlk * (kHD / 8); idx += kUThreads) {
      const int mat = idx / (kUBlk * (kHD / 8));
      const int rem = idx % (kUBlk * (kHD / 8));
      const int row = rem / (kHD / 8), ch = rem % (kHD / 8);
      const int key = kb_lo + row;
      const void* src = kb;
      int bytes = 0;
      if (key < kb_hi) {
        src = (mat ? vb : kb) + ((size_t)(r * B + key - Tc) * nkv + g) * kHD + ch * 8;
        bytes = 16;
      }
      cp_async16_u(s_reg + (mat ? kOffBV : kOffBK) + (ch >> 3) * (kUBlk * 128) + swz(row, ch),
                   src, bytes);
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> UMMA
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  // a bounded wait that also gives up once another role has given up
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
      if (*(volatile int*)&s_abort || global_ns() - t0 > kWaitNs) {
        *(volatile int*)&s_abort = 1;
        return false;
      }
    }
    return true;
  };
  bool ok = true;

  if (warp == 2) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      for (int t = 0; t < nt; ++t) {
        const int st = t % kUStages;
        if (t >= kUStages && !wait(empty(st), ((t / kUStages) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(full(st), 2 * kUTile);
        // the tile's first key position; a paged store finds its row through
        // the request's page table (a tile never crosses a page)
        const int p0 = k0 + t * kUKeys;
        int y = pg.table == nullptr ? row_base + p0
                                    : (int)kv_row(pg, layer, batch, r, nkv, g, cap, p0);
        if (!DFLASH_CHECK(y >= 0 && y < kv_rows, err)) y = 0;  // a tile inside the store
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tma_load_2d(sK(st) + h * kUKeys * 128, &tmK, full(st), h * 64, y, pol);
          tma_load_2d(sV(st) + h * kUKeys * 128, &tmV, full(st), h * 64, y, pol);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s64 = idesc_f16kind(128, kUKeys, false);
      const uint32_t id_s16 = idesc_f16kind(128, kUBlk, false);
      const uint32_t id_o = idesc_f16kind(128, kHD, false) | (1u << 16);  // B MN-major
      auto issue_pv = [&](int t) {  // O += P V of tile t (P already in shared memory)
        const bool blk = t == nt;
        const int steps = blk ? 1 : kUKeys / 16;
        for (int kk = 0; kk < steps; ++kk) {
          const uint64_t bdesc = blk ? desc_mn_sw128(s_reg + kOffBV, kUBlk * 128)
                                     : desc_mn_sw128(sV(t % kUStages) + kk * 16 * 128,
                                                     kUKeys * 128);
          umma_f16(tmem + kColO, smem_desc_sw128(s_reg + pbuf(t) + kk * 32), bdesc, id_o,
                   (t > 0 || kk > 0) ? 1u : 0u);
        }
        if (!blk) umma_commit(empty(t % kUStages));
        umma_commit(p_free(t & 1));
      };
      for (int t = 0; t < ntot && ok; ++t) {
        const bool blk = t == nt;
        const int b = t & 1;
        if (!blk && !wait(full(t % kUStages), (t / kUStages) & 1)) { ok = false; break; }
        if (t >= 2 && !wait(s_free(b), ((t / 2) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < kHD / 16; ++ks) {
          const uint32_t a = s_reg + ((ks >> 2) ? kOffQ1 : kOffQ0) + (ks & 3) * 32;
          const uint32_t bk = blk ? s_reg + kOffBK + (ks >> 2) * (kUBlk * 128) + (ks & 3) * 32
                                  : sK(t % kUStages) + (ks >> 2) * (kUKeys * 128) + (ks & 3) * 32;
          umma_f16(tmem + kColS + b * 64, smem_desc_sw128(a), smem_desc_sw128(bk),
                   blk ? id_s16 : id_s64, ks > 0 ? 1u : 0u);
        }
        umma_commit(s_full(b));
        if (t >= 1) {
          if (!wait(p_full, (t - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv(t - 1);
        }
      }
      if (ok && ntot > 0) {
        if (wait(p_full, (ntot - 1) & 1)) {
          tc_fence_after();
          issue_pv(ntot - 1);
          umma_commit(o_done);
        } else {
          ok = false;
        }
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ softmax, one thread per row
    const float sl2 = rsqrtf((float)kHD) * 1.4426950408889634f;  // log2(e) / sqrt(hd)
    float m = -INFINITY, l = 0.f;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    for (int t = 0; t < ntot && ok; ++t) {
      const bool blk = t == nt;
      const int b = t & 1;
      const int nk = blk ? kUBlk : kUKeys;
      const int nvalid = blk ? kb_hi - kb_lo : min(kUKeys, kc_end - (k0 + t * kUKeys));
      if (!__all_sync(0xffffffffu, wait(s_full(b), (t / 2) & 1))) { ok = false; break; }
      tc_fence_after();
      float s[64];
      {
        float v[32];
        tmem_ld32(lane_addr + kColS + b * 64, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = v[j];
        if (!blk) {
          tmem_ld32(lane_addr + kColS + b * 64 + 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) s[32 + j] = v[j];
        } else {
#pragma unroll
          for (int j = 32; j < 64; ++j) s[j] = -INFINITY;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free(b));
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        if (j >= nvalid) s[j] = -INFINITY;  // past the context or the tile, or past the block
        mx = fmaxf(mx, s[j]);
      }
      // The reference max moves only when the tile's max passes it by more
      // than kLazy (or on the first tile): P = 2^(s sl2 - m) then stays below
      // 2^kLazy, well inside fp16, and O is rescaled in TMEM only on such a move.
      const bool move = __any_sync(0xffffffffu, mx * sl2 > m + kLazy);
      const float mn = move ? fmaxf(m, mx * sl2) : m;
      // P, rounded to fp16, while the previous tile's O += P V may still run
      // (it reads the P buffer and O)
      uint32_t pw[kUKeys / 2];
      float ps = 0.f;
#pragma unroll
      for (int k = 0; k < kUKeys / 2; ++k) {
        const float e0 = mn == -INFINITY ? 0.f : ex2_ftz(fmaf(s[2 * k], sl2, -mn));
        const float e1 = mn == -INFINITY ? 0.f : ex2_ftz(fmaf(s[2 * k + 1], sl2, -mn));
        ps += e0 + e1;
        const __half2 h = __floats2half2_rn(e0, e1);
        pw[k] = *reinterpret_cast<const uint32_t*>(&h);
      }
      // P buffer t & 1 is free once O += P V of tile t - 2 is done; O may be
      // rescaled only once O += P V of tile t - 1 is done
      if (t >= 2 &&
          !__all_sync(0xffffffffu, wait(p_free(t & 1), ((t / 2) - 1) & 1))) {
        ok = false;
        break;
      }
      if (t >= 1 && move) {
        if (!__all_sync(0xffffffffu, wait(p_free((t - 1) & 1), ((t - 1) / 2) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float cf = (m == -INFINITY || mn == -INFINITY) ? 1.f : exp2f(m - mn);
#pragma unroll 1
        for (int cc = 0; cc < kHD; cc += 32) {
          float v[32];
          tmem_ld32(lane_addr + kColO + cc, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= cf;
          tmem_st32(lane_addr + kColO + cc, v);
        }
        l *= cf;
      }
      // this row of the P tile (keys as K), 16 bytes per 8 keys
      uint8_t* prow = smem + pbuf(t);
#pragma unroll
      for (int ch = 0; ch < kUKeys / 8; ++ch) {
        if (ch * 8 >= nk) break;
        *reinterpret_cast<uint4*>(prow + swz(lane, ch)) =
            make_uint4(pw[4 * ch], pw[4 * ch + 1], pw[4 * ch + 2], pw[4 * ch + 3]);
      }
      l += ps;
      m = mn;
      if (!blk && nvalid < kUKeys) {
        // rows past the context hold other cache positions: zero them in V so
        // that masked keys contribute exactly nothing
        uint8_t* v = smem + kURegion + (t % kUStages) * kUStage + kUTile;
        for (int idx = lane; idx < (kUKeys - nvalid) * (kHD / 8); idx += 32) {
          const int row = nvalid + idx / (kHD / 8), ch = idx % (kHD / 8);
          *reinterpret_cast<uint4*>(v + (ch >> 3) * (kUKeys * 128) + swz(row, ch)) =
              make_uint4(0, 0, 0, 0);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // P and zeros -> UMMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // the chunk's partial: O (unnormalised), max in natural-log units of the
    // scaled score, sum
    if (ok && __all_sync(0xffffffffu, wait(o_done, 0))) {
      tc_fence_after();
      const size_t pbase = (((size_t)r * nkv + g) * n_chunks + c) * kAttnMaxRows;
      const int row = lane;
#pragma unroll 1
      for (int cc = 0; cc < kHD; cc += 32) {
        float v[32];
        tmem_ld32(lane_addr + kColO + cc, v);
        if (row < R) {
          float4* dst = reinterpret_cast<float4*>(part_o + (pbase + row) * kHD + cc);
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
      if (row < R)
        *reinterpret_cast<float2*>(part_ml + (pbase + row) * 2) =
            make_float2(m * 0.6931471805599453f, l);
      __threadfence();  // this chunk's partial is visible before the chunk is counted
    } else {
      ok = false;
    }
  }
  if (!ok) set_error(err, DFLASH_DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  attn_chunk_combine<kHD, kUThreads>(reinterpret_cast<float*>(smem + kURegion), r, g, R, B, G, nq,
                                     nkv, Tc,
                                     chunk, n_chunks, part_o, part_ml, cnt, out);
}

}  // namespace

int launch_attn_umma(const CUtensorMap& tk, const CUtensorMap& tv, const __half* q,
                     const __half* kb, const __half* vb, const KvPages& pg, long long kv_rows,
                     int layer, int batch, int cap, const int32_t* ctx_len,
                     const int32_t* req_valid, int B, int nq, int nkv, int chunk, int n_chunks,
                     float* part_o, float* part_ml, unsigned* cnt, __half* o, int32_t* err,
                     cudaStream_t s) {
  if (B * (nq / nkv) > 32 || B > kUBlk || pg.table != nullptr || n_chunks > kAttnMaxChunks)
    return DFLASH_EUNSUPPORTED;
  if (cudaFuncSetAttribute(attn_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kUSmem) != cudaSuccess)
    return DFLASH_ECUDA;
  const dim3 grid(n_chunks, nkv, batch);
  const cudaError_t e =
      launch_pdl(attn_umma_kernel, grid, dim3(kUThreads), kUSmem, s, 1, tk, tv, q, kb, vb, pg,
                 kv_rows, layer, batch, cap, ctx_len, req_valid, B, nq, nkv, chunk, n_chunks,
                 part_o, part_ml, cnt, o, err);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace dflash
