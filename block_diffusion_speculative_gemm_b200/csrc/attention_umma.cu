// Block-vs-context attention on the 5th-generation tensor cores (tcgen05):
// head dim 128, up to 32 query rows per kv head, fp16 rows over an fp16 K/V
// cache.  Same grid, partials and chunk combine as the mma.sync kernel
// (attention_tc.cu): a CTA handles (key chunk, kv head, request).
//
// Per 64-key context tile (then one tile of the block's own keys, at most 16):
//   S^T = K Q^T  UMMA M = 128 (keys; the tile's 64 keys are rows 0-63), N = 32
//                query rows, K = 128 head dims; both operands K-major in the
//                128-byte swizzled layout TMA writes; S^T lands in one of two
//                TMEM buffers with a key per lane.
//   softmax      warps 0 and 1, one thread per key: each reads its 32 scores,
//                the column (query row) maxima come from a five-round shuffle
//                transpose and one exchange between the two warps; a
//                reference max per row (log2 units) moves only when a row's
//                max grew by more than 2^8, and then warp 0 (whose TMEM lanes
//                hold the 32 O rows) rescales O; each thread keeps its keys'
//                share of the 32 row sums and writes its P column (fp16) into
//                one of two shared-memory buffers.
//   O += P V     UMMA M = 128 (query rows; only the first 32 are real),
//                N = 128 (head dim), K = 64 keys; V is the MN-major B operand
//                (its rows are keys, head dim contiguous).
// Warp 2 issues the MMAs (S^T of tile t + 1 before O += P V of tile t), warp
// 3 streams K and V tiles with TMA through rings of their own: a K slot is
// free once its S^T MMA is done, long before the tile's P V, so K runs ahead
// in 2 slots while V has 3.  Tiles may run past a chunk's end; those keys are
// masked.  The unused rows of the M = 128 operands (the keys past 64, and the
// query rows past 32) are never read back: their descriptors run over the
// neighbouring buffers instead of zero padding, so two CTAs fit on an SM.
//
// Memory-bound: 4 * B * G flop per cache byte read, every cache byte read once.
#include "attn_combine.cuh"
#include "common.cuh"
#include "internal.h"

namespace dflash {

namespace {

constexpr int kHD = 128;
constexpr int kUKeys = 64;                       // keys per context tile
constexpr int kUBlk = 16;                        // rows of the block tile
constexpr int kUKStages = 2, kUVStages = 3;
constexpr int kUThreads = 128;
constexpr int kUTile = kUKeys * kHD * 2;         // K or V of one tile (16 KB)
constexpr int kUHalf = kUKeys * 128;             // one 64-column half of a tile
// region (1024-byte aligned offsets): block K and V (two 16-row halves of 2 KB
// each), Q (32 rows, two halves of 4 KB), P buffers (32 rows x 64 keys), then
// the K ring and the V ring.  Operands whose descriptors cover more rows than
// are real (block K and the K tiles as M = 128, P as M = 128) read into the
// buffers after them, always inside the allocation.
constexpr int kOffBK = 0, kOffBV = 4096, kOffQ0 = 8192, kOffQ1 = 12288, kOffP0 = 16384,
              kOffP1 = 20480;
constexpr int kOffKR = 24576;
constexpr int kOffVR = kOffKR + kUKStages * kUTile;
constexpr int kURegionEnd = kOffVR + kUVStages * kUTile;
constexpr int kUSmem = kURegionEnd + 1024;  // + alignment slack
constexpr uint32_t kColS = 0;    // two S^T buffers of 32 columns
constexpr uint32_t kColO = 128;  // O: 128 columns
constexpr uint32_t kTmemCols = 256;
constexpr float kLazy = 8.f;  // log2 growth of the row max before O is rescaled

static_assert(kUKStages * kUTile >= 2 * kAttnMaxChunks * kAttnMaxRows * 4, "combine scratch");
// the M = 128 K operand of the last K slot reads 8 KB past it (into the V ring)
static_assert(kOffKR + (kUKStages - 1) * kUTile + kUHalf + 128 * 128 <= kURegionEnd, "K overrun");
static_assert(kOffBK + kUBlk * 128 + 128 * 128 <= kURegionEnd, "block K overrun");
static_assert(kOffP1 + 128 * 128 <= kURegionEnd, "P overrun");

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

// Lane i ends with column i of the 32 x 32 block the warp holds one row per
// lane (v[j] = column j), reduced over the lanes by max (MAX) or sum.  Round o
// splits each lane's remaining columns in two: a lane with bit o set keeps the
// upper half, its partner lane ^ o the lower, and each combines the half it
// keeps with the same half from its partner.
template <bool MAX>
__device__ __forceinline__ float lane_column_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < o; ++j) {
      const float give = up ? v[j] : v[j + o];
      const float keep = up ? v[j + o] : v[j];
      const float got = __shfl_xor_sync(0xffffffffu, give, o);
      v[j] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
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
                     int nkv, int chunk_host, const int32_t* plan_dev, int n_chunks,
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
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // full/empty per K slot and per V slot, S^T full/free x2, P full, P free x2,
  // O done, column-max exchange x2, row-sum exchange
  constexpr int kNB = 2 * kUKStages + 2 * kUVStages + 4 + 1 + 2 + 1 + 2 + 1;
  __shared__ __align__(8) uint64_t bars[kNB];
  __shared__ float s_xch[2][2][32];  // [tile parity][warp][query row]
  __shared__ float s_lsum[32];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int G = nq / nkv;
  const int R = B * G;
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
  auto sK = [&](int st) { return s_base + kOffKR + st * kUTile; };
  auto sV = [&](int st) { return s_base + kOffVR + st * kUTile; };
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto full_k = [&](int st) { return bar(st); };
  auto empty_k = [&](int st) { return bar(kUKStages + st); };
  auto full_v = [&](int st) { return bar(2 * kUKStages + st); };
  auto empty_v = [&](int st) { return bar(2 * kUKStages + kUVStages + st); };
  constexpr int kB0 = 2 * kUKStages + 2 * kUVStages;
  auto s_full = [&](int b) { return bar(kB0 + b); };
  auto s_free = [&](int b) { return bar(kB0 + 2 + b); };
  const uint32_t p_full = bar(kB0 + 4);
  auto p_free = [&](int b) { return bar(kB0 + 5 + b); };  // per P buffer
  const uint32_t o_done = bar(kB0 + 7);
  auto x_full = [&](int b) { return bar(kB0 + 8 + b); };
  const uint32_t l_full = bar(kB0 + 10);

  if (tid == 0) {
    for (int st = 0; st < kUKStages; ++st) {
      mbar_init(full_k(st), 1);
      mbar_init(empty_k(st), 1);
    }
    for (int st = 0; st < kUVStages; ++st) {
      mbar_init(full_v(st), 1);
      mbar_init(empty_v(st), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), 2);  // both softmax warps
      mbar_init(p_free(b), 1);
      mbar_init(x_full(b), 2);
    }
    mbar_init(p_full, 2);
    mbar_init(o_done, 1);
    mbar_init(l_full, 1);
    fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&s_tmem), kTmemCols);
    tmem_relinquish();
  }
  // Warps 0-2 fetch the query rows of this kv head (row i = block position
  // i / G, head g G + i % G; rows R..31 zero) and the block's own keys by
  // cp.async while warp 3 already streams the first K/V tiles.
  constexpr int kLoaders = 96;
  if (warp < 3) {
    for (int idx = tid; idx < 32 * (kHD / 8); idx += kLoaders) {
      const int row = idx / (kHD / 8), ch = idx % (kHD / 8);
      const void* src = q;
      int bytes = 0;
      if (row < R) {
        src = q + ((size_t)(r * B + row / G) * nq + g * G + row % G) * kHD + ch * 8;
        bytes = 16;
      }
      cp_async16_u(s_base + (ch < 8 ? kOffQ0 : kOffQ1) + swz(row, ch), src, bytes);
    }
    if (has_blk) {
      for (int idx = tid; idx < 2 * kUBlk * (kHD / 8); idx += kLoaders) {
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
        cp_async16_u(s_base + (mat ? kOffBV : kOffBK) + (ch >> 3) * (kUBlk * 128) + swz(row, ch),
                     src, bytes);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();  // barrier init and the TMEM address visible
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  if (warp < 3) {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> UMMA
    // every loader's rows are in place before the first S^T MMA (warps 0-2
    // all reach this barrier: nothing before it can exit or wait)
    asm volatile("bar.sync 1, %0;" ::"n"(kLoaders) : "memory");
  }

  // a bounded wait that also gives up once another role has given up
  auto wait = [&](uint32_t b, uint32_t parity) -> bool {
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(b, parity)) {
      if (*(volatile int*)&s_abort || global_ns() - t0 > kWaitNs) {
        *(volatile int*)&s_abort = 1;
        return false;
      }
    }
    return true;
  };
  bool ok = true;

  if (warp == 3) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      for (int t = 0; t < nt; ++t) {
        const int p0 = k0 + t * kUKeys;  // the tile's first key position
        int y = pg.table == nullptr ? row_base + p0
                                    : (int)kv_row(pg, layer, batch, r, nkv, g, cap, p0);
        if (!DFLASH_CHECK(y >= 0 && y < kv_rows, err)) y = 0;  // a tile inside the store
        const int sk = t % kUKStages, sv = t % kUVStages;
        if (t >= kUKStages && !wait(empty_k(sk), ((t / kUKStages) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(full_k(sk), kUTile);
        tma_load_2d(sK(sk), &tmK, full_k(sk), 0, y, pol);
        tma_load_2d(sK(sk) + kUHalf, &tmK, full_k(sk), 64, y, pol);
        if (t >= kUVStages && !wait(empty_v(sv), ((t / kUVStages) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(full_v(sv), kUTile);
        tma_load_2d(sV(sv), &tmV, full_v(sv), 0, y, pol);
        tma_load_2d(sV(sv) + kUHalf, &tmV, full_v(sv), 64, y, pol);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_f16kind(128, 32, false);                // S^T, both K-major
      const uint32_t id_o = idesc_f16kind(128, kHD, false) | (1u << 16);  // B MN-major
      // Descriptors are built once: the start address sits in the low 14 bits
      // (in 16-byte units) and every operand lies below 256 KB of shared
      // memory, so moving inside a tile is an add of (offset >> 4).
      const uint64_t dq0 = smem_desc_sw128(s_base + kOffQ0), dq1 = smem_desc_sw128(s_base + kOffQ1);
      const uint64_t dk0 = smem_desc_sw128(sK(0)), dbk = smem_desc_sw128(s_base + kOffBK);
      const uint64_t dp0 = smem_desc_sw128(s_base + kOffP0), dp1 = smem_desc_sw128(s_base + kOffP1);
      const uint64_t dv0 = desc_mn_sw128(sV(0), kUHalf);
      const uint64_t dbv = desc_mn_sw128(s_base + kOffBV, kUBlk * 128);
      constexpr uint64_t kTileD = kUTile >> 4;
      auto issue_pv = [&](int u) -> bool {  // O += P V of tile u (P already in shared memory)
        const bool blk = u == nt;
        if (!blk && !wait(full_v(u % kUVStages), (u / kUVStages) & 1)) return false;
        tc_fence_after();
        const uint64_t ap = (u & 1) ? dp1 : dp0;
        const uint64_t bv = blk ? dbv : dv0 + (uint64_t)(u % kUVStages) * kTileD;
        const int steps = blk ? 1 : kUKeys / 16;
        for (int kk = 0; kk < steps; ++kk)
          umma_f16(tmem + kColO, ap + (uint64_t)(kk * 2), bv + (uint64_t)(kk * 128), id_o,
                   (u > 0 || kk > 0) ? 1u : 0u);
        if (!blk) umma_commit(empty_v(u % kUVStages));
        umma_commit(p_free(u & 1));
        return true;
      };
      for (int t = 0; t < ntot && ok; ++t) {
        const bool blk = t == nt;
        const int b = t & 1;
        if (!blk && !wait(full_k(t % kUKStages), (t / kUKStages) & 1)) { ok = false; break; }
        if (t >= 2 && !wait(s_free(b), ((t / 2) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint64_t a0 = blk ? dbk : dk0 + (uint64_t)(t % kUKStages) * kTileD;
        const uint64_t ahalf = blk ? (uint64_t)(kUBlk * 128 >> 4) : (uint64_t)(kUHalf >> 4);
#pragma unroll
        for (int ks = 0; ks < kHD / 16; ++ks)
          umma_f16(tmem + kColS + b * 32,
                   a0 + (uint64_t)(ks >> 2) * ahalf + (uint64_t)((ks & 3) * 2),
                   ((ks >> 2) ? dq1 : dq0) + (uint64_t)((ks & 3) * 2), id_s, ks > 0 ? 1u : 0u);
        if (!blk) umma_commit(empty_k(t % kUKStages));
        umma_commit(s_full(b));
        if (t >= 1) {
          if (!wait(p_full, (t - 1) & 1) || !issue_pv(t - 1)) { ok = false; break; }
        }
      }
      if (ok && ntot > 0) {
        if (wait(p_full, (ntot - 1) & 1) && issue_pv(ntot - 1))
          umma_commit(o_done);
        else
          ok = false;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax, one thread per key
    const float sl2 = rsqrtf((float)kHD) * 1.4426950408889634f;  // log2(e) / sqrt(hd)
    const int kk = warp * 32 + lane;  // key of the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    float mq = -INFINITY;  // reference max of query row `lane` (log2 units)
    float mrep[32];        // every row's reference max
    float lsum[32];        // this key lane's share of every row's sum
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      mrep[j] = 0.f;
      lsum[j] = 0.f;
    }
    for (int t = 0; t < ntot && ok; ++t) {
      const bool blk = t == nt;
      const int b = t & 1;
      const int nvalid = blk ? kb_hi - kb_lo : min(kUKeys, kc_end - (k0 + t * kUKeys));
      const bool valid = kk < nvalid;
      if (!__all_sync(0xffffffffu, wait(s_full(b), (t / 2) & 1))) { ok = false; break; }
      tc_fence_after();
      float sc[32];
      tmem_ld32(lane_addr + kColS + b * 32, sc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free(b));
      // column maxima over the tile's valid keys: this warp's, then both warps'
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = valid ? sc[j] : -INFINITY;
      s_xch[b][warp][lane] = lane_column_reduce<true>(v, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(x_full(b));
      if (!__all_sync(0xffffffffu, wait(x_full(b), (t / 2) & 1))) { ok = false; break; }
      const float mx = fmaxf(s_xch[b][0][lane], s_xch[b][1][lane]) * sl2;
      // The reference max moves only when the tile's max passes it by more
      // than kLazy (or on the first tile): P = 2^(s sl2 - m) then stays below
      // 2^kLazy, well inside fp16, and O is rescaled in TMEM only on such a move.
      const bool move = __any_sync(0xffffffffu, mx > mq + kLazy);
      float cf = 1.f;  // O and sum factor of row `lane` on a move
      if (move) {
        const float mn = fmaxf(mq, mx);
        cf = mq == -INFINITY ? 1.f : exp2f(mq - mn);
        mq = mn;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          mrep[j] = __shfl_sync(0xffffffffu, mn, j);
          lsum[j] *= __shfl_sync(0xffffffffu, cf, j);
        }
      }
      // P column of this key, rounded to fp16, while the previous tile's
      // O += P V may still run (it reads the other P buffer and O)
      __half ph[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float e = valid ? ex2_ftz(fmaf(sc[j], sl2, -mrep[j])) : 0.f;
        lsum[j] += e;
        ph[j] = __float2half_rn(e);
      }
      // P buffer t & 1 is free once O += P V of tile t - 2 is done; O may be
      // rescaled only once O += P V of tile t - 1 is done
      if (t >= 2 &&
          !__all_sync(0xffffffffu, wait(p_free(t & 1), ((t / 2) - 1) & 1))) {
        ok = false;
        break;
      }
      if (t >= 1 && move && warp == 0) {
        if (!__all_sync(0xffffffffu, wait(p_free((t - 1) & 1), ((t - 1) / 2) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < kHD; cc += 32) {
          float o[32];
          tmem_ld32(lane_addr + kColO + cc, o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] *= cf;
          tmem_st32(lane_addr + kColO + cc, o);
        }
      }
      // column kk of the P tile: query row j, key kk (K-major rows of 64 keys)
      uint8_t* pbuf = smem + (b ? kOffP1 : kOffP0) + (kk & 7) * 2;
#pragma unroll
      for (int j = 0; j < 32; ++j) *reinterpret_cast<__half*>(pbuf + swz(j, kk >> 3)) = ph[j];
      if (!blk && !valid) {
        // a key past the context holds another cache position: zero its V row
        // (once the tile has landed) so that it contributes exactly nothing
        const int sv = t % kUVStages;
        if (wait(full_v(sv), (t / kUVStages) & 1)) {
          uint8_t* vrow = smem + kOffVR + sv * kUTile;
#pragma unroll
          for (int ch = 0; ch < kHD / 8; ++ch)
            *reinterpret_cast<uint4*>(vrow + (ch >> 3) * kUHalf + swz(kk, ch)) =
                make_uint4(0, 0, 0, 0);
        } else {
          ok = false;
        }
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // P and zeros -> UMMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // the chunk's partial: O (unnormalised), max in natural-log units of the
    // scaled score, sum
    if (ok) {
      const float l = lane_column_reduce<false>(lsum, lane);  // this warp's share of row `lane`
      if (warp == 1) {
        s_lsum[lane] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(l_full);
      } else if (__all_sync(0xffffffffu, wait(o_done, 0) && wait(l_full, 0))) {
        tc_fence_after();
        const float lt = l + s_lsum[lane];
        const size_t pbase = (((size_t)r * nkv + g) * n_chunks + c) * kAttnMaxRows;
        const int row = lane;
#pragma unroll 1
        for (int cc = 0; cc < kHD; cc += 32) {
          float o[32];
          tmem_ld32(lane_addr + kColO + cc, o);
          if (row < R) {
            float4* dst = reinterpret_cast<float4*>(part_o + (pbase + row) * kHD + cc);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          }
        }
        if (row < R)
          *reinterpret_cast<float2*>(part_ml + (pbase + row) * 2) =
              make_float2(mq * 0.6931471805599453f, lt);
        __threadfence();  // this chunk's partial is visible before the chunk is counted
      } else {
        ok = false;
      }
    }
  }
  if (!ok) set_error(err, DFLASH_DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, kTmemCols);
  attn_chunk_combine<kHD, kUThreads>(reinterpret_cast<float*>(smem + kOffKR), r, g, R, B, G, nq,
                                     nkv, Tc, chunk, n_chunks, part_o, part_ml, cnt, out);
}

}  // namespace

int attn_umma_ctas_per_sm() {
  static const int n = [] {  // thread-safe one-time initialisation
    int v = 0;
    if (cudaFuncSetAttribute(attn_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kUSmem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, attn_umma_kernel, kUThreads, kUSmem) !=
            cudaSuccess)
      v = 1;
    return v > 0 ? v : 1;
  }();
  return n;
}

int launch_attn_umma(const CUtensorMap& tk, const CUtensorMap& tv, const __half* q,
                     const __half* kb, const __half* vb, const KvPages& pg, long long kv_rows,
                     int layer, int batch, int cap, const int32_t* ctx_len,
                     const int32_t* req_valid, int B, int nq, int nkv, int chunk,
                     const int32_t* plan_dev, int n_chunks, float* part_o, float* part_ml,
                     unsigned* cnt, __half* o, int32_t* err, cudaStream_t s) {
  if (B * (nq / nkv) > 32 || B > kUBlk || pg.table != nullptr || n_chunks > kAttnMaxChunks ||
      chunk % kUKeys != 0)
    return DFLASH_EUNSUPPORTED;
  if (cudaFuncSetAttribute(attn_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kUSmem) != cudaSuccess)
    return DFLASH_ECUDA;
  const dim3 grid = plan_dev != nullptr ? dim3(n_chunks * nkv * batch) : dim3(n_chunks, nkv, batch);
  const cudaError_t e =
      launch_pdl(attn_umma_kernel, grid, dim3(kUThreads), kUSmem, s, 1, tk, tv, q, kb, vb, pg,
                 kv_rows, layer, batch, cap, ctx_len, req_valid, B, nq, nkv, chunk, plan_dev,
                 n_chunks, part_o, part_ml, cnt, o, err);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace dflash
