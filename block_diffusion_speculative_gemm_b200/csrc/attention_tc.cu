// Tensor-core block-vs-context attention (split-KV partials) for fp16 block
// activations over a bf16 K/V cache.
//
// A CTA handles (key chunk, kv head, request) with 4 warps.  The chunk's keys
// -- cache positions below T_r, then the block's own B keys -- are streamed in
// 64-key tiles through a 3-stage cp.async ring of 16-byte copies, each key row
// XOR-swizzled in 16-byte units so that ldmatrix reads are conflict-free.
// Cache rows arrive as bf16 and are rewritten as fp16 in shared memory by the
// thread that copied them (exact for the cache's value range), so every
// product is an fp16 x fp16 -> fp32 mma.sync.m16n8k16.  Warp (mt, kg) owns
// query rows [16 mt, 16 mt + 16) and key group kg of every tile; it keeps the
// online-softmax state (row max m, row sum l, unnormalised O) in registers.
// The key groups of a row tile are merged through shared memory and one
// (m, l, O) partial per query row is written; a combine kernel merges chunks.
//
// Memory-bound at 2 * 4 * B * G flop per cache byte: the cache is read once,
// in 512-byte rows per key per matrix, and every stage is in flight while the
// previous tiles are multiplied.
#include "common.cuh"
#include "internal.h"

namespace dflash {

namespace {

constexpr int kThreads = 128;
constexpr int kKeys = 64;    // keys per tile
constexpr int kStages = 3;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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

template <int HD>
struct Layout {
  static constexpr int kRowBytes = HD * 2;
  static constexpr int kChunks = kRowBytes / 16;      // 16-byte chunks per key row
  static constexpr int kTileBytes = kKeys * kRowBytes;  // K or V of one tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQBytes = kAttnMaxRows * kRowBytes;
  static constexpr int kSmem = kStages * kStageBytes + kQBytes;
  __device__ static __forceinline__ uint32_t off(int row, int ch) {
    return (uint32_t)(row * kRowBytes + ((ch ^ (row & 7)) << 4));
  }
};

template <int HD>
__global__ void __launch_bounds__(kThreads)
    attn_tc_kernel(const __half* __restrict__ q, const __half* __restrict__ kb,
                   const __half* __restrict__ vb, const __nv_bfloat16* __restrict__ kc,
                   const __nv_bfloat16* __restrict__ vc, int layer, int batch, int cap,
                   const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ req_valid,
                   int B, int nq, int nkv, int chunk, int n_chunks, float* __restrict__ part_o,
                   float* __restrict__ part_ml) {
  using LY = Layout<HD>;
  constexpr int NT = HD / 8;   // n8 tiles of the output row
  constexpr int KS = HD / 16;  // k16 steps of q.k
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base + kStages * LY::kStageBytes;

  const int c = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int G = nq / nkv;
  const int R = B * G;
  const int Tc = req_valid[r] ? ctx_len[r] : 0;
  const int total = Tc + B;
  const int k0 = c * chunk;
  if (k0 >= total) return;
  const int k1 = min(total, k0 + chunk);
  const int ntiles = (k1 - k0 + kKeys - 1) / kKeys;
  const int MT = (R + 15) / 16;
  const int KG = (MT == 1) ? 4 : (MT == 2 ? 2 : 1);
  const int keys_per_warp = kKeys / KG;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt = warp % MT, kg = warp / MT;
  const bool computes = warp < MT * KG;
  const size_t cache_base = (((size_t)layer * batch + r) * nkv + g) * (size_t)cap * HD;

  // query rows of this kv head: row i = (block position i / G, head g*G + i % G)
  for (int idx = tid; idx < MT * 16 * LY::kChunks; idx += kThreads) {
    const int row = idx / LY::kChunks, ch = idx % LY::kChunks;
    const void* src = q;
    int bytes = 0;
    if (row < R) {
      src = q + ((size_t)(r * B + row / G) * nq + g * G + row % G) * HD + ch * 8;
      bytes = 16;
    }
    cp_async16(s_q + LY::off(row, ch), src, bytes);
  }

  auto load_tile = [&](int t, int st) {
    const uint32_t sb = s_base + st * LY::kStageBytes;
    for (int idx = tid; idx < 2 * kKeys * LY::kChunks; idx += kThreads) {
      const int mat = idx / (kKeys * LY::kChunks);
      const int rem = idx % (kKeys * LY::kChunks);
      const int row = rem / LY::kChunks, ch = rem % LY::kChunks;
      const int key = k0 + t * kKeys + row;
      const void* src = kc;
      int bytes = 0;
      if (key < Tc) {
        src = (mat ? vc : kc) + cache_base + (size_t)key * HD + ch * 8;
        bytes = 16;
      } else if (key < k1) {
        src = (mat ? vb : kb) + ((size_t)(r * B + key - Tc) * nkv + g) * HD + ch * 8;
        bytes = 16;
      }
      cp_async16(sb + mat * LY::kTileBytes + LY::off(row, ch), src, bytes);
    }
  };
  // cache rows were copied as bf16: the copying thread rewrites its chunks as fp16
  auto convert_tile = [&](int t, int st) {
    uint8_t* sb = smem + st * LY::kStageBytes;
    for (int idx = tid; idx < 2 * kKeys * LY::kChunks; idx += kThreads) {
      const int mat = idx / (kKeys * LY::kChunks);
      const int rem = idx % (kKeys * LY::kChunks);
      const int row = rem / LY::kChunks, ch = rem % LY::kChunks;
      if (k0 + t * kKeys + row >= Tc) continue;
      uint4* p = reinterpret_cast<uint4*>(sb + mat * LY::kTileBytes + LY::off(row, ch));
      uint4 u = *p;
      uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float lo = __uint_as_float(w[k] << 16);
        const float hi = __uint_as_float(w[k] & 0xffff0000u);
        w[k] = pack_h2(lo, hi);
      }
      *p = u;
    }
  };

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < ntiles) load_tile(s, s);
    cp_async_commit();
  }

  uint32_t qa[KS][4];
  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float scale = rsqrtf((float)HD);
  const int tq = lane & 3;                  // thread inside an mma row group
  const int mi = lane >> 3, li = lane & 7;  // ldmatrix: matrix index, row inside it

  for (int t = 0; t < ntiles; ++t) {
    const int st = t % kStages;
    if (t + kStages - 1 < ntiles) load_tile(t + kStages - 1, (t + kStages - 1) % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    convert_tile(t, st);
    __syncthreads();
    if (t == 0 && computes) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int row = mt * 16 + (mi & 1) * 8 + li;
        ldsm_x4(s_q + LY::off(row, ks * 2 + (mi >> 1)), qa[ks][0], qa[ks][1], qa[ks][2],
                qa[ks][3]);
      }
    }
    if (computes) {
      const uint32_t sK = s_base + st * LY::kStageBytes;
      const uint32_t sV = sK + LY::kTileBytes;
      for (int kb16 = 0; kb16 < keys_per_warp / 16; ++kb16) {
        const int key0 = kg * keys_per_warp + kb16 * 16;  // tile-local
        if (k0 + t * kKeys + key0 >= k1) break;           // all 16 keys past the chunk
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b0, b1, b2, b3;
          const int row = key0 + (mi >> 1) * 8 + li;
          ldsm_x4(sK + LY::off(row, ks * 2 + (mi & 1)), b0, b1, b2, b3);
          mma16816(s[0], qa[ks], b0, b1);
          mma16816(s[1], qa[ks], b2, b3);
        }
        // scale, mask keys past the chunk, online softmax for rows gq and gq + 8
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = k0 + t * kKeys + key0 + n * 8 + 2 * tq + (e & 1);
            s[n][e] = key < k1 ? s[n][e] * scale : -INFINITY;
            if (e < 2) mx0 = fmaxf(mx0, s[n][e]); else mx1 = fmaxf(mx1, s[n][e]);
          }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float c0 = (m0 == -INFINITY) ? 0.f : expf(m0 - n0);
        const float c1 = (m1 == -INFINITY) ? 0.f : expf(m1 - n1);
        float p[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float mref = e < 2 ? n0 : n1;
            p[n][e] = s[n][e] == -INFINITY ? 0.f : expf(s[n][e] - mref);
          }
        l0 = l0 * c0 + p[0][0] + p[0][1] + p[1][0] + p[1][1];
        l1 = l1 * c1 + p[0][2] + p[0][3] + p[1][2] + p[1][3];
        m0 = n0;
        m1 = n1;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          o[n][0] *= c0;
          o[n][1] *= c0;
          o[n][2] *= c1;
          o[n][3] *= c1;
        }
        const uint32_t pa[4] = {pack_h2(p[0][0], p[0][1]), pack_h2(p[0][2], p[0][3]),
                                pack_h2(p[1][0], p[1][1]), pack_h2(p[1][2], p[1][3])};
#pragma unroll
        for (int nd = 0; nd < NT; nd += 2) {
          uint32_t b0, b1, b2, b3;
          const int row = key0 + (mi & 1) * 8 + li;
          ldsm_x4_t(sV + LY::off(row, nd + (mi >> 1)), b0, b1, b2, b3);
          mma16816(o[nd], pa, b0, b1);
          mma16816(o[nd + 1], pa, b2, b3);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // row sums over the quad, then merge the key groups of each row tile
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* scratch = reinterpret_cast<float*>(smem);  // stage buffers are idle now
  constexpr int kSlot = NT * 4 + 4;
  static_assert(4 * 32 * kSlot * 4 <= kStages * Layout<HD>::kStageBytes, "merge scratch");
  if (computes && kg > 0) {
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
  if (!computes || kg > 0) return;
  for (int k = 1; k < KG; ++k) {
    const float* sl = scratch + ((size_t)(k * MT + mt) * 32 + lane) * kSlot;
    const float pm0 = sl[NT * 4 + 0], pm1 = sl[NT * 4 + 1];
    const float nm0 = fmaxf(m0, pm0), nm1 = fmaxf(m1, pm1);
    const float a0 = m0 == -INFINITY ? 0.f : expf(m0 - nm0);
    const float a1 = m1 == -INFINITY ? 0.f : expf(m1 - nm1);
    const float b0 = pm0 == -INFINITY ? 0.f : expf(pm0 - nm0);
    const float b1 = pm1 == -INFINITY ? 0.f : expf(pm1 - nm1);
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
  const size_t pbase = (((size_t)r * nkv + g) * n_chunks + c) * kAttnMaxRows;
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
}

template <int HD>
int launch_hd(const __half* q, const __half* kb, const __half* vb, const __nv_bfloat16* kc,
              const __nv_bfloat16* vc, int layer, int batch, int cap, const int32_t* ctx_len,
              const int32_t* req_valid, int B, int nq, int nkv, int chunk, int n_chunks,
              float* part_o, float* part_ml, cudaStream_t s) {
  const int smem = Layout<HD>::kSmem;
  if (cudaFuncSetAttribute(attn_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return DFLASH_ECUDA;
  dim3 grid(n_chunks, nkv, batch);
  attn_tc_kernel<HD><<<grid, kThreads, smem, s>>>(q, kb, vb, kc, vc, layer, batch, cap, ctx_len,
                                                  req_valid, B, nq, nkv, chunk, n_chunks, part_o,
                                                  part_ml);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace

int launch_attn_partial_tc(const __half* q, const __half* kb, const __half* vb,
                           const __nv_bfloat16* kc, const __nv_bfloat16* vc, int layer, int batch,
                           int cap, const int32_t* ctx_len, const int32_t* req_valid, int B,
                           int nq, int nkv, int hd, int chunk, int n_chunks, float* part_o,
                           float* part_ml, cudaStream_t s) {
  if (B * (nq / nkv) > kAttnMaxRows || chunk % kKeys != 0) return DFLASH_EUNSUPPORTED;
  TimedScope ts(s, TC_ATTN);
  if (hd == 128)
    return launch_hd<128>(q, kb, vb, kc, vc, layer, batch, cap, ctx_len, req_valid, B, nq, nkv,
                          chunk, n_chunks, part_o, part_ml, s);
  if (hd == 64)
    return launch_hd<64>(q, kb, vb, kc, vc, layer, batch, cap, ctx_len, req_valid, B, nq, nkv,
                         chunk, n_chunks, part_o, part_ml, s);
  return DFLASH_EUNSUPPORTED;
}

}  // namespace dflash
