// C ABI of the DFlash hot path: argument checks, model prepacking, workspace
// layout and the launch sequences of inject / draft / verify.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

using namespace dflash;

namespace {
// One NVTX range per C-ABI call, named after the call: profilers show the
// library's calls on the host timeline (no cost without a tool attached).
struct NvtxCall {
  explicit NvtxCall(const char* name) { nvtxRangePushA(name); }
  ~NvtxCall() { nvtxRangePop(); }
};
}  // namespace

static_assert(sizeof(LmStat) == sizeof(dflash_lm_stat), "shard record layout");
static_assert(sizeof(ArgPart) == sizeof(dflash_row_argmax), "verify shard record layout");

// ============================================================== timing
namespace dflash {
namespace timing_detail {
struct Pending {
  int cls;
  cudaEvent_t a, b;
};
std::mutex g_tmu;
bool g_timing = false;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;
std::vector<std::pair<int, cudaEvent_t>> g_open;  // begin events waiting for their end
double g_ms[TC_N];
int64_t g_cnt[TC_N];

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e;
  cudaEventCreate(&e);
  return e;
}
}  // namespace timing_detail
using namespace timing_detail;

void timing_begin(cudaStream_t s, int cls) {
  if (!g_timing) return;
  std::lock_guard<std::mutex> lk(g_tmu);
  cudaEvent_t e = take_event();
  cudaEventRecord(e, s);
  g_open.push_back({cls, e});
}
void timing_end(cudaStream_t s, int cls) {
  if (!g_timing) return;
  std::lock_guard<std::mutex> lk(g_tmu);
  if (g_open.empty()) return;
  auto p = g_open.back();
  g_open.pop_back();
  cudaEvent_t e = take_event();
  cudaEventRecord(e, s);
  g_pending.push_back({cls, p.second, e});
}
}  // namespace dflash
using namespace dflash::timing_detail;

extern "C" int dflash_timing_enable(int on) {
  std::lock_guard<std::mutex> lk(g_tmu);
  g_timing = on != 0;
  return DFLASH_OK;
}

extern "C" int dflash_timing_read(double* ms, int64_t* cnt, int n) {
  std::lock_guard<std::mutex> lk(g_tmu);
  for (auto& p : g_pending) {
    float t = 0.f;
    if (cudaEventSynchronize(p.b) != cudaSuccess) return DFLASH_ECUDA;
    cudaEventElapsedTime(&t, p.a, p.b);
    g_ms[p.cls] += t;
    g_cnt[p.cls] += 1;
    g_pool.push_back(p.a);
    g_pool.push_back(p.b);
  }
  g_pending.clear();
  for (int i = 0; i < n && i < TC_N; ++i) {
    if (ms) ms[i] = g_ms[i];
    if (cnt) cnt[i] = g_cnt[i];
    g_ms[i] = 0.0;
    g_cnt[i] = 0;
  }
  return DFLASH_OK;
}

// ============================================================== model
struct LayerPack {
  void* Wqkv = nullptr;  // [qkv_out, d]
  void* Wo = nullptr;    // [d, nq*hd]
  void* Wgu = nullptr;   // [2I, d]
  void* Wd = nullptr;    // [d, I]
  float* g_in = nullptr;
  float* g_post = nullptr;
  WeightMap mqkv, mo, mgu, md;
};

struct dflash_model {
  dflash_config cfg;
  int device = 0;
  int vocab_lo = 0, vocab_hi = 0;  // LM-head rows held: [vocab_lo, vocab_hi) of the vocabulary
  int32_t* range_flag = nullptr;     // set by the packing kernels: a weight overflowed fp16
  size_t esz = 2;
  void* emb = nullptr;
  void* W_fc = nullptr;
  void* W_kv = nullptr;  // [L*2*nkv*hd, d]: for each layer [Wk; Wv]
  void* W_lm = nullptr;
  float* g_ctx = nullptr;
  float* g_final = nullptr;
  float* rope_cos = nullptr;
  float* rope_sin = nullptr;
  std::vector<LayerPack> layers;
  WeightMap mfc, mkv, mlm;
  std::vector<void*> allocs;
};

namespace {

template <typename T>
__global__ void gain_to_f32_kernel(const T* __restrict__ g, float* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = to_f(g[i]);
}

// cos/sin of p * base^(-2i/hd), evaluated in double precision, stored fp32.
__global__ void rope_table_kernel(float* __restrict__ cs, float* __restrict__ sn, int max_pos,
                                  int half, double base) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)max_pos * half) return;
  const int p = (int)(idx / half), i = (int)(idx % half);
  const double theta = pow(base, -2.0 * (double)i / (2.0 * half));
  const double ang = (double)p * theta;
  cs[idx] = (float)cos(ang);
  sn[idx] = (float)sin(ang);
}

void* dmalloc(dflash_model* m, size_t bytes) {
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return nullptr;
  m->allocs.push_back(p);
  return p;
}

void free_model(dflash_model* m) {
  for (void* p : m->allocs) cudaFree(p);
  m->allocs.clear();
}

bool copy_rows(void* dst, const void* src, size_t bytes) {
  return src != nullptr && cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToDevice) == cudaSuccess;
}

// range: set to 1 when a weight does not fit fp16 (|w| >= 65520 rounds to inf).
__global__ void bf16_to_f16_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst,
                                   size_t n, int32_t* range) {
  bool bad = false;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float v = __bfloat162float(src[i]);
    dst[i] = __float2half_rn(v);
    bad |= narrow_bad<__half>(v);
  }
  if (bad) *range = 1;
}

// Copies `elems` weight elements into a prepacked buffer.  For the bf16 model
// type the GEMM weights are stored as fp16: every bf16 value of magnitude in
// [2^-14, 65504] is exactly representable in fp16 (10 vs 7 mantissa bits);
// smaller values land on fp16 subnormals (absolute error <= 2^-25).  fp16
// operands let the activations that feed the tensor cores be stored with 3
// more mantissa bits at the same tcgen05 rate.
bool pack_weights(const dflash_model* m, void* dst, const void* src, size_t elems) {
  if (!src) return false;
  if (m->cfg.dtype != DFLASH_BF16) return copy_rows(dst, src, elems * sizeof(float));
  const unsigned blocks = (unsigned)std::min<size_t>((elems + 255) / 256, 148 * 32);
  bf16_to_f16_kernel<<<blocks, 256>>>(static_cast<const __nv_bfloat16*>(src),
                                      static_cast<__half*>(dst), elems, m->range_flag);
  return cudaGetLastError() == cudaSuccess;
}

float* gain_copy(dflash_model* m, const void* g) {
  const int d = m->cfg.d;
  float* out = static_cast<float*>(dmalloc(m, sizeof(float) * d));
  if (!out || !g) return nullptr;
  if (m->cfg.dtype == DFLASH_BF16)
    gain_to_f32_kernel<<<(d + 255) / 256, 256>>>(static_cast<const __nv_bfloat16*>(g), out, d);
  else
    gain_to_f32_kernel<<<(d + 255) / 256, 256>>>(static_cast<const float*>(g), out, d);
  return out;
}

bool config_ok(const dflash_config& c) {
  if (c.dtype != DFLASH_F32 && c.dtype != DFLASH_BF16) return false;
  if (c.H_t <= 0 || c.n_tap < 1 || c.n_tap > kMaxSeg || c.n_layers < 1 || c.d <= 0) return false;
  if (c.n_q <= 0 || c.n_kv <= 0 || c.n_q % c.n_kv) return false;
  if (c.head_dim <= 0 || c.head_dim % 2 || c.head_dim > 256 || c.inter <= 0) return false;
  if (c.vocab < 2 || c.mask_id < 0 || c.mask_id >= c.vocab || c.max_pos < 1) return false;
  if (!(c.eps >= 0.f) || !(c.rope_base > 0.0)) return false;
  if (c.d > 4096) return false;  // row kernels hold a row in registers (16 per thread)
  return true;
}

bool config_supported(const dflash_config& c) {
  if (c.head_dim != 64 && c.head_dim != 128) return false;
  if (c.inter % 64) return false;  // gate/up rows are packed in 64-row blocks
  if (c.d % 64) return false;      // row kernels move 16-byte vectors
  if (c.dtype == DFLASH_BF16) {
    if (c.d % 64 || c.H_t % 64 || (c.n_q * c.head_dim) % 128) return false;
    // fused epilogues need every 128-row weight tile to hold whole heads
    if ((c.n_kv * c.head_dim) % 128) return false;
  } else {
    const int kmax = std::max(std::max(c.n_tap * c.H_t, c.d), std::max(c.inter, c.n_q * c.head_dim));
    if (kmax > 12288) return false;  // SIMT GEMM keeps one token row in shared memory
  }
  return true;
}

int qkv_out(const dflash_config& c) { return (c.n_q + 2 * c.n_kv) * c.head_dim; }

// ---------------------------------------------------------------- workspace layout
// Workspace header: the device error word (byte 0), then 32768 completion
// counters: verify uses one per request, the draft attention one per
// (request, kv head).  No call writes the header except through those words,
// every call leaves the counters it used at zero (calls sharing a workspace
// never overlap), and each call's own buffers start after the header.
constexpr size_t kCntOff = 256;
constexpr size_t kHeader = kCntOff + (size_t(128) << 10);
constexpr int kMaxChunks = 64;
int g_attn_chunk = 0;  // split-KV chunk override in keys (tests and tuning; 0 = rule)
// GEMM schedules.  0 (default): the LM head streams K evenly over all workers
// (stream-K; its tiles are mostly whole, so little is left to finish in the
// kernel, and the last partial wave of 1187 vocabulary tiles disappears), the
// projections and the injection take fixed K splits, whose partials the
// following reduction kernels sum over hundreds of CTAs.  1: fixed splits
// everywhere.  2: stream-K everywhere (each split tile finished by its last
// piece inside the GEMM; measured 2x slower for the 256-token projections,
// whose few tiles split 3-5 ways).
int g_gemm_sched = 0;
bool sk_projections() { return g_gemm_sched == 2; }
// Draft attention schedule: 0 (default) the split-KV grid, its chunk planned on
// the device per forward;
// 1 persistent (every CTA the same number of key tiles, one TMA ring across
// (request, head) segments), which measured 15% slower at the 8B batch of 32
// (0.92-0.95 against 0.79-0.80 ms per draft): the SMs' idle time is not what
// bounds this kernel, its latency-bound mma.sync chains at ~9 warps per SM are.
int g_attn_sched = 0;
bool sk_lm_head() { return g_gemm_sched != 1; }
constexpr int kAttnRows = 64;
constexpr int kInjectChunkRows = 16384;
constexpr int kMaxSplits = 16;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct DraftLayout {
  size_t tokens, zrow, lm_rows, cstep, req_valid, lm_tok, lm_conf, x, h, q, kb, vb, o, act, part,
      sk, attn_o, attn_ml, seg, attn_chunk, stats, draw, logits, end;
  size_t part_elems;  // fp32 elements of split-K partials
};

struct InjectLayout {
  size_t c, u, part, sk, req_ok, end;
  size_t part_elems;
  int chunk_rows;
};

int draft_part_cols(const dflash_config& c) {
  return std::max(std::max(qkv_out(c), c.d), 2 * c.inter);
}

DraftLayout draft_layout(const dflash_config& c, int batch, int B) {
  DraftLayout L{};
  const size_t M = (size_t)batch * B;
  const size_t esz = c.dtype == DFLASH_BF16 ? 2 : 4;
  const int n_vt = (c.vocab + kTileN - 1) / kTileN;
  size_t off = kHeader;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.tokens = take(4 * M);
  L.zrow = take(4 * M);
  L.lm_rows = take(4 * M);
  L.cstep = take(4 * M);
  L.req_valid = take(4 * (size_t)batch);
  L.lm_tok = take(4 * M);
  L.lm_conf = take(4 * M);
  L.x = take(4 * M * c.d);
  L.h = take(esz * M * std::max(c.d, c.n_q * c.head_dim));
  L.q = take(esz * M * c.n_q * c.head_dim);
  L.kb = take(esz * M * c.n_kv * c.head_dim);
  L.vb = take(esz * M * c.n_kv * c.head_dim);
  L.o = take(esz * M * c.n_q * c.head_dim);
  L.act = take(esz * M * c.inter);
  // split-K partials: room for 4 splits of the widest projection
  L.part_elems = 4 * M * (size_t)draft_part_cols(c);
  L.part = take(4 * L.part_elems);
  L.sk = take(gemm_sk_slot_bytes((int)M));  // stream-K fixup shares
  // attention partials: the split-KV grid's [batch][nkv][chunk][64 rows], or
  // the persistent schedule's (2 * SMs + batch * nkv) slots of 64 rows
  const size_t arows = std::max((size_t)batch * c.n_kv * kMaxChunks * kAttnRows,
                                ((size_t)2 * num_sms() + (size_t)batch * c.n_kv) * kAttnRows);
  L.attn_o = take(4 * arows * c.head_dim);
  L.attn_ml = take(8 * arows);
  L.seg = take(4 * ((size_t)batch * c.n_kv + 1));  // persistent schedule: segment prefix
  // split-KV grid: the plan made on the device for a forward ({chunk, items, item...})
  L.attn_chunk = take(4 * (4 + 2 * (size_t)batch * c.n_kv * kMaxChunks));
  L.stats = take(sizeof(LmStat) * M * n_vt);
  // sampled drafting's draw partials: rows x chunks never exceeds M + 600 (the
  // chunk count falls as the row count grows)
  L.draw = take(std::max(sampled_draw_part_bytes((int)M, sampled_draw_chunks((int)M, c.vocab)),
                         sampled_draw_part_bytes((int)M + 600, 1)));
  L.logits = c.dtype == DFLASH_F32 ? take(4 * M * (size_t)c.vocab) : off;
  L.end = off;
  return L;
}

// batch: requests of a paged injection (one page-check flag each), 0 otherwise.
InjectLayout inject_layout(const dflash_config& c, int max_rows, int batch = 0) {
  InjectLayout L{};
  const size_t esz = c.dtype == DFLASH_BF16 ? 2 : 4;
  L.chunk_rows = std::min(std::max(max_rows, 1), kInjectChunkRows);
  const size_t n = L.chunk_rows;
  const size_t ncol = std::max((size_t)c.d, (size_t)c.n_layers * 2 * c.n_kv * c.head_dim);
  size_t off = kHeader;
  L.c = off;
  off = align256(off + esz * n * c.d);
  L.u = off;  // fc output before its RMSNorm (fp32)
  off = align256(off + 4 * n * c.d);
  // row counts up to 256 may split K up to kMaxSplits ways: room for the
  // largest of those, so a workspace sized for n rows also serves fewer rows
  L.part_elems = std::max((size_t)kMaxSplits * std::min<size_t>(n, 256), n) * ncol;
  L.part = off;
  off = align256(off + 4 * L.part_elems);
  L.sk = off;
  off = align256(off + gemm_sk_slot_bytes(L.chunk_rows));
  L.req_ok = off;
  off = align256(off + 4 * (size_t)std::max(batch, 0));
  L.end = off;
  return L;
}

// verify workspace: header (error word, completion counters) | argmax
// partials (8 bytes per row and chunk)
size_t verify_bytes(int batch, int B, int V) {
  const int rows = batch * B;
  return kHeader + align256((size_t)rows * verify_chunks(rows, V) * 8);
}

int32_t* err_word(void* ws) { return static_cast<int32_t*>(ws); }

// Stream-K scratch of a GEMM: the layout's share slots and the header's
// completion counters (every kernel using them waits for its predecessor to
// finish first and leaves them at zero).
void use_stream_k(GemmOut& o, void* ws, size_t slots_off) {
  o.sk_slots = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + slots_off);
  o.sk_cnt = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) + kCntOff);
  o.sk_cnt_cap = (int)((kHeader - kCntOff) / sizeof(unsigned));
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int cuda_status() { return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA; }

// Split count for a draft/inject GEMM: the picker's choice, lowered until the
// split partials fit the workspace; always a count gemm_tc runs unchanged.
// One split means the GEMM applies the following step itself (fused op).
int splits_for(int M, int N, int K, size_t cap_elems) {
  int s = gemm_pick_splits(M, N, K, kMaxSplits);
  const size_t fit = std::max<size_t>(1, cap_elems / ((size_t)M * N));
  while (s > 1 && (size_t)s > fit) s = gemm_effective_splits(K, s - 1);
  return s;
}

// Gate and up projections packed for the fused SwiGLU epilogue: 128-row blocks
// holding 64 gate rows, then the 64 up rows of the same features.
template <typename Tin, typename Tout>
__global__ void pack_gu_kernel(const Tin* __restrict__ wg, const Tin* __restrict__ wu,
                               Tout* __restrict__ out, int I, int d, int32_t* range) {
  const size_t total = (size_t)2 * I * d;
  bool bad = false;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(idx / d), k = (int)(idx % d);
    const int blk = n >> 7, w = n & 127;
    const Tin* src = (w < 64 ? wg : wu) + ((size_t)(blk * 64 + (w & 63))) * d + k;
    const float v = to_f(*src);
    out[idx] = from_f<Tout>(v);
    bad |= narrow_bad<Tout>(v);
  }
  if (bad) *range = 1;
}

}  // namespace

extern "C" const char* dflash_status_str(int st) {
  switch (st) {
    case DFLASH_OK: return "ok";
    case DFLASH_EINVAL: return "invalid argument";
    case DFLASH_EUNSUPPORTED: return "unsupported shape or dtype";
    case DFLASH_ECUDA: return "CUDA error";
    case DFLASH_ENOMEM: return "out of device memory";
    case DFLASH_EWORKSPACE: return "workspace too small";
    case DFLASH_ESCRATCH: return "request exceeds the fixed scratch of dflash_verify_noalloc";
    default: return "unknown status";
  }
}

namespace {

int model_create(const dflash_config* cfg, const dflash_weights* w, int vocab_lo, int vocab_hi,
                 dflash_model** out) {
  if (!cfg || !w || !out || !w->layers) return DFLASH_EINVAL;
  *out = nullptr;
  if (!config_ok(*cfg)) return DFLASH_EINVAL;
  if (!config_supported(*cfg)) return DFLASH_EUNSUPPORTED;
  if (vocab_lo < 0 || vocab_hi > cfg->vocab || vocab_hi <= vocab_lo) return DFLASH_EINVAL;
  const bool shard = vocab_lo != 0 || vocab_hi != cfg->vocab;
  if (shard && cfg->dtype != DFLASH_BF16) return DFLASH_EUNSUPPORTED;
  const dflash_config& c = *cfg;
  dflash_model* m = new dflash_model();
  m->cfg = c;
  m->vocab_lo = vocab_lo;
  m->vocab_hi = vocab_hi;
  const size_t Vs = (size_t)(vocab_hi - vocab_lo);  // LM-head rows held
  cudaGetDevice(&m->device);
  m->esz = c.dtype == DFLASH_BF16 ? 2 : 4;
  const size_t e = m->esz;
  const size_t d = c.d, hd = c.head_dim, nq = c.n_q, nkv = c.n_kv, I = c.inter, V = c.vocab;
  auto fail = [&](int code) {
    free_model(m);
    delete m;
    return code;
  };
  m->range_flag = static_cast<int32_t*>(dmalloc(m, sizeof(int32_t)));
  if (!m->range_flag || cudaMemset(m->range_flag, 0, sizeof(int32_t)) != cudaSuccess)
    return fail(DFLASH_ENOMEM);
  m->emb = dmalloc(m, e * V * d);
  m->W_fc = dmalloc(m, e * d * c.n_tap * c.H_t);
  m->W_lm = dmalloc(m, e * Vs * d);
  m->W_kv = dmalloc(m, e * c.n_layers * 2 * nkv * hd * d);
  if (!m->emb || !m->W_fc || !m->W_lm || !m->W_kv) return fail(DFLASH_ENOMEM);
  // embedding and fc stay in the model dtype (their inputs are exact in it);
  // every other GEMM weight goes through pack_weights
  if (!copy_rows(m->emb, w->emb, e * V * d) ||
      !copy_rows(m->W_fc, w->W_fc, e * d * c.n_tap * c.H_t) ||
      !w->W_lm ||
      !pack_weights(m, m->W_lm, static_cast<const uint8_t*>(w->W_lm) + e * vocab_lo * d, Vs * d))
    return fail(DFLASH_EINVAL);
  m->g_ctx = gain_copy(m, w->g_ctx);
  m->g_final = gain_copy(m, w->g_final);
  if (!m->g_ctx || !m->g_final) return fail(w->g_ctx && w->g_final ? DFLASH_ENOMEM : DFLASH_EINVAL);
  m->layers.resize(c.n_layers);
  const size_t kvrows = nkv * hd;
  for (int l = 0; l < c.n_layers; ++l) {
    const dflash_layer_weights& lw = w->layers[l];
    LayerPack& P = m->layers[l];
    P.Wqkv = dmalloc(m, e * qkv_out(c) * d);
    P.Wo = dmalloc(m, e * d * nq * hd);
    P.Wgu = dmalloc(m, e * 2 * I * d);
    P.Wd = dmalloc(m, e * d * I);
    if (!P.Wqkv || !P.Wo || !P.Wgu || !P.Wd) return fail(DFLASH_ENOMEM);
    uint8_t* qkv = static_cast<uint8_t*>(P.Wqkv);
    uint8_t* gu = static_cast<uint8_t*>(P.Wgu);
    uint8_t* kv = static_cast<uint8_t*>(m->W_kv) + (size_t)l * 2 * kvrows * d * e;
    if (!pack_weights(m, qkv, lw.Wq, nq * hd * d) ||
        !pack_weights(m, qkv + e * nq * hd * d, lw.Wk, kvrows * d) ||
        !pack_weights(m, qkv + e * (nq * hd + kvrows) * d, lw.Wv, kvrows * d) ||
        !pack_weights(m, P.Wo, lw.Wo, d * nq * hd) || !lw.Wg || !lw.Wu ||
        !pack_weights(m, P.Wd, lw.Wd, d * I) ||
        !pack_weights(m, kv, lw.Wk, kvrows * d) || !pack_weights(m, kv + e * kvrows * d, lw.Wv, kvrows * d))
      return fail(DFLASH_EINVAL);
    {
      const unsigned blocks = (unsigned)std::min<size_t>((2 * I * d + 255) / 256, 148 * 32);
      if (c.dtype == DFLASH_BF16)
        pack_gu_kernel<__nv_bfloat16, __half><<<blocks, 256>>>(
            static_cast<const __nv_bfloat16*>(lw.Wg), static_cast<const __nv_bfloat16*>(lw.Wu),
            static_cast<__half*>((void*)gu), (int)I, (int)d, m->range_flag);
      else
        pack_gu_kernel<float, float><<<blocks, 256>>>(static_cast<const float*>(lw.Wg),
                                                     static_cast<const float*>(lw.Wu),
                                                     static_cast<float*>((void*)gu), (int)I,
                                                     (int)d, m->range_flag);
    }
    P.g_in = gain_copy(m, lw.g_in);
    P.g_post = gain_copy(m, lw.g_post);
    if (!P.g_in || !P.g_post) return fail(DFLASH_EINVAL);
  }
  const int half = c.head_dim / 2;
  m->rope_cos = static_cast<float*>(dmalloc(m, sizeof(float) * (size_t)c.max_pos * half));
  m->rope_sin = static_cast<float*>(dmalloc(m, sizeof(float) * (size_t)c.max_pos * half));
  if (!m->rope_cos || !m->rope_sin) return fail(DFLASH_ENOMEM);
  {
    const int64_t n = (int64_t)c.max_pos * half;
    rope_table_kernel<<<(unsigned)((n + 255) / 256), 256>>>(m->rope_cos, m->rope_sin, c.max_pos,
                                                             half, c.rope_base);
  }
  if (c.dtype == DFLASH_BF16) {
    const int H = DFLASH_F16;
    bool ok = encode_weight_map(m->mfc, m->W_fc, c.d, c.n_tap * c.H_t, DFLASH_BF16) &&
              encode_weight_map(m->mkv, m->W_kv, c.n_layers * 2 * kvrows, c.d, H) &&
              encode_weight_map(m->mlm, m->W_lm, (int)Vs, c.d, H);
    for (int l = 0; l < c.n_layers && ok; ++l) {
      LayerPack& P = m->layers[l];
      ok = encode_weight_map(P.mqkv, P.Wqkv, qkv_out(c), c.d, H) &&
           encode_weight_map(P.mo, P.Wo, c.d, c.n_q * c.head_dim, H) &&
           encode_weight_map(P.mgu, P.Wgu, 2 * c.inter, c.d, H) &&
           encode_weight_map(P.md, P.Wd, c.d, c.inter, H);
    }
    if (!ok) return fail(DFLASH_ECUDA);
    // pre-tile every GEMM weight for bulk streaming, then drop the row-major copies
    std::vector<void*> row_major;
    auto tile_into = [&](WeightMap& wm, void* rm, int N, int K) -> bool {
      void* t = dmalloc(m, tiled_bytes(N, K));
      if (!t) return false;
      tile_weights(rm, t, N, K, 0);
      if (!set_tiled_weights(wm, t)) return false;
      row_major.push_back(rm);
      return true;
    };
    ok = tile_into(m->mfc, m->W_fc, c.d, c.n_tap * c.H_t) &&
         tile_into(m->mkv, m->W_kv, c.n_layers * 2 * kvrows, c.d) &&
         tile_into(m->mlm, m->W_lm, (int)Vs, c.d);
    for (int l = 0; l < c.n_layers && ok; ++l) {
      LayerPack& P = m->layers[l];
      ok = tile_into(P.mqkv, P.Wqkv, qkv_out(c), c.d) &&
           tile_into(P.mo, P.Wo, c.d, c.n_q * c.head_dim) &&
           tile_into(P.mgu, P.Wgu, 2 * c.inter, c.d) &&
           tile_into(P.md, P.Wd, c.d, c.inter);
    }
    if (!ok) return fail(DFLASH_ENOMEM);
    if (cudaDeviceSynchronize() != cudaSuccess) return fail(DFLASH_ECUDA);
    for (void* rm : row_major) {
      cudaFree(rm);
      m->allocs.erase(std::find(m->allocs.begin(), m->allocs.end(), rm));
    }
    m->W_fc = m->W_kv = m->W_lm = nullptr;
    for (auto& P : m->layers) P.Wqkv = P.Wo = P.Wgu = P.Wd = nullptr;
    // the tensor maps stay valid as descriptors only; the GEMMs read `tiled`
    m->mfc.ptr = m->mkv.ptr = m->mlm.ptr = nullptr;
    for (auto& P : m->layers) P.mqkv.ptr = P.mo.ptr = P.mgu.ptr = P.md.ptr = nullptr;
  }
  if (cudaDeviceSynchronize() != cudaSuccess || cudaGetLastError() != cudaSuccess)
    return fail(DFLASH_ECUDA);
  // the bf16 model type multiplies in fp16: a weight past fp16's range is refused
  int32_t range = 0;
  if (cudaMemcpy(&range, m->range_flag, sizeof(range), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(DFLASH_ECUDA);
  if (range) return fail(DFLASH_EUNSUPPORTED);
  *out = m;
  return DFLASH_OK;
}

bool whole_vocab(const dflash_model* m) {
  return m->vocab_lo == 0 && m->vocab_hi == m->cfg.vocab;
}

}  // namespace

extern "C" int dflash_model_create(const dflash_config* cfg, const dflash_weights* w,
                                   dflash_model** out) {
  return model_create(cfg, w, 0, cfg ? cfg->vocab : 0, out);
}

extern "C" int dflash_model_create_shard(const dflash_config* cfg, const dflash_weights* w,
                                         int vocab_lo, int vocab_hi, dflash_model** out) {
  return model_create(cfg, w, vocab_lo, vocab_hi, out);
}

extern "C" int dflash_model_destroy(dflash_model* m) {
  if (!m) return DFLASH_OK;
  cudaDeviceSynchronize();
  free_model(m);
  delete m;
  return DFLASH_OK;
}

extern "C" size_t dflash_workspace_size(const dflash_model* m, int max_batch, int B,
                                        int max_inject_rows) {
  if (!m || max_batch < 0 || B < 0 || max_inject_rows < 0) return 0;
  size_t s = kHeader;
  if (max_batch > 0 && B > 0) {
    s = std::max(s, draft_layout(m->cfg, max_batch, B).end);
    s = std::max(s, verify_bytes(max_batch, B, m->cfg.vocab));
  }
  if (max_inject_rows > 0)
    s = std::max(s, inject_layout(m->cfg, max_inject_rows, std::max(max_batch, 0)).end);
  return s;
}

extern "C" size_t dflash_verify_workspace_size(int batch, int B, int V) {
  if (batch < 0 || B < 0 || V < 1) return 0;
  if (batch == 0 || B == 0) return kHeader;
  return verify_bytes(batch, B, V);
}

extern "C" int dflash_workspace_init(void* ws, size_t bytes, void* stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return DFLASH_EINVAL;
  return cudaMemsetAsync(ws, 0, bytes, (cudaStream_t)stream) == cudaSuccess ? DFLASH_OK
                                                                           : DFLASH_ECUDA;
}

extern "C" int dflash_get_error(void* ws, void* stream, int32_t* bits) {
  if (!ws || !bits) return DFLASH_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return DFLASH_ECUDA;
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return DFLASH_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DFLASH_ECUDA;
  *bits = h;
  return DFLASH_OK;
}

// ============================================================== inject
namespace {

// Injection into the contiguous cache (pg.table == nullptr) or into paged
// pools; `cap` is the positions a request can hold.
int inject_impl(const dflash_model* m, const void* const* taps, const int32_t* cu_rows,
                const int32_t* start_pos, int batch, int n_rows, void* k_cache, void* v_cache,
                int cache_cap, KvPages pg, void* ws, cudaStream_t s) {
  const dflash_config& c = m->cfg;
  const InjectLayout L = inject_layout(c, n_rows, pg.table ? batch : 0);
  int32_t* err = err_word(ws);
  const int kvN = c.n_layers * 2 * c.n_kv * c.head_dim;
  const size_t e = m->esz;
  if (pg.table != nullptr) {
    pg.req_ok = at<int32_t>(ws, L.req_ok);
    launch_inject_page_check(cu_rows, start_pos, batch, pg, at<int32_t>(ws, L.req_ok), err, s);
  }
  const int64_t kv_ls = pg.table ? (int64_t)pg.n_pages * c.n_kv * pg.page
                                 : (int64_t)batch * c.n_kv * cache_cap;
  const int64_t kv_hs = pg.table ? pg.page : cache_cap;
  for (int r0 = 0; r0 < n_rows; r0 += L.chunk_rows) {
    const int n = std::min(L.chunk_rows, n_rows - r0);
    const void* seg[kMaxSeg];
    for (int t = 0; t < c.n_tap; ++t)
      seg[t] = static_cast<const uint8_t*>(taps[t]) + (size_t)r0 * c.H_t * e;
    float* part = at<float>(ws, L.part);
    void* cbuf = at<void>(ws, L.c);
    int st;
    if (c.dtype == DFLASH_BF16) {
      // u = concat(taps) W_fc^T, c = RMSNorm(u; g_ctx).  Stream-K: the GEMM
      // finishes every tile itself and stores u; fixed splits leave partials
      const bool skm = sk_projections();
      const int s1 = skm ? 1 : splits_for(n, c.d, c.n_tap * c.H_t, L.part_elems);
      GemmOut o1;
      if (s1 == 1) {
        o1.op = OP_STORE;
        o1.f32 = at<float>(ws, L.u);
      } else {
        o1.part = part;
      }
      if (skm) use_stream_k(o1, ws, L.sk);
      st = gemm_tc(m->mfc, seg, c.n_tap, c.H_t, c.H_t, n, skm ? 0 : s1, EPI_PARTIAL, o1, err, s);
      if (st) return st;
      launch_ctx_norm<__half>(s1 == 1 ? o1.f32 : part, s1, n, c.d, m->g_ctx,
                              static_cast<__half*>(cbuf), c.eps, err, s);
      // every layer's K (RoPE) and V into the cache
      const int s2 = skm ? 1 : splits_for(n, kvN, c.d, L.part_elems);
      const void* cseg[1] = {cbuf};
      GemmOut o2;
      if (s2 == 1) {
        o2.op = OP_KV;
        o2.h1 = static_cast<__half*>(k_cache);
        o2.h2 = static_cast<__half*>(v_cache);
        o2.cos_t = m->rope_cos;
        o2.sin_t = m->rope_sin;
        o2.cu_rows = cu_rows;
        o2.start_pos = start_pos;
        o2.nkv = c.n_kv;
        o2.hd = c.head_dim;
        o2.row0 = r0;
        o2.batch = batch;
        o2.cap = cache_cap;
        o2.max_pos = c.max_pos;
        o2.pages = pg;
        o2.kv_ls = kv_ls;
        o2.kv_hs = kv_hs;
      } else {
        o2.part = part;
      }
      if (skm) use_stream_k(o2, ws, L.sk);
      st = gemm_tc(m->mkv, cseg, 1, c.d, c.d, n, skm ? 0 : s2, EPI_PARTIAL, o2, err, s);
      if (st) return st;
      if (s2 > 1)
        launch_kv_scatter<__half>(part, s2, n, r0, c.n_layers, c.n_kv, c.head_dim, cu_rows,
                                  start_pos, batch, cache_cap, pg, m->rope_cos, m->rope_sin,
                                  c.max_pos, static_cast<__half*>(k_cache),
                                  static_cast<__half*>(v_cache), err, s);
    } else {
      const float* fseg[kMaxSeg];
      for (int t = 0; t < c.n_tap; ++t) fseg[t] = static_cast<const float*>(seg[t]);
      gemm_simt_f32(static_cast<const float*>(m->W_fc), c.d, c.n_tap * c.H_t, fseg, c.n_tap,
                    c.H_t, n, part, s);
      launch_ctx_norm<float>(part, 1, n, c.d, m->g_ctx, static_cast<float*>(cbuf), c.eps, err, s);
      const float* cseg[1] = {static_cast<const float*>(cbuf)};
      gemm_simt_f32(static_cast<const float*>(m->W_kv), kvN, c.d, cseg, 1, c.d, n, part, s);
      launch_kv_scatter<float>(part, 1, n, r0, c.n_layers, c.n_kv, c.head_dim, cu_rows,
                               start_pos, batch, cache_cap, pg, m->rope_cos, m->rope_sin,
                               c.max_pos, static_cast<float*>(k_cache),
                               static_cast<float*>(v_cache), err, s);
    }
    if ((st = cuda_status())) return st;
  }
  return DFLASH_OK;
}

// Host checks of a paged K/V description shared by the paged calls.
int check_pages(const dflash_model* m, const void* k_pool, const void* v_pool, int n_pages,
                int page_size, const int32_t* page_table, int max_pages) {
  const dflash_config& c = m->cfg;
  if (!k_pool || !v_pool || !page_table || n_pages < 1 || max_pages < 1 || page_size < 1)
    return DFLASH_EINVAL;
  if (!aligned16(k_pool) || !aligned16(v_pool)) return DFLASH_EINVAL;
  if (c.dtype != DFLASH_BF16) return DFLASH_EUNSUPPORTED;  // the tensor-core attention only
  if (page_size % 64 != 0) return DFLASH_EUNSUPPORTED;     // whole 64-key attention tiles
  if ((int64_t)c.n_layers * n_pages * c.n_kv * page_size > 0x7fffffffLL)
    return DFLASH_EUNSUPPORTED;
  if ((int64_t)max_pages * page_size > 0x7fffffffLL) return DFLASH_EUNSUPPORTED;
  return DFLASH_OK;
}

}  // namespace

extern "C" int dflash_inject_kv(const dflash_model* m, const void* const* taps,
                                const int32_t* cu_rows, const int32_t* start_pos, int batch,
                                int n_rows, void* k_cache, void* v_cache, int cache_cap, void* ws,
                                size_t ws_bytes, void* stream) {
  NvtxCall nvtx_("dflash_inject_kv");
  if (!m || batch < 1 || n_rows < 0 || cache_cap < 1) return DFLASH_EINVAL;
  if (n_rows == 0) return DFLASH_OK;
  const dflash_config& c = m->cfg;
  if (!taps || !cu_rows || !start_pos || !k_cache || !v_cache || !ws) return DFLASH_EINVAL;
  for (int t = 0; t < c.n_tap; ++t)
    if (!taps[t] || !aligned16(taps[t])) return DFLASH_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return DFLASH_EINVAL;
  if (ws_bytes < inject_layout(c, n_rows).end) return DFLASH_EWORKSPACE;
  return inject_impl(m, taps, cu_rows, start_pos, batch, n_rows, k_cache, v_cache, cache_cap,
                     KvPages{}, ws, (cudaStream_t)stream);
}

extern "C" int dflash_inject_kv_paged(const dflash_model* m, const void* const* taps,
                                      const int32_t* cu_rows, const int32_t* start_pos,
                                      int batch, int n_rows, void* k_pool, void* v_pool,
                                      int n_pages, int page_size, const int32_t* page_table,
                                      int max_pages, void* ws, size_t ws_bytes, void* stream) {
  NvtxCall nvtx_("dflash_inject_kv_paged");
  if (!m || batch < 1 || n_rows < 0) return DFLASH_EINVAL;
  if (n_rows == 0) return DFLASH_OK;
  const dflash_config& c = m->cfg;
  if (!taps || !cu_rows || !start_pos || !ws) return DFLASH_EINVAL;
  for (int t = 0; t < c.n_tap; ++t)
    if (!taps[t] || !aligned16(taps[t])) return DFLASH_EINVAL;
  if (reinterpret_cast<uintptr_t>(ws) & 255) return DFLASH_EINVAL;
  int st = check_pages(m, k_pool, v_pool, n_pages, page_size, page_table, max_pages);
  if (st) return st;
  if (ws_bytes < inject_layout(c, n_rows, batch).end) return DFLASH_EWORKSPACE;
  KvPages pg;
  pg.table = page_table;
  pg.max_pages = max_pages;
  pg.page = page_size;
  pg.n_pages = n_pages;
  return inject_impl(m, taps, cu_rows, start_pos, batch, n_rows, k_pool, v_pool,
                     max_pages * page_size, pg, ws, (cudaStream_t)stream);
}

// ============================================================== draft
namespace {

// Sampled drafting: temperature, Philox key and offset, and the caller's
// draft-logits output (fp32 or bf16 [batch, B, V]).
struct SampleArgs {
  float tau;
  uint64_t seed, offset;
  void* q;
  int q_bf16;
};

// T: activation / GEMM operand type; TC: K/V cache type; TE: embedding type.
// samp == nullptr: greedy drafting (argmax, max-probability confidence).
// Which parts of a draft one call runs.  The whole draft (dflash_draft_block)
// runs them all; a vocabulary-parallel draft runs them one at a time so that the
// per-row LM-head statistics of every vocabulary shard can be exchanged between
// the forward and the commit of each step.
struct DraftPhase {
  bool init = true;                // block initialisation (and the request checks)
  bool forward = true;             // embedding, layers and LM head of the steps run
  bool commit = true;              // token choice and commit of the steps run
  bool finish = true;              // copy-out of the draft tokens and commit steps
  int t0 = 0, t1 = 1 << 30;        // the steps run: [t0, min(t1, n_steps))
  LmStat* shard_stats = nullptr;   // forward only: per-row statistics of this shard (out)
  const LmStat* gathered = nullptr;  // commit: [world][rows] statistics of every shard
  int world = 0;
};

// Masked positions per request before step t of an n_steps draft of block B.
int masked_before(int B, int n_steps, int t) {
  int rem = B - 1;
  for (int u = 0; u < t && u < n_steps; ++u) rem -= (rem + (n_steps - u) - 1) / (n_steps - u);
  return rem;
}

// pg.table set: the context is read from paged pools, cap = positions per
// request (the RoPE bound on ctx_len + B).
template <typename T, typename TC, typename TE>
int draft_impl(const dflash_model* m, const int32_t* anchor, const int32_t* ctx_len,
               const void* k_cache, const void* v_cache, int cap, const KvPages& pg, int batch,
               int B, int n_steps, int32_t* draft_tokens, int32_t* commit_step, float* logits_dbg,
               const SampleArgs* samp, void* ws, cudaStream_t s,
               const DraftPhase& ph = DraftPhase()) {
  const dflash_config& c = m->cfg;
  const DraftLayout L = draft_layout(c, batch, B);
  const int M = batch * B;
  const int hd = c.head_dim, nq = c.n_q, nkv = c.n_kv;
  int32_t* err = err_word(ws);
  int32_t* tokens = at<int32_t>(ws, L.tokens);
  int32_t* zrow = at<int32_t>(ws, L.zrow);
  int32_t* lm_rows = at<int32_t>(ws, L.lm_rows);
  int32_t* cstep = at<int32_t>(ws, L.cstep);
  int32_t* valid = at<int32_t>(ws, L.req_valid);
  int32_t* lm_tok = at<int32_t>(ws, L.lm_tok);
  float* lm_conf = at<float>(ws, L.lm_conf);
  float* x = at<float>(ws, L.x);
  T* h = at<T>(ws, L.h);
  T* q = at<T>(ws, L.q);
  T* kb = at<T>(ws, L.kb);
  T* vb = at<T>(ws, L.vb);
  T* o = at<T>(ws, L.o);
  T* act = at<T>(ws, L.act);
  float* part = at<float>(ws, L.part);
  float* attn_o = at<float>(ws, L.attn_o);
  float* attn_ml = at<float>(ws, L.attn_ml);
  unsigned* attn_cnt = at<unsigned>(ws, kCntOff);  // per (request, kv head), zero between calls
  LmStat* stats = at<LmStat>(ws, L.stats);
  const TC* kc = static_cast<const TC*>(k_cache);
  const TC* vc = static_cast<const TC*>(v_cache);
  // LM-head vocabulary tiles this model holds (all of them unless it is a shard)
  const int n_vt = (m->vocab_hi - m->vocab_lo + kTileN - 1) / kTileN;
  const bool bf16 = c.dtype == DFLASH_BF16;
  int32_t* seg_start = bf16 && g_attn_sched == 1 ? at<int32_t>(ws, L.seg) : nullptr;

  // split-KV chunk: a multiple of the attention tile (64 keys) sized for
  // about four CTAs per SM over the whole (request, kv head, chunk) grid as if
  // every request were at capacity, and at most kMaxChunks chunks per request.
  // Unless a chunk is forced, a planning kernel then picks each forward's
  // chunk (at least this one, so the grid's n_chunks columns cover it) from the
  // actual context lengths, and grid columns past a request's last chunk exit.
  // Without the planner (fp32 models, the persistent schedule) the chunk stays
  // at most 768 keys: each chunk's partial is merged by the last CTA of its
  // request and head.
  const bool forced = g_attn_chunk > 0 && (cap + B + g_attn_chunk - 1) / g_attn_chunk <= kMaxChunks;
  const bool planned = bf16 && g_attn_sched == 0 && !forced && c.n_kv <= 255;
  int chunk = (int)std::min<int64_t>(planned ? INT32_MAX : 768,
                                     (int64_t)(cap + B) * batch * c.n_kv / (4 * num_sms()));
  chunk = std::max(64, (chunk + 63) / 64 * 64);
  chunk = std::max(chunk, (cap + B + kMaxChunks - 1) / kMaxChunks);
  chunk = (chunk + 63) / 64 * 64;
  if (forced) chunk = g_attn_chunk;
  const int n_chunks = (cap + B + chunk - 1) / chunk;
  int32_t* plan_dev = planned ? at<int32_t>(ws, L.attn_chunk) : nullptr;
  const int attn_slots =
      plan_dev ? attn_grid_slots(hd, B * (nq / nkv), B, pg.table != nullptr) : 0;

  if (ph.init)
    launch_draft_init(anchor, ctx_len, batch, B, c.vocab, c.mask_id, cap, pg, tokens, zrow,
                      lm_rows, cstep, valid, err, s);
  auto gemm = [&](const WeightMap& W, const void* wptr, int N, int K, const T* X, float* out,
                  size_t cap_elems, int* splits_out) -> int {
    if (bf16) {
      const int sp = splits_for(M, N, K, cap_elems);
      *splits_out = sp;
      GemmOut go;
      go.part = out;
      const void* seg[1] = {X};
      return gemm_tc(W, seg, 1, K, K, M, sp, EPI_PARTIAL, go, err, s);
    }
    *splits_out = 1;
    const float* seg[1] = {reinterpret_cast<const float*>(X)};
    gemm_simt_f32(static_cast<const float*>(wptr), N, K, seg, 1, K, M, out, s);
    return DFLASH_OK;
  };

  int rem = masked_before(B, n_steps, ph.t0);
  int st = DFLASH_OK;
  for (int t = ph.t0; t < std::min(ph.t1, n_steps); ++t) {
    const int k = (rem + (n_steps - t) - 1) / (n_steps - t);
    const int rows = batch * rem;
    if (!ph.forward) goto choose;
    if (bf16 && g_attn_sched == 1 &&
        (st = launch_attn_plan(ctx_len, valid, batch, nkv, seg_start, s)))
      return st;
    launch_embed_norm<TE, T>(tokens, static_cast<const TE*>(m->emb), m->layers[0].g_in, x, h, M, c.d,
                         c.eps, err, s);
    // planned right before the first QKV GEMM, whose weight prefetch (issued
    // before its dependency wait) covers the planning kernel
    if (plan_dev && (st = launch_attn_chunk_plan(ctx_len, valid, batch, B, nkv, chunk, plan_dev,
                                                  attn_slots, s)))
      return st;
    for (int l = 0; l < c.n_layers; ++l) {
      const LayerPack& P = m->layers[l];
      const float* g_next = l + 1 < c.n_layers ? m->layers[l + 1].g_in : m->g_final;
      const int32_t* next_rows = l + 1 < c.n_layers ? nullptr : zrow;
      if (bf16) {
        // an unsplit GEMM applies the next step in its epilogue; a split one
        // leaves partials (in L2) for the reduction kernel of that step
        GemmOut go;
        go.part = part;
        go.cos_t = m->rope_cos;
        go.sin_t = m->rope_sin;
        go.ctx_len = ctx_len;
        go.req_valid = valid;
        go.B = B;
        go.nq = nq;
        go.nkv = nkv;
        go.hd = hd;
        go.I = c.inter;
        // stream-K (default): every GEMM applies its fused op itself;
        // fixed splits: split GEMMs leave partials for the reduction kernels
        int sp = 1;
        auto run = [&](const WeightMap& W, int N, int K, const void* X, int op) {
          const bool skm = sk_projections();
          sp = skm ? 1 : splits_for(M, N, K, L.part_elems);
          GemmOut g2 = go;
          g2.op = sp == 1 ? op : OP_PARTIAL;
          if (skm) use_stream_k(g2, ws, L.sk);
          const void* seg[1] = {X};
          return gemm_tc(W, seg, 1, K, K, M, skm ? 0 : sp, EPI_PARTIAL, g2, err, s);
        };
        go.h1 = reinterpret_cast<__half*>(q);
        go.h2 = reinterpret_cast<__half*>(kb);
        go.h3 = reinterpret_cast<__half*>(vb);
        if ((st = run(P.mqkv, qkv_out(c), c.d, h, OP_QKV))) return st;
        if (sp > 1)
          launch_qkv_post<T>(part, sp, M, B, ctx_len, valid, nq, nkv, hd, m->rope_cos,
                             m->rope_sin, q, kb, vb, err, s);
        if ((st = launch_block_attention<T, TC>(q, kb, vb, kc, vc, pg, l, c.n_layers, batch, cap,
                                                ctx_len, valid, B, nq, nkv, hd, attn_o, attn_ml,
                                                n_chunks, chunk, plan_dev, seg_start, o, attn_cnt,
                                                err, s)))
          return st;
        go.f32 = x;
        if ((st = run(P.mo, c.d, nq * hd, o, OP_RESID))) return st;
        launch_residual_norm<T>(sp > 1 ? part : nullptr, sp, M, c.d, x, P.g_post, h, nullptr,
                                c.eps, err, s);
        go.h1 = reinterpret_cast<__half*>(act);
        if ((st = run(P.mgu, 2 * c.inter, c.d, h, OP_SWIGLU))) return st;
        if (sp > 1) launch_swiglu<T>(part, sp, M, c.inter, act, err, s);
        if ((st = run(P.md, c.d, c.inter, act, OP_RESID))) return st;
        launch_residual_norm<T>(sp > 1 ? part : nullptr, sp, M, c.d, x, g_next, h, next_rows,
                                c.eps, err, s);
        continue;
      }
      int sp = 1;
      if ((st = gemm(P.mqkv, P.Wqkv, qkv_out(c), c.d, h, part, L.part_elems, &sp))) return st;
      launch_qkv_post<T>(part, sp, M, B, ctx_len, valid, nq, nkv, hd, m->rope_cos, m->rope_sin,
                         q, kb, vb, err, s);
      if ((st = launch_block_attention<T, TC>(q, kb, vb, kc, vc, pg, l, c.n_layers, batch, cap,
                                              ctx_len, valid, B, nq, nkv, hd, attn_o, attn_ml,
                                              n_chunks, chunk, nullptr, nullptr, o, attn_cnt, err,
                                              s)))
        return st;
      if ((st = gemm(P.mo, P.Wo, c.d, nq * hd, o, part, L.part_elems, &sp))) return st;
      launch_residual_norm<T>(part, sp, M, c.d, x, P.g_post, h, nullptr, c.eps, err, s);
      if ((st = gemm(P.mgu, P.Wgu, 2 * c.inter, c.d, h, part, L.part_elems, &sp))) return st;
      launch_swiglu<T>(part, sp, M, c.inter, act, err, s);
      if ((st = gemm(P.md, P.Wd, c.d, c.inter, act, part, L.part_elems, &sp))) return st;
      launch_residual_norm<T>(part, sp, M, c.d, x, g_next, h, next_rows, c.eps, err, s);
    }
    // LM head over the still-masked rows (compact, request-major).  Sampled
    // drafting writes every masked row's logits into the caller's draft-logits
    // rows (a position's row is last written at the step that commits it) and
    // draws from them; greedy drafting reduces the tile statistics.
    {
    void* dbg = logits_dbg ? logits_dbg + (size_t)t * M * c.vocab : nullptr;
    int dbg_bf16 = 0;
    const int32_t* dbg_valid = nullptr;
    if (samp) {
      dbg = samp->q;
      dbg_bf16 = samp->q_bf16;
      dbg_valid = valid;  // a request that writes nothing leaves its rows untouched
    }
    if (bf16) {
      GemmOut go;
      go.stats = stats;
      go.vocab_offset = m->vocab_lo;
      go.dbg = dbg;
      go.dbg_rows = lm_rows;
      go.dbg_ld = c.vocab;
      go.dbg_bf16 = dbg_bf16;
      go.dbg_valid = dbg_valid;
      go.B = B;
      const bool skm = sk_lm_head();
      if (skm) use_stream_k(go, ws, L.sk);
      const void* seg[1] = {h};
      if ((st = gemm_tc(m->mlm, seg, 1, c.d, c.d, rows, skm ? 0 : 1, EPI_LMHEAD, go, err, s)))
        return st;
    } else {
      float* logits = at<float>(ws, L.logits);
      const float* seg[1] = {reinterpret_cast<const float*>(h)};
      gemm_simt_f32(static_cast<const float*>(m->W_lm), c.vocab, c.d, seg, 1, c.d, rows, logits,
                    s);
      launch_lm_stats_from_logits(logits, rows, c.vocab, stats, dbg, lm_rows, c.vocab, dbg_bf16,
                                  dbg_valid, B, s);
    }
    if (ph.shard_stats) {
      // this shard's per-row (max, id, sum): the caller exchanges them
      launch_lm_reduce(stats, n_vt, rows, n_vt, 1, nullptr, nullptr, ph.shard_stats, s);
    } else if (samp) {
      if ((st = launch_sampled_draw(samp->q, samp->q_bf16, lm_rows, valid, rows, B, c.vocab, t,
                                    samp->tau, samp->seed, samp->offset, lm_tok, lm_conf,
                                    at<void>(ws, L.draw), sampled_draw_chunks(rows, c.vocab),
                                    attn_cnt, s)))
        return st;
    } else if (ph.commit) {
      launch_lm_reduce(stats, n_vt, rows, n_vt, 1, lm_tok, lm_conf, nullptr, s);
    }
    }
  choose:
    if (ph.commit) {
      // every shard's statistics, shards in vocabulary order: the argmax over the
      // whole vocabulary and its max-probability
      if (ph.gathered)
        launch_lm_reduce(ph.gathered, ph.world, rows, 1, rows, lm_tok, lm_conf, nullptr, s);
      launch_commit(lm_tok, lm_conf, batch, B, rem, k, t, tokens, zrow, lm_rows, cstep, err, s);
    }
    rem -= k;
  }
  if (ph.finish) launch_draft_finish(tokens, cstep, valid, batch, B, draft_tokens, commit_step, s);
  return cuda_status();
}

}  // namespace

extern "C" int dflash_draft_block(const dflash_model* m, const int32_t* anchor,
                                  const int32_t* ctx_len, const void* k_cache, const void* v_cache,
                                  int cache_cap, int batch, int B, int n_steps,
                                  int32_t* draft_tokens, int32_t* commit_step, float* logits_dbg,
                                  void* ws, size_t ws_bytes, void* stream) {
  NvtxCall nvtx_("dflash_draft_block");
  if (!m || batch < 0 || B < 2 || B > 16 || n_steps < 1 || n_steps > B - 1 || cache_cap < 1)
    return DFLASH_EINVAL;
  if (batch == 0) return DFLASH_OK;
  const dflash_config& c = m->cfg;
  if (!anchor || !ctx_len || !k_cache || !v_cache || !draft_tokens || !ws) return DFLASH_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return DFLASH_EINVAL;
  if (cache_cap > c.max_pos) return DFLASH_EINVAL;
  if (!whole_vocab(m)) return DFLASH_EUNSUPPORTED;  // a shard drafts through the step calls
  if (B * (c.n_q / c.n_kv) > kAttnRows) return DFLASH_EUNSUPPORTED;
  if ((size_t)batch * B > 65535) return DFLASH_EUNSUPPORTED;
  if ((size_t)batch * c.n_kv * 4 > kHeader - kCntOff) return DFLASH_EUNSUPPORTED;
  if (ws_bytes < draft_layout(c, batch, B).end) return DFLASH_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (c.dtype == DFLASH_BF16)
    return draft_impl<__half, __half, __nv_bfloat16>(m, anchor, ctx_len, k_cache, v_cache,
                                                     cache_cap, KvPages{}, batch, B, n_steps,
                                                     draft_tokens, commit_step, logits_dbg,
                                                     nullptr, ws, s);
  return draft_impl<float, float, float>(m, anchor, ctx_len, k_cache, v_cache, cache_cap,
                                         KvPages{}, batch, B, n_steps, draft_tokens, commit_step,
                                         logits_dbg, nullptr, ws, s);
}

extern "C" int dflash_draft_block_paged(const dflash_model* m, const int32_t* anchor,
                                        const int32_t* ctx_len, const void* k_pool,
                                        const void* v_pool, int n_pages, int page_size,
                                        const int32_t* page_table, int max_pages, int batch, int B,
                                        int n_steps, int32_t* draft_tokens, int32_t* commit_step,
                                        float* logits_dbg, void* ws, size_t ws_bytes,
                                        void* stream) {
  NvtxCall nvtx_("dflash_draft_block_paged");
  if (!m || batch < 0 || B < 2 || B > 16 || n_steps < 1 || n_steps > B - 1) return DFLASH_EINVAL;
  if (batch == 0) return DFLASH_OK;
  const dflash_config& c = m->cfg;
  if (!anchor || !ctx_len || !draft_tokens || !ws) return DFLASH_EINVAL;
  if (reinterpret_cast<uintptr_t>(ws) & 255) return DFLASH_EINVAL;
  int st = check_pages(m, k_pool, v_pool, n_pages, page_size, page_table, max_pages);
  if (st) return st;
  if (!whole_vocab(m)) return DFLASH_EUNSUPPORTED;
  if (B * (c.n_q / c.n_kv) > kAttnRows) return DFLASH_EUNSUPPORTED;
  if ((size_t)batch * B > 65535) return DFLASH_EUNSUPPORTED;
  if ((size_t)batch * c.n_kv * 4 > kHeader - kCntOff) return DFLASH_EUNSUPPORTED;
  if (ws_bytes < draft_layout(c, batch, B).end) return DFLASH_EWORKSPACE;
  KvPages pg;
  pg.table = page_table;
  pg.max_pages = max_pages;
  pg.page = page_size;
  pg.n_pages = n_pages;
  // positions a request can reach: its table row, and the RoPE table for the block
  const int cap = (int)std::min<int64_t>((int64_t)max_pages * page_size + B, c.max_pos);
  return draft_impl<__half, __half, __nv_bfloat16>(m, anchor, ctx_len, k_pool, v_pool, cap, pg,
                                                   batch, B, n_steps, draft_tokens, commit_step,
                                                   logits_dbg, nullptr, ws, (cudaStream_t)stream);
}

extern "C" int dflash_draft_block_sampled(const dflash_model* m, const int32_t* anchor,
                                          const int32_t* ctx_len, const void* k_cache,
                                          const void* v_cache, int cache_cap, int batch, int B,
                                          int n_steps, float temperature, uint64_t seed,
                                          uint64_t offset, int32_t* draft_tokens,
                                          int32_t* commit_step, void* draft_logits,
                                          int draft_logits_dtype, void* ws, size_t ws_bytes,
                                          void* stream) {
  NvtxCall nvtx_("dflash_draft_block_sampled");
  if (!m || batch < 0 || B < 2 || B > 16 || n_steps < 1 || n_steps > B - 1 || cache_cap < 1)
    return DFLASH_EINVAL;
  if (!(temperature >= 1e-4f && temperature <= 1e4f)) return DFLASH_EINVAL;
  if (draft_logits_dtype != DFLASH_F32 && draft_logits_dtype != DFLASH_BF16) return DFLASH_EINVAL;
  if (batch == 0) return DFLASH_OK;
  const dflash_config& c = m->cfg;
  if (!anchor || !ctx_len || !k_cache || !v_cache || !draft_tokens || !draft_logits || !ws)
    return DFLASH_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(draft_logits) ||
      (reinterpret_cast<uintptr_t>(ws) & 255))
    return DFLASH_EINVAL;
  if (cache_cap > c.max_pos) return DFLASH_EINVAL;
  if (!whole_vocab(m)) return DFLASH_EUNSUPPORTED;
  if (B * (c.n_q / c.n_kv) > kAttnRows) return DFLASH_EUNSUPPORTED;
  // one completion counter per masked row of the draw
  if ((size_t)batch * B * 4 > kHeader - kCntOff) return DFLASH_EUNSUPPORTED;
  if ((size_t)batch * c.n_kv * 4 > kHeader - kCntOff) return DFLASH_EUNSUPPORTED;
  if (ws_bytes < draft_layout(c, batch, B).end) return DFLASH_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  SampleArgs sa{temperature, seed, offset, draft_logits, draft_logits_dtype == DFLASH_BF16};
  if (c.dtype == DFLASH_BF16)
    return draft_impl<__half, __half, __nv_bfloat16>(m, anchor, ctx_len, k_cache, v_cache,
                                                     cache_cap, KvPages{}, batch, B, n_steps,
                                                     draft_tokens, commit_step, nullptr, &sa, ws,
                                                     s);
  return draft_impl<float, float, float>(m, anchor, ctx_len, k_cache, v_cache, cache_cap,
                                         KvPages{}, batch, B, n_steps, draft_tokens, commit_step,
                                         nullptr, &sa, ws, s);
}

// ============================================================== vocabulary-parallel draft
namespace {

// Shared host checks of the draft step calls (contiguous K/V, bf16 models).
int check_steps(const dflash_model* m, int batch, int B, int n_steps, int step, void* ws,
                size_t ws_bytes) {
  if (!m || batch < 1 || B < 2 || B > 16 || n_steps < 1 || n_steps > B - 1) return DFLASH_EINVAL;
  if (step < 0 || step >= n_steps || !ws || (reinterpret_cast<uintptr_t>(ws) & 255))
    return DFLASH_EINVAL;
  const dflash_config& c = m->cfg;
  if (c.dtype != DFLASH_BF16) return DFLASH_EUNSUPPORTED;
  if (B * (c.n_q / c.n_kv) > kAttnRows) return DFLASH_EUNSUPPORTED;
  if ((size_t)batch * B > 65535) return DFLASH_EUNSUPPORTED;
  if ((size_t)batch * c.n_kv * 4 > kHeader - kCntOff) return DFLASH_EUNSUPPORTED;
  if (ws_bytes < draft_layout(c, batch, B).end) return DFLASH_EWORKSPACE;
  return DFLASH_OK;
}

int run_phase(const dflash_model* m, const int32_t* anchor, const int32_t* ctx_len,
              const void* k_cache, const void* v_cache, int cap, int batch, int B, int n_steps,
              int32_t* draft_tokens, int32_t* commit_step, void* ws, void* stream,
              const DraftPhase& ph) {
  return draft_impl<__half, __half, __nv_bfloat16>(m, anchor, ctx_len, k_cache, v_cache, cap,
                                                   KvPages{}, batch, B, n_steps, draft_tokens,
                                                   commit_step, nullptr, nullptr, ws,
                                                   (cudaStream_t)stream, ph);
}

}  // namespace

extern "C" int dflash_draft_rows(int batch, int B, int n_steps, int step) {
  if (batch < 1 || B < 2 || n_steps < 1 || n_steps > B - 1 || step < 0 || step >= n_steps)
    return DFLASH_EINVAL;
  return batch * masked_before(B, n_steps, step);
}

extern "C" int dflash_draft_begin(const dflash_model* m, const int32_t* anchor,
                                  const int32_t* ctx_len, int cache_cap, int batch, int B,
                                  int n_steps, void* ws, size_t ws_bytes, void* stream) {
  NvtxCall nvtx_("dflash_draft_begin");
  int st = check_steps(m, batch, B, n_steps, 0, ws, ws_bytes);
  if (st) return st;
  if (!anchor || !ctx_len || cache_cap < 1 || cache_cap > m->cfg.max_pos) return DFLASH_EINVAL;
  DraftPhase ph;
  ph.forward = ph.commit = ph.finish = false;
  ph.t1 = 0;
  return run_phase(m, anchor, ctx_len, nullptr, nullptr, cache_cap, batch, B, n_steps, nullptr,
                   nullptr, ws, stream, ph);
}

extern "C" int dflash_draft_forward_shard(const dflash_model* m, const int32_t* ctx_len,
                                          const void* k_cache, const void* v_cache,
                                          int cache_cap, int batch, int B, int n_steps, int step,
                                          void* shard_stats, void* ws, size_t ws_bytes,
                                          void* stream) {
  NvtxCall nvtx_("dflash_draft_forward_shard");
  int st = check_steps(m, batch, B, n_steps, step, ws, ws_bytes);
  if (st) return st;
  if (!ctx_len || !k_cache || !v_cache || !shard_stats || cache_cap < 1 ||
      cache_cap > m->cfg.max_pos)
    return DFLASH_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(shard_stats)) return DFLASH_EINVAL;
  DraftPhase ph;
  ph.init = ph.commit = ph.finish = false;
  ph.t0 = step;
  ph.t1 = step + 1;
  ph.shard_stats = static_cast<LmStat*>(shard_stats);
  return run_phase(m, nullptr, ctx_len, k_cache, v_cache, cache_cap, batch, B, n_steps, nullptr,
                   nullptr, ws, stream, ph);
}

extern "C" int dflash_draft_commit_shards(const dflash_model* m, const void* gathered, int world,
                                          int batch, int B, int n_steps, int step, void* ws,
                                          size_t ws_bytes, void* stream) {
  NvtxCall nvtx_("dflash_draft_commit_shards");
  int st = check_steps(m, batch, B, n_steps, step, ws, ws_bytes);
  if (st) return st;
  if (!gathered || world < 1 || !aligned16(gathered)) return DFLASH_EINVAL;
  DraftPhase ph;
  ph.init = ph.forward = ph.finish = false;
  ph.t0 = step;
  ph.t1 = step + 1;
  ph.gathered = static_cast<const LmStat*>(gathered);
  ph.world = world;
  // cap only sizes the attention chunks, which this phase does not launch
  return run_phase(m, nullptr, nullptr, nullptr, nullptr, m->cfg.max_pos, batch, B, n_steps,
                   nullptr, nullptr, ws, stream, ph);
}

extern "C" int dflash_draft_end(const dflash_model* m, int batch, int B, int n_steps,
                                int32_t* draft_tokens, int32_t* commit_step, void* ws,
                                size_t ws_bytes, void* stream) {
  NvtxCall nvtx_("dflash_draft_end");
  int st = check_steps(m, batch, B, n_steps, 0, ws, ws_bytes);
  if (st) return st;
  if (!draft_tokens) return DFLASH_EINVAL;
  DraftPhase ph;
  ph.init = ph.forward = ph.commit = false;
  ph.t1 = 0;
  return run_phase(m, nullptr, nullptr, nullptr, nullptr, m->cfg.max_pos, batch, B, n_steps,
                   draft_tokens, commit_step, ws, stream, ph);
}

// ============================================================== verify
extern "C" int dflash_verify(const void* target_logits, int logits_dtype,
                             const int32_t* draft_tokens, int batch, int B, int V,
                             int32_t* out_tokens, int32_t* out_len, int out_cap, int32_t* seq_lens,
                             int32_t* accept_len, int32_t* next_anchor, void* ws, size_t ws_bytes,
                             void* stream) {
  NvtxCall nvtx_("dflash_verify");
  if (batch < 0 || B < 2 || B > 32 || V < 1 || out_cap < 1) return DFLASH_EINVAL;
  if (logits_dtype != DFLASH_BF16 && logits_dtype != DFLASH_F32) return DFLASH_EINVAL;
  if (batch == 0) return DFLASH_OK;
  if (!target_logits || !draft_tokens || !out_tokens || !out_len || !seq_lens || !accept_len ||
      !next_anchor || !ws)
    return DFLASH_EINVAL;
  if (!aligned16(target_logits) || (reinterpret_cast<uintptr_t>(ws) & 255)) return DFLASH_EINVAL;
  if ((int64_t)batch * B > 65535) return DFLASH_EUNSUPPORTED;
  if (ws_bytes < verify_bytes(batch, B, V)) return DFLASH_EWORKSPACE;
  const int chunks = verify_chunks(batch * B, V);
  return launch_verify(target_logits, logits_dtype, draft_tokens, batch, B, V, out_tokens,
                       out_len, out_cap, seq_lens, accept_len, next_anchor,
                       at<void>(ws, kHeader), chunks, at<unsigned>(ws, kCntOff), err_word(ws),
                       (cudaStream_t)stream);
}

// ============================================================== vocabulary-parallel verify
extern "C" int dflash_verify_shard(const void* logits_shard, int logits_dtype, int batch, int B,
                                   int Vs, int vocab_offset, void* row_argmax, void* ws,
                                   size_t ws_bytes, void* stream) {
  NvtxCall nvtx_("dflash_verify_shard");
  if (batch < 0 || B < 2 || B > 32 || Vs < 1 || vocab_offset < 0) return DFLASH_EINVAL;
  if (logits_dtype != DFLASH_BF16 && logits_dtype != DFLASH_F32) return DFLASH_EINVAL;
  if ((int64_t)vocab_offset + Vs > 0x7fffffffLL) return DFLASH_EINVAL;
  if (batch == 0) return DFLASH_OK;
  if (!logits_shard || !row_argmax || !ws) return DFLASH_EINVAL;
  if (!aligned16(logits_shard) || (reinterpret_cast<uintptr_t>(ws) & 255)) return DFLASH_EINVAL;
  if ((int64_t)batch * B > 65535) return DFLASH_EUNSUPPORTED;
  if (ws_bytes < verify_bytes(batch, B, Vs)) return DFLASH_EWORKSPACE;
  const int chunks = verify_chunks(batch * B, Vs);
  return launch_verify_shard(logits_shard, logits_dtype, batch, B, Vs, vocab_offset,
                             static_cast<ArgPart*>(row_argmax), at<void>(ws, kHeader), chunks,
                             at<unsigned>(ws, kCntOff), (cudaStream_t)stream);
}

extern "C" int dflash_verify_merge(const void* gathered, int world, const int32_t* draft_tokens,
                                   int batch, int B, int V, int32_t* out_tokens, int32_t* out_len,
                                   int out_cap, int32_t* seq_lens, int32_t* accept_len,
                                   int32_t* next_anchor, void* ws, size_t ws_bytes,
                                   void* stream) {
  NvtxCall nvtx_("dflash_verify_merge");
  if (batch < 0 || B < 2 || B > 32 || V < 1 || out_cap < 1 || world < 1) return DFLASH_EINVAL;
  if (batch == 0) return DFLASH_OK;
  if (!gathered || !draft_tokens || !out_tokens || !out_len || !seq_lens || !accept_len ||
      !next_anchor || !ws)
    return DFLASH_EINVAL;
  if (!aligned16(gathered) || (reinterpret_cast<uintptr_t>(ws) & 255)) return DFLASH_EINVAL;
  if (ws_bytes < kHeader) return DFLASH_EWORKSPACE;
  return launch_verify_merge(static_cast<const ArgPart*>(gathered), world, draft_tokens, batch, B,
                             V, out_tokens, out_len, out_cap, seq_lens, accept_len, next_anchor,
                             err_word(ws), (cudaStream_t)stream);
}

// ============================================================== sampled verify
extern "C" size_t dflash_verify_sampled_workspace_size(int batch, int B, int V) {
  if (batch < 0 || B < 0 || V < 1) return 0;
  if (batch == 0 || B == 0) return kHeader;
  return kHeader + sampled_verify_bytes(batch, B, V);
}

extern "C" int dflash_verify_sampled(const void* target_logits, const void* draft_logits,
                                     int logits_dtype, const int32_t* draft_tokens, int batch,
                                     int B, int V, float temperature, uint64_t seed,
                                     uint64_t offset, int32_t* out_tokens, int32_t* out_len,
                                     int out_cap, int32_t* seq_lens, int32_t* accept_len,
                                     int32_t* next_anchor, void* ws, size_t ws_bytes,
                                     void* stream) {
  NvtxCall nvtx_("dflash_verify_sampled");
  if (batch < 0 || B < 2 || B > 32 || V < 1 || out_cap < 1) return DFLASH_EINVAL;
  if (logits_dtype != DFLASH_BF16 && logits_dtype != DFLASH_F32) return DFLASH_EINVAL;
  if (!(temperature >= 1e-4f && temperature <= 1e4f)) return DFLASH_EINVAL;
  if (batch == 0) return DFLASH_OK;
  if (!target_logits || !draft_logits || !draft_tokens || !out_tokens || !out_len || !seq_lens ||
      !accept_len || !next_anchor || !ws)
    return DFLASH_EINVAL;
  if (!aligned16(target_logits) || !aligned16(draft_logits) ||
      (reinterpret_cast<uintptr_t>(ws) & 255))
    return DFLASH_EINVAL;
  // target and draft rows share one grid dimension
  if ((int64_t)2 * batch * B > 65535) return DFLASH_EUNSUPPORTED;
  if (ws_bytes < kHeader + sampled_verify_bytes(batch, B, V)) return DFLASH_EWORKSPACE;
  return launch_sampled_verify(target_logits, draft_logits, logits_dtype, draft_tokens, batch, B,
                               V, temperature, seed, offset, out_tokens, out_len, out_cap,
                               seq_lens, accept_len, next_anchor, at<void>(ws, kHeader),
                               at<unsigned>(ws, kCntOff), err_word(ws), (cudaStream_t)stream);
}

// ============================================================== test hooks (dflash_debug.h)
#include "../../include/dflash_debug.h"

extern "C" int dflash_debug_gemm(const void* W, int N, int K, const void* X, int M, int elem,
                                 int splits, float* out, int* splits_used, void* err_ws,
                                 void* stream) {
  if (!W || !X || !out || !err_ws || N < 1 || K < 64 || K % 64 || M < 1) return DFLASH_EINVAL;
  if (!aligned16(W) || !aligned16(X)) return DFLASH_EINVAL;
  WeightMap wm;
  if (elem != DFLASH_BF16 && elem != DFLASH_F16) return DFLASH_EINVAL;
  if (!encode_weight_map(wm, W, N, K, elem)) return DFLASH_ECUDA;
  splits = gemm_effective_splits(K, splits);
  if (splits_used) *splits_used = splits;
  GemmOut o;
  o.part = out;
  const void* seg[1] = {X};
  return gemm_tc(wm, seg, 1, K, K, M, splits, EPI_PARTIAL, o, err_word(err_ws),
                 (cudaStream_t)stream);
}

extern "C" int dflash_debug_gemm_tiled(const void* Wt, int N, int K, const void* X, int M,
                                       int elem, int splits, float* out, int* splits_used,
                                       void* err_ws, void* stream) {
  if (!Wt || !X || !out || !err_ws || N < 1 || K < 64 || K % 64 || M < 1) return DFLASH_EINVAL;
  if (!aligned16(Wt) || !aligned16(X)) return DFLASH_EINVAL;
  if (elem != DFLASH_BF16 && elem != DFLASH_F16) return DFLASH_EINVAL;
  WeightMap wm;
  memset(&wm.map, 0, sizeof(wm.map));
  wm.N = N;
  wm.K = K;
  wm.elem = elem;
  if (!set_tiled_weights(wm, Wt)) return DFLASH_ECUDA;
  splits = gemm_effective_splits(K, splits);
  if (splits_used) *splits_used = splits;
  GemmOut o;
  o.part = out;
  const void* seg[1] = {X};
  return gemm_tc(wm, seg, 1, K, K, M, splits, EPI_PARTIAL, o, err_word(err_ws),
                 (cudaStream_t)stream);
}

extern "C" size_t dflash_debug_gemm_streamk_ws_bytes(int M) {
  if (M < 1) return 0;
  return kHeader + align256(gemm_sk_slot_bytes(M));
}

extern "C" int dflash_debug_gemm_streamk(const void* Wt, int N, int K, const void* X, int M,
                                         int elem, float* out, void* ws, size_t ws_bytes,
                                         void* stream) {
  if (!Wt || !X || !out || !ws || N < 1 || K < 64 || K % 64 || M < 1) return DFLASH_EINVAL;
  if (!aligned16(Wt) || !aligned16(X) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return DFLASH_EINVAL;
  if (elem != DFLASH_BF16 && elem != DFLASH_F16) return DFLASH_EINVAL;
  if (ws_bytes < kHeader + gemm_sk_slot_bytes(M)) return DFLASH_EWORKSPACE;
  WeightMap wm;
  memset(&wm.map, 0, sizeof(wm.map));
  wm.N = N;
  wm.K = K;
  wm.elem = elem;
  if (!set_tiled_weights(wm, Wt)) return DFLASH_ECUDA;
  GemmOut o;
  o.op = OP_STORE;
  o.f32 = out;
  use_stream_k(o, ws, kHeader);
  const void* seg[1] = {X};
  return gemm_tc(wm, seg, 1, K, K, M, 0, EPI_PARTIAL, o, err_word(ws), (cudaStream_t)stream);
}

extern "C" size_t dflash_debug_tiled_bytes(int N, int K) {
  if (N < 1 || K < 64 || K % 64) return 0;
  return tiled_bytes(N, K);
}

extern "C" int dflash_debug_tile_weights(const void* W, void* Wt, int N, int K, void* stream) {
  if (!W || !Wt || N < 1 || K < 64 || K % 64 || !aligned16(W) || !aligned16(Wt))
    return DFLASH_EINVAL;
  tile_weights(W, Wt, N, K, (cudaStream_t)stream);
  return cuda_status();
}

namespace {
// One thread waits, through the library's bounded mbarrier wait, for a phase
// that no arrival ever completes: after the wait limit it gives up and sets
// DFLASH_DEV_TIMEOUT, as every pipeline wait of the library does.
__global__ void debug_timeout_kernel(int32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    if (!mbar_wait(smem_u32(&bar), 0)) set_error(err, DFLASH_DEV_TIMEOUT);
  }
}
}  // namespace

extern "C" int dflash_debug_wait_timeout(void* err_ws, void* stream) {
  if (!err_ws || (reinterpret_cast<uintptr_t>(err_ws) & 255)) return DFLASH_EINVAL;
  debug_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(err_word(err_ws));
  return cuda_status();
}

extern "C" int dflash_debug_sample_math(const uint64_t* w, const float* d, int n, float* g2,
                                        float* l2, void* stream) {
  if (n < 0 || (n > 0 && (!w || !d || !g2 || !l2))) return DFLASH_EINVAL;
  return launch_sample_math(w, d, n, g2, l2, (cudaStream_t)stream);
}

extern "C" int dflash_debug_pick_splits(int M, int N, int K) {
  if (M < 1 || N < 1 || K < 64 || K % 64) return DFLASH_EINVAL;
  return gemm_pick_splits(M, N, K, kMaxSplits);
}

extern "C" int dflash_debug_attn_chunk(int keys) {
  if (keys < 0 || keys % 64 != 0) return DFLASH_EINVAL;
  g_attn_chunk = keys;
  return DFLASH_OK;
}

extern "C" int dflash_debug_attn_plan(const int32_t* ctx_len, const int32_t* req_valid, int batch,
                                      int B, int n_kv, int cap, int chunk_min, int slots,
                                      int32_t* plan_out, long long plan_cap, void* stream) {
  if (!ctx_len || !req_valid || !plan_out || batch <= 0 || B <= 0 || n_kv <= 0 || n_kv > 255 ||
      slots <= 0 || cap < B || chunk_min <= 0 || chunk_min % 64 != 0 ||
      (cap + chunk_min - 1) / chunk_min > 255)
    return DFLASH_EINVAL;
  if (plan_cap < 4 + 2LL * batch * n_kv * ((cap + chunk_min - 1) / chunk_min) ||
      (reinterpret_cast<uintptr_t>(plan_out) & 7) != 0)
    return DFLASH_EINVAL;
  return launch_attn_chunk_plan(ctx_len, req_valid, batch, B, n_kv, chunk_min, plan_out, slots,
                                (cudaStream_t)stream);
}

extern "C" int dflash_debug_attn_slots(int head_dim, int rows, int B) {
  if (head_dim <= 0 || rows <= 0 || B <= 0) return DFLASH_EINVAL;
  return attn_grid_slots(head_dim, rows, B, false);
}

extern "C" int dflash_debug_split_weight(float w) {
  if (!(w >= 0.f && w <= 64.f)) return DFLASH_EINVAL;
  gemm_set_split_weight(w);
  return DFLASH_OK;
}

extern "C" int dflash_debug_attn_schedule(int sched) {
  if (sched < 0 || sched > 2) return DFLASH_EINVAL;
  g_attn_sched = sched == 1 ? 1 : 0;
  g_attn_umma = sched == 2 ? 1 : 0;
  return DFLASH_OK;
}

extern "C" int dflash_debug_gemm_schedule(int sched) {
  if (sched < 0 || sched > 2) return DFLASH_EINVAL;
  g_gemm_sched = sched;
  return DFLASH_OK;
}

extern "C" int dflash_debug_gemm_mode(int mode) {
  if (mode < 0 || mode > 2) return DFLASH_EINVAL;
  gemm_set_mode(mode);
  return DFLASH_OK;
}

extern "C" int dflash_debug_lmhead_tiled(const void* Wt, int N, int K, const void* X, int M,
                                         int elem, void* stats, float* logits, void* err_ws,
                                         void* stream) {
  if (!Wt || !X || !stats || !err_ws || N < 1 || K < 64 || K % 64 || M < 1) return DFLASH_EINVAL;
  if (!aligned16(Wt) || !aligned16(X)) return DFLASH_EINVAL;
  if (elem != DFLASH_BF16 && elem != DFLASH_F16) return DFLASH_EINVAL;
  WeightMap wm;
  memset(&wm.map, 0, sizeof(wm.map));
  wm.N = N;
  wm.K = K;
  wm.elem = elem;
  if (!set_tiled_weights(wm, Wt)) return DFLASH_ECUDA;
  GemmOut o;
  o.stats = static_cast<LmStat*>(stats);
  o.dbg = logits;
  o.dbg_rows = nullptr;
  o.dbg_ld = N;
  const void* seg[1] = {X};
  return gemm_tc(wm, seg, 1, K, K, M, 1, EPI_LMHEAD, o, err_word(err_ws), (cudaStream_t)stream);
}

extern "C" int dflash_debug_lmhead(const void* W, int N, int K, const void* X, int M, int elem,
                                   void* stats, float* logits, void* err_ws, void* stream) {
  if (!W || !X || !stats || !err_ws || N < 1 || K < 64 || K % 64 || M < 1) return DFLASH_EINVAL;
  if (!aligned16(W) || !aligned16(X)) return DFLASH_EINVAL;
  WeightMap wm;
  if (elem != DFLASH_BF16 && elem != DFLASH_F16) return DFLASH_EINVAL;
  if (!encode_weight_map(wm, W, N, K, elem)) return DFLASH_ECUDA;
  GemmOut o;
  o.stats = static_cast<LmStat*>(stats);
  o.dbg = logits;
  o.dbg_rows = nullptr;
  o.dbg_ld = N;
  const void* seg[1] = {X};
  return gemm_tc(wm, seg, 1, K, K, M, 1, EPI_LMHEAD, o, err_word(err_ws), (cudaStream_t)stream);
}
