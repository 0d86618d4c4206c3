// Greedy verify for callers that cannot allocate device memory.
//
// Some hosts own every byte of device memory through their own pool (an
// inference server that reserves its arena at start-up and forbids later
// allocation, or a plugin running inside another framework's allocator), and
// latency-critical loops avoid cudaMalloc because it may synchronise the
// device.  Such callers cannot provide the workspace dflash_verify needs.
// dflash_verify_noalloc runs the same kernel with its scratch (the per-chunk
// argmax partials, the per-request completion counters and the device error
// word) in a fixed array in the library's own device memory.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dflash {
namespace {

// Scratch of the no-alloc verify: a 256-byte header (word 0 = device error
// bits), the argmax partials (8 bytes each), then one completion counter per
// request.  The counters start at zero (device globals are zero-initialised)
// and every call leaves them at zero.  Every GPU that loads the library holds
// this array until the process exits.
constexpr size_t kNoAllocHeader = 256;
constexpr size_t kNoAllocPart = size_t(256) << 10;  // 256 KiB of partials: <= 32768 rows
constexpr size_t kNoAllocCnt = size_t(64) << 10;    // 16384 requests (B >= 2 with <= 32768 rows)
constexpr size_t kNoAllocBytes = kNoAllocHeader + kNoAllocPart + kNoAllocCnt;
static __device__ __align__(256) unsigned char g_verify_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DFLASH_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || p == nullptr)
      return DFLASH_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return DFLASH_OK;
}

__global__ void copy_error_word(const int32_t* __restrict__ src, int32_t* __restrict__ dst) {
  pdl_trigger();
  pdl_wait();
  *dst = *src;
}

}  // namespace
}  // namespace dflash

using namespace dflash;

extern "C" int dflash_verify_noalloc(const void* target_logits, int logits_dtype,
                                     const int32_t* draft_tokens, int batch, int B, int V,
                                     int32_t* out_tokens, int32_t* out_len, int out_cap,
                                     int32_t* seq_lens, int32_t* accept_len,
                                     int32_t* next_anchor, int32_t* error_bits, void* stream) {
  if (batch < 0 || B < 2 || B > 32 || V < 1 || out_cap < 1) return DFLASH_EINVAL;
  if (logits_dtype != DFLASH_BF16 && logits_dtype != DFLASH_F32) return DFLASH_EINVAL;
  if (batch == 0) return DFLASH_OK;
  if (!target_logits || !draft_tokens || !out_tokens || !out_len || !seq_lens || !accept_len ||
      !next_anchor)
    return DFLASH_EINVAL;
  if ((reinterpret_cast<uintptr_t>(target_logits) & 15) != 0) return DFLASH_EINVAL;
  if ((int64_t)batch * B > 65535) return DFLASH_EUNSUPPORTED;
  const int rows = batch * B;
  const int chunks = verify_chunks(rows, V);
  if ((size_t)rows * chunks * 8 > kNoAllocPart || (size_t)batch * 4 > kNoAllocCnt)
    return DFLASH_ESCRATCH;
  void* scratch = nullptr;
  int st = scratch_address(&scratch);
  if (st != DFLASH_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* err = static_cast<int32_t*>(scratch);
  // the array keeps the previous call's contents: the error word must start at zero
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess) return DFLASH_ECUDA;
  unsigned char* base = static_cast<unsigned char*>(scratch);
  st = launch_verify(target_logits, logits_dtype, draft_tokens, batch, B, V, out_tokens, out_len,
                     out_cap, seq_lens, accept_len, next_anchor, base + kNoAllocHeader, chunks,
                     reinterpret_cast<unsigned*>(base + kNoAllocHeader + kNoAllocPart), err, s);
  if (st != DFLASH_OK) return st;
  if (error_bits) {
    launch_pdl(copy_error_word, dim3(1), dim3(1), 0, s, 1, err, error_bits);
    if (cudaGetLastError() != cudaSuccess) return DFLASH_ECUDA;
  }
  return DFLASH_OK;
}
