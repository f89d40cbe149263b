// Decode attention for callers that cannot allocate device memory.
//
// headq_decode_attn needs a caller-provided workspace for the per-split partial
// results.  Some callers have no way to obtain one: code running inside a
// CUDA-graph replay or a custom allocator's own hooks, plugins handed only
// input/output buffers by a host framework, or environments where cudaMalloc is
// forbidden after start-up.  headq_decode_attn_noalloc serves them by using a
// fixed scratch array that is part of the library image itself
// (kNoAllocScratchBytes per GPU, resident on every GPU that loads the library
// until the process exits) and otherwise runs the exact same code as
// headq_decode_attn.
#include <mutex>

#include "headq_internal.cuh"

#define HEADQ_API extern "C" __attribute__((visibility("default")))

namespace headq {
namespace {

// 4 MiB covers the five reference decode layers at full size (the largest,
// batch 64 x 28 heads, needs about 1.9 MB of partials).
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: the address is looked up per device below.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices];  // device address per device, set once

// Once per device, with that device current: find the array's device address
// and zero it (the device error word and the split arrival counters must start
// at zero; every decode call leaves the counters at zero again).  Synchronous.
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) return e;
    e = cudaMemset(ptr, 0, kNoAllocScratchBytes);
    if (e != cudaSuccess) return e;
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace headq

using namespace headq;

HEADQ_API headq_status headq_decode_attn_noalloc(const headq_cache* cache, const void* q,
                                                 headq_dtype q_dtype, int Hq,
                                                 const int32_t* seq_lens, int T,
                                                 const float* U, float sm_scale,
                                                 int corr_sign, float* out, float* lse,
                                                 headq_stream_t stream) {
  const size_t need = headq_decode_workspace_bytes(cache, Hq, T);
  if (need > kNoAllocScratchBytes) return HEADQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) {
    cudaGetLastError();
    return HEADQ_ERR_CUDA;
  }
  return headq_decode_attn(cache, q, q_dtype, Hq, seq_lens, T, U, sm_scale, corr_sign, out,
                           lse, scratch, kNoAllocScratchBytes, stream);
}

// The device error word of the built-in scratch (its first 4 bytes, as in a
// caller workspace).  A no-alloc call whose kernel gave up a bounded wait or met
// a block-table entry outside the page pool raises it, exactly as it would in a
// caller workspace; the caller never sees the array's address, so this call
// reads and clears the word of the current device for it.
HEADQ_API headq_status headq_decode_noalloc_status(headq_stream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return HEADQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return HEADQ_ERR_CUDA;
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    ptr = g_scratch_addr[dev];
  }
  if (ptr == nullptr) return HEADQ_OK;  // no no-alloc call has run on this device
  return headq_workspace_status(ptr, stream);
}
