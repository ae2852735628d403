// kvq_noalloc.cu -- decode attention for callers that cannot allocate.
//
// kvq_decode_attention needs a caller-provided device workspace for its
// per-split partial records.  Some callers have no way to provide one: code
// running inside a host framework whose callback contract forbids device
// allocation (an inference-engine plugin's enqueue, for instance), or a
// latency-critical decode loop that must never call cudaMalloc, which can
// block and synchronise the device.  kvq_decode_attention_noalloc serves
// them: it is the same computation, but the partial records live in the
// fixed-size scratch array below, which the library owns.
//
// The array is a file-scope __device__ variable, so every GPU that loads
// libkvq.so holds kScratchBytes of device memory for it until the process
// exits.  Host code must not pass the array's name to a kernel (on the host
// that name is only a stand-in); the device address is resolved with
// cudaGetSymbolAddress, once per device, by the first call made while that
// device is current.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "kvq.h"
#include "kvq_internal.h"

constexpr size_t kScratchBytes = size_t(4) << 20;   // 4 MiB

// The scratch for the partial records (file scope, one per device).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (resolved on
// the first call per device).
cudaError_t scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int kvq_decode_attention_noalloc(kvq_cache_t cache, int layer, const void* q,
                                            int q_heads, float softmax_scale, float* out,
                                            void* stream) {
  if (!cache) return kvq::report_error(KVQ_ERR_INVALID_ARG, "kvq_decode_attention_noalloc: null cache");
  const size_t need = kvq_workspace_bytes(cache, q_heads);
  if (need == 0) return kvq_decode_attention(cache, layer, q, q_heads, softmax_scale, out, nullptr,
                                             0, stream);   // reports the argument error
  if (need > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "kvq_decode_attention_noalloc: this cache and q_heads=%d may need %zu bytes of "
             "scratch; the built-in scratch holds %zu (use kvq_decode_attention with a workspace)",
             q_heads, need, kScratchBytes);
    return kvq::report_error(KVQ_ERR_WORKSPACE, msg);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess && (dev < 0 || dev >= kMaxDevices)) e = cudaErrorInvalidDevice;
  void* scratch = nullptr;
  if (e == cudaSuccess) e = scratch_address(dev, &scratch);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "kvq_decode_attention_noalloc: scratch set-up failed: %s",
             cudaGetErrorString(e));
    return kvq::report_error(KVQ_ERR_CUDA, msg);
  }
  // The records in the scratch are always written before they are read
  // within one call, so nothing in it has to start at zero; the completion
  // counters live in the cache buffer and are zero between calls.
  return kvq_decode_attention(cache, layer, q, q_heads, softmax_scale, out, scratch, kScratchBytes,
                              stream);
}
