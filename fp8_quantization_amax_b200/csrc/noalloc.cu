// fp8_kv_quantize_noalloc: the KV-cache quantizer for callers that cannot allocate device
// memory.
//
// Who needs it: code that runs where a cudaMalloc is not allowed or not possible -- inside an
// allocator-free runtime (a serving engine that owns all device memory up front and hands out
// only fixed tensors), in a real-time path where an allocation could stall or fail, or in a
// plug-in whose host API gives it tensors but no way to ask for workspace.  The regular
// fp8_kv_quantize needs a caller-provided workspace for the per-CTA partial maxima of its
// two-pass granularities; this entry point instead keeps that scratch in a fixed array that
// lives in the library's own device memory.
//
// The scratch: g_kv_partials below, kNoAllocMaxHeads heads' worth (256 KB), one copy on every
// GPU that loads the library, held until the process exits.  Its device address is looked up
// once per device with cudaGetSymbolAddress on the first call on that device (with the device
// current), so that first call should happen before any stream capture.  Pass 1 overwrites
// every entry pass 2 reads, so nothing needs to be cleared between calls; but all calls share
// the one array, so two calls whose kernels overlap on the GPU (different streams, no ordering
// between them) race on it and must not be issued.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp8q.h"
#include "internal.h"

namespace {

constexpr int64_t kNoAllocMaxHeads = 32;
constexpr size_t kScratchFloats = (size_t)fp8q::kMaxPartials * 2 * kNoAllocMaxHeads;

static __device__ __align__(256) float g_kv_partials[kScratchFloats];

// device address of g_kv_partials on the current device; nullptr if it cannot be resolved
float* scratch_address() {
  static float* cache[128] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kv_partials) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<float*>(p);
  }
  return cache[dev];
}

}  // namespace

extern "C" {

fp8q_status fp8_kv_quantize_noalloc(const void* k, const void* v, int64_t tokens, int64_t heads, int64_t head_dim,
                                    fp8q_format f, fp8q_kv_granularity g, uint8_t* k_codes, uint8_t* v_codes,
                                    float* k_scales, float* v_scales, fp8q_stream_t stream) {
  // the per-head partials need 2 * heads floats per pass-1 CTA; refuse what the array cannot hold
  if (g == FP8Q_KV_PER_HEAD && heads > kNoAllocMaxHeads) return FP8Q_ERR_WORKSPACE;
  const size_t need = fp8q_kv_workspace_bytes(tokens, heads, head_dim, g);
  if (need > kScratchFloats * sizeof(float)) return FP8Q_ERR_WORKSPACE;
  float* ws = nullptr;
  if (need > 0) {
    ws = scratch_address();
    if (!ws) return FP8Q_ERR_CUDA;
  }
  return fp8_kv_quantize(k, v, tokens, heads, head_dim, f, g, k_codes, v_codes, k_scales, v_scales, ws,
                         need > 0 ? kScratchFloats * sizeof(float) : 0, stream);
}

}  // extern "C"
