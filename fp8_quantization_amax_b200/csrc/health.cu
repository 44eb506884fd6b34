// Scale health (charles2530.github.io "量化：FP8 与混合精度推理", "scale 是控制面": the scales and
// the overflow / underflow they cause should be observable).
//   k_scale_hist       256-bucket histogram of scales by power of two: fp32 scales by their
//                      biased exponent field (0: zero or subnormal, 255: Inf / NaN), MX scale
//                      bytes by value; per-block shared bins, one global add per non-empty bin.
//   k_count_underflow  nonzero, non-NaN bf16 inputs whose FP8 code is +-0: 16-byte loads of x and
//                      8-byte loads of the codes, one 64-bit atomic per block.  HBM-bound
//                      (3 bytes read per element).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "internal.h"

namespace fp8q {
namespace {

constexpr int kHistThreads = 256;

template <int KIND>
__global__ void __launch_bounds__(kHistThreads) k_scale_hist(const void* __restrict__ scales, int64_t n,
                                                           uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[256];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    uint32_t b;
    if constexpr (KIND == 0)
      b = (__float_as_uint(__ldg(static_cast<const float*>(scales) + i)) >> 23) & 0xFFu;
    else
      b = __ldg(static_cast<const uint8_t*>(scales) + i);
    atomicAdd(&h[b], 1u);
  }
  __syncthreads();
  if (h[threadIdx.x]) atomicAdd(&hist[threadIdx.x], h[threadIdx.x]);
}

__device__ __forceinline__ uint32_t underflow8(uint4 x, uint2 c) {
  uint32_t n = 0;
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
  const uint32_t cs[2] = {c.x, c.y};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t h = (xs[j >> 1] >> ((j & 1) * 16)) & 0x7FFFu;            // |x| bits
    const uint32_t code = (cs[j >> 2] >> ((j & 3) * 8)) & 0x7Fu;            // |code| bits
    n += (h != 0u && h <= 0x7F80u && code == 0u) ? 1u : 0u;                // nonzero, not NaN, code +-0
  }
  return n;
}

__global__ void __launch_bounds__(256) k_count_underflow(const uint4* __restrict__ x, const uint2* __restrict__ c,
                                                        int64_t n8, const uint16_t* __restrict__ xt,
                                                        const uint8_t* __restrict__ ct, int tail,
                                                        unsigned long long* __restrict__ count) {
  uint32_t local = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride)
    local += underflow8(__ldg(x + i), __ldg(c + i));
  if (blockIdx.x == 0 && (int)threadIdx.x < tail) {
    const uint32_t h = xt[threadIdx.x] & 0x7FFFu;
    local += (h != 0u && h <= 0x7F80u && (ct[threadIdx.x] & 0x7Fu) == 0u) ? 1u : 0u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xFFFFFFFFu, local, o);
  __shared__ uint32_t w[8];
  if ((threadIdx.x & 31) == 0) w[threadIdx.x >> 5] = local;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long s = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += w[i];
    if (s) atomicAdd(count, s);
  }
}

}  // namespace

cudaError_t launch_scale_histogram(const void* scales, int64_t n, int kind, uint32_t* hist, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + kHistThreads - 1) / kHistThreads, (int64_t)device_sm_count() * 4);
  if (kind == 0)
    k_scale_hist<0><<<(unsigned)blocks, kHistThreads, 0, st>>>(scales, n, hist);
  else
    k_scale_hist<1><<<(unsigned)blocks, kHistThreads, 0, st>>>(scales, n, hist);
  return cudaGetLastError();
}

cudaError_t launch_count_underflow(const uint16_t* x, const uint8_t* codes, int64_t n, unsigned long long* count,
                                   cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t n8 = n / 8;
  const int tail = (int)(n - n8 * 8);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, (int64_t)device_sm_count() * 8));
  k_count_underflow<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint4*>(x),
                                                      reinterpret_cast<const uint2*>(codes), n8, x + n8 * 8,
                                                      codes + n8 * 8, tail, count);
  return cudaGetLastError();
}

}  // namespace fp8q
