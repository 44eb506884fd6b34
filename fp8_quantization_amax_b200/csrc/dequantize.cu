// Dequantization and the element-wise FP8 codec (sm_100a).
//
// Dequantize: charles2530.github.io "量化：FP8 与混合精度推理", section "E4M3 和 E5M2 是范围与
// 格点的取舍" (x_hat = s * x_fp8), and wangyu.me "大语言模型量化技术（五）：FP8", section
// "什么是 FP8 量化" (restore x ~ x_hat * s).  Codes are widened exactly through the hardware
// FP8 -> f16x2 convert (every E4M3 / E5M2 value is an f16 value), multiplied by the group's
// fp32 scale with one rounding, and rounded to bf16 (nearest even).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "fp8q_device.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace fp8q {

__device__ __forceinline__ uint32_t fdiv_u32(uint32_t n, const FastDiv& f) {
  return (uint32_t)(((uint64_t)__umulhi(n, f.m) + n) >> f.s);
}

template <int FMT>
__device__ __forceinline__ uint32_t dequant2(uint32_t codes16, float s) {
  const uint32_t h2 = fp8x2_to_f16x2<FMT>((uint16_t)codes16);
  return f32x2_to_bf16x2(__fmul_rn(f16_lo_to_f32(h2), s), __fmul_rn(f16_hi_to_f32(h2), s));
}

// eight codes -> eight bf16
template <int FMT>
__device__ __forceinline__ uint4 dequant8(uint2 c, float s) {
  return make_uint4(dequant2<FMT>(c.x & 0xFFFFu, s), dequant2<FMT>(c.x >> 16, s), dequant2<FMT>(c.y & 0xFFFFu, s),
                    dequant2<FMT>(c.y >> 16, s));
}

// Each thread handles 8-element pieces (8 code bytes in, 16 bf16 bytes out) of the flattened
// tensor; the row of a piece comes from a multiply-shift division by the pieces per row.
template <int FMT, int GRAN, int UNROLL>
__global__ void __launch_bounds__(256) k_dequant(const uint8_t* __restrict__ codes, const float* __restrict__ scales,
                                                 uint16_t* __restrict__ y, uint32_t npieces, FastDiv ppr,
                                                 uint32_t rows, uint32_t nbc) {
  allow_dependent_launch();
  grid_dependency_wait();
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i0 = blockIdx.x * blockDim.x + threadIdx.x; i0 < npieces; i0 += stride * UNROLL) {
    uint2 c[UNROLL];
    float s[UNROLL];
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) {
      const uint32_t i = i0 + k * stride;
      if (i < npieces) {
        c[k] = ld_stream_v2(codes + (size_t)i * 8);
        const uint32_t r = fdiv_u32(i, ppr);
        const uint32_t col = (i - r * ppr.d) * 8;
        if (GRAN == 0) {
          s[k] = __ldg(scales);
        } else if (GRAN == 1) {
          s[k] = __ldg(scales + (size_t)(col >> 7) * rows + r);
        } else if (GRAN == 2) {
          s[k] = __ldg(scales + (size_t)(r >> 7) * nbc + (col >> 7));
        } else {
          // MX: byte exponents [rows][cols / 32] (nbc = cols / 32), scale 2^(b - 127); 255 is NaN
          const uint32_t b = __ldg(reinterpret_cast<const uint8_t*>(scales) + (size_t)r * nbc + (col >> 5));
          s[k] = __uint_as_float(b == 255u ? 0x7FC00000u : (b == 0u ? 0x00400000u : b << 23));
        }
      }
    }
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) {
      const uint32_t i = i0 + k * stride;
      if (i < npieces) st_stream_v4(y + (size_t)i * 8, dequant8<FMT>(c[k], s[k]));
    }
  }
}

template <int FMT, int GRAN>
static cudaError_t launch_dequant_impl(const uint8_t* codes, const float* scales, int64_t rows, int64_t cols,
                                       uint16_t* y, cudaStream_t st) {
  const int64_t npieces = rows * cols / 8;
  if (npieces == 0) return cudaSuccess;
  constexpr int kUnroll = 4;
  static int occ = 0;
  if (occ == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_dequant<FMT, GRAN, kUnroll>, 256, 0) != cudaSuccess ||
        occ <= 0)
      occ = 4;
  }
  const int64_t need = (npieces + 256 * kUnroll - 1) / (256 * kUnroll);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)device_sm_count() * occ));
  return launch_pdl(k_dequant<FMT, GRAN, kUnroll>, dim3(grid), dim3(256), 0, st, codes, scales, y,
                    (uint32_t)npieces, make_fastdiv((uint32_t)(cols / 8)), (uint32_t)rows,
                    (uint32_t)(GRAN == 3 ? cols / 32 : (cols + 127) / 128));
}

template <int FMT>
static cudaError_t launch_dequant_fmt(const uint8_t* codes, const float* scales, int64_t rows, int64_t cols,
                                      int gran, uint16_t* y, cudaStream_t st) {
  if (gran == 0) return launch_dequant_impl<FMT, 0>(codes, scales, rows, cols, y, st);
  if (gran == 1) return launch_dequant_impl<FMT, 1>(codes, scales, rows, cols, y, st);
  if (gran == 2) return launch_dequant_impl<FMT, 2>(codes, scales, rows, cols, y, st);
  return launch_dequant_impl<FMT, 3>(codes, scales, rows, cols, y, st);   // MX: byte exponents
}

cudaError_t launch_dequant(const uint8_t* codes, const float* scales, int64_t rows, int64_t cols, int fmt,
                           int gran, uint16_t* y, cudaStream_t st) {
  return fmt == kE4M3 ? launch_dequant_fmt<kE4M3>(codes, scales, rows, cols, gran, y, st)
                      : launch_dequant_fmt<kE5M2>(codes, scales, rows, cols, gran, y, st);
}

// ============================================================================ codec

template <int FMT>
__global__ void __launch_bounds__(256) k_encode(const float* __restrict__ q, int64_t n, uint8_t* __restrict__ codes) {
  allow_dependent_launch();
  grid_dependency_wait();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t n4 = n / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 v = __ldcs(reinterpret_cast<const float4*>(q) + i);
    const uint32_t w = cvt2<FMT>(v.x, v.y) | (cvt2<FMT>(v.z, v.w) << 16);
    __stcs(reinterpret_cast<unsigned int*>(codes) + i, w);
  }
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n - n4 * 4) codes[n4 * 4 + t] = (uint8_t)(cvt2<FMT>(q[n4 * 4 + t], 0.0f) & 0xFFu);
}

template <int FMT>
__global__ void __launch_bounds__(256) k_decode(const uint8_t* __restrict__ codes, int64_t n, float* __restrict__ out) {
  allow_dependent_launch();
  grid_dependency_wait();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t n4 = n / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const uint32_t w = __ldcs(reinterpret_cast<const unsigned int*>(codes) + i);
    const uint32_t a = fp8x2_to_f16x2<FMT>((uint16_t)(w & 0xFFFFu));
    const uint32_t b = fp8x2_to_f16x2<FMT>((uint16_t)(w >> 16));
    __stcs(reinterpret_cast<float4*>(out) + i,
           make_float4(f16_lo_to_f32(a), f16_hi_to_f32(a), f16_lo_to_f32(b), f16_hi_to_f32(b)));
  }
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n - n4 * 4) out[n4 * 4 + t] = f16_lo_to_f32(fp8x2_to_f16x2<FMT>((uint16_t)codes[n4 * 4 + t]));
}

static int codec_grid(int64_t n) {
  const int64_t need = (n / 4 + 255) / 256 + 1;
  return (int)std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)device_sm_count() * 8));
}

cudaError_t launch_encode(const float* q, int64_t n, int fmt, uint8_t* codes, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  return fmt == kE4M3 ? launch_pdl(k_encode<kE4M3>, dim3(codec_grid(n)), dim3(256), 0, st, q, n, codes)
                      : launch_pdl(k_encode<kE5M2>, dim3(codec_grid(n)), dim3(256), 0, st, q, n, codes);
}

cudaError_t launch_decode(const uint8_t* codes, int64_t n, int fmt, float* out, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  return fmt == kE4M3 ? launch_pdl(k_decode<kE4M3>, dim3(codec_grid(n)), dim3(256), 0, st, codes, n, out)
                      : launch_pdl(k_decode<kE5M2>, dim3(codec_grid(n)), dim3(256), 0, st, codes, n, out);
}

}  // namespace fp8q
