// Device helpers shared by the quantize / dequantize kernels (sm_100a).
//
// Number formats follow the table on wangyu.me "大语言模型量化技术（五）：FP8", section
// "FP8 是什么": E4M3 (max 448) and E5M2 (max 57344), round to nearest with ties to even,
// saturating.  The conversions use the hardware FP8 convert instructions (cvt ... e4m3x2 /
// e5m2x2 with .satfinite), which round to nearest-even and clamp finite overflow and Inf to
// the largest finite value.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp8q {

constexpr int kE4M3 = 0;
constexpr int kE5M2 = 1;

template <int FMT>
struct Fmt;
template <>
struct Fmt<kE4M3> {
  static constexpr float kMax = 448.0f;
};
template <>
struct Fmt<kE5M2> {
  static constexpr float kMax = 57344.0f;
};

// ---------------------------------------------------------------- memory

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream_v2(void* p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------- amax on packed bf16
//
// |x| of a bf16 is its bit pattern with the sign cleared; for non-negative bf16 values the
// unsigned integer order of the 16-bit patterns is the numeric order, with Inf above every
// finite value and every NaN above Inf.  So a packed unsigned 16x2 max of the sign-cleared
// words is an exact amax in which any NaN dominates.

__device__ __forceinline__ uint32_t umax16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t absmax_v4(uint32_t m, uint4 v) {
  m = umax16x2(m, v.x & 0x7FFF7FFFu);
  m = umax16x2(m, v.y & 0x7FFF7FFFu);
  m = umax16x2(m, v.z & 0x7FFF7FFFu);
  m = umax16x2(m, v.w & 0x7FFF7FFFu);
  return m;
}

// packed pair max -> fp32 amax
__device__ __forceinline__ float packed_amax_to_f32(uint32_t m) {
  uint32_t lo = m & 0xFFFFu, hi = m >> 16;
  return __uint_as_float((lo > hi ? lo : hi) << 16);
}

// ---------------------------------------------------------------- scale and quotient
//
// The scale is s = amax / FMAX (one IEEE division) and every element's quotient must be the
// IEEE round-to-nearest fp32 value of x / s.  A per-element division is too slow for an HBM
// bound kernel, so groups whose scale is a comfortably normal number use the reciprocal
// r = RN(1/s) once per group and Markstein's correction per element:
//   q0 = RN(x * r);  e = x - q0 * s (exact, one FMA);  q = RN(q0 + e * r)
// (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990), which yields RN(x / s) when r is the correctly
// rounded reciprocal and nothing underflows.  The sign of a zero quotient is restored from x
// (the correction adds +0 to -0).  Groups with tiny, zero, infinite or NaN scales fall back
// to the IEEE division per element; an all-zero group keeps the sign of each zero.
// Exactness of the fast path is verified exhaustively over every (bf16 x, bf16 amax) pair
// by the GPU parity tests.

struct GroupScale {
  float s;     // stored scale
  float sd;    // divisor used for the quotient
  float r;     // RN(1 / sd) for the fast path
  bool fast;   // Markstein path valid for this group
};

template <int FMT>
__device__ __forceinline__ GroupScale make_group_scale(float amax) {
  GroupScale g;
  g.s = __fdiv_rn(amax, Fmt<FMT>::kMax);
  // fast path: s in [2^-80, FLT_MAX]; s == 0 (all-zero group) uses divisor 1: q = x exactly
  const bool normal_s = g.s >= 0x1.0p-80f && g.s <= 3.4028234663852886e38f;
  g.sd = (g.s == 0.0f) ? 1.0f : g.s;
  g.fast = normal_s || g.s == 0.0f;
  g.r = g.fast ? __frcp_rn(g.sd) : 0.0f;
  return g;
}

__device__ __forceinline__ float quotient(float x, const GroupScale& g) {
  if (g.fast) {
    float q0 = __fmul_rn(x, g.r);
    float e = __fmaf_rn(-q0, g.sd, x);
    float q = __fmaf_rn(e, g.r, q0);
    return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(x) & 0x80000000u));
  }
  return __fdiv_rn(x, g.sd);
}

// ---------------------------------------------------------------- FP8 conversions

// two fp32 -> two FP8 codes; `lo` lands in the low byte
template <int FMT>
__device__ __forceinline__ uint32_t cvt2(float lo, float hi) {
  uint16_t d;
  if constexpr (FMT == kE4M3) {
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  } else {
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  }
  return d;
}

// two FP8 codes (low byte first) -> packed f16x2 (exact)
template <int FMT>
__device__ __forceinline__ uint32_t fp8x2_to_f16x2(uint16_t c) {
  uint32_t d;
  if constexpr (FMT == kE4M3) {
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(c));
  } else {
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(d) : "h"(c));
  }
  return d;
}

__device__ __forceinline__ float f16_lo_to_f32(uint32_t h2) {
  float f;
  asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; cvt.f32.f16 %0, l; }" : "=f"(f) : "r"(h2));
  return f;
}

__device__ __forceinline__ float f16_hi_to_f32(uint32_t h2) {
  float f;
  asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; cvt.f32.f16 %0, h; }" : "=f"(f) : "r"(h2));
  return f;
}

// two fp32 -> packed bf16x2 (round to nearest even); `lo` in the low half
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// bf16 pair in a 32-bit word -> fp32 (exact)
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// quantize four bf16 (two words) into four codes packed in a 32-bit word
template <int FMT>
__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, const GroupScale& g) {
  uint32_t a = cvt2<FMT>(quotient(bf16_lo(w0), g), quotient(bf16_hi(w0), g));
  uint32_t b = cvt2<FMT>(quotient(bf16_lo(w1), g), quotient(bf16_hi(w1), g));
  return a | (b << 16);
}

// quantize eight bf16 (16 bytes) into eight codes (8 bytes)
template <int FMT>
__device__ __forceinline__ uint2 quant8(uint4 v, const GroupScale& g) {
  return make_uint2(quant4<FMT>(v.x, v.y, g), quant4<FMT>(v.z, v.w, g));
}

}  // namespace fp8q
