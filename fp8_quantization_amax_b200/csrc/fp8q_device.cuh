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

// ---------------------------------------------------------------- global memory

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
// max.NaN.xorsign.abs.bf16x2 keeps the larger magnitude of each half (the result's sign is the
// xor of the inputs' signs, which never matters: every use takes magnitudes again) and
// propagates NaN.  bf16 comparison is exact, so the group amax is exact and order-free.

__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t absmax_v4(uint32_t m, uint4 v) {
  return absmax2(absmax2(m, v.x), absmax2(absmax2(v.y, v.z), v.w));
}

// packed pair -> fp32 amax of the two halves (any NaN gives NaN)
__device__ __forceinline__ float packed_amax_to_f32(uint32_t m) {
  const uint32_t r = absmax2(m, m >> 16) & 0x7FFFu;
  return __uint_as_float(r << 16);
}

// ---------------------------------------------------------------- scale and quotient
//
// Every element's quotient must be the IEEE round-to-nearest fp32 value of x / s.  A division
// per element is far too slow for an HBM-bound kernel, so groups whose amax is an ordinary
// normal number use Markstein's correction (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with
// r = RN(1/d) and q0 = RN(x * r), the residual x - q0 * d is exact in one FMA and
// RN(q0 + (x - q0 * d) * r) = RN(x / d) when nothing overflows or underflows.  The residual is
// formed negated, e' = q0 * d - x, and applied as q = q0 - e' * r: the same value for x != 0,
// and for x = -0 it yields -0 (q0 = -0, e' = +0, -0 + -0 = -0), so zero signs need no fix-up.
// The same step with the constant RN(1/FMAX) gives the scale s = RN(amax / FMAX).  Groups with
// a tiny, infinite or NaN amax take IEEE divisions instead.  An all-zero group has s = 0 and
// divides by 1 (every x is +-0).  The fast path is checked against the oracle for every
// (bf16 x, bf16 amax) pair.

struct GroupScale {
  float s;     // stored scale
  float d;     // divisor used for the quotients
  float r;     // RN(1 / d) (fast path)
  bool fast;
};

__device__ __forceinline__ float markstein_div(float x, float d, float r) {
  const float q0 = __fmul_rn(x, r);
  const float en = __fmaf_rn(q0, d, -x);     // -(x - q0 * d), exact
  return __fmaf_rn(-en, r, q0);
}

template <int FMT>
__device__ __forceinline__ GroupScale make_group_scale(float amax) {
  constexpr float kMax = Fmt<FMT>::kMax;
  constexpr float kInvMax = 1.0f / Fmt<FMT>::kMax;            // RN(1 / FMAX)
  GroupScale g;
  if (amax >= 0x1.0p-60f && amax <= 3.4028234663852886e38f) {
    g.s = markstein_div(amax, kMax, kInvMax);
    g.d = g.s;
    g.r = __frcp_rn(g.s);
    g.fast = true;
  } else if (amax == 0.0f) {
    g.s = 0.0f;
    g.d = 1.0f;
    g.r = 1.0f;
    g.fast = true;
  } else {
    g.s = __fdiv_rn(amax, kMax);
    g.d = g.s;
    g.r = 0.0f;
    g.fast = false;
  }
  return g;
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

// four bf16 (two words) -> four codes, fast path
template <int FMT>
__device__ __forceinline__ uint32_t quant4_fast(uint32_t w0, uint32_t w1, float d, float r) {
  // The same three rounded steps as markstein_div, on fp32 pairs (one FMUL2 / FFMA2 per pair)
  // and with every value negated, so no operand needs a sign flip: p = RN(x * -r) = -q0,
  // f = RN(p * d + x) = x - q0 * d (exact), n = RN(f * -r + p) = -RN(q0 + (x - q0 * d) * r)
  // = -q, because round-to-nearest is odd-symmetric (a zero residual is +0 in both forms, and
  // x = +-0 gives n = -+0).  The codes of -q are those of q with the sign bit flipped, and the
  // saturating conversion is sign-symmetric, so one XOR restores them.
  const float2 d2 = make_float2(d, d), nr2 = make_float2(-r, -r);
  const float2 x0 = make_float2(bf16_lo(w0), bf16_hi(w0)), x1 = make_float2(bf16_lo(w1), bf16_hi(w1));
  const float2 p0 = __fmul2_rn(x0, nr2), p1 = __fmul2_rn(x1, nr2);
  const float2 f0 = __ffma2_rn(p0, d2, x0), f1 = __ffma2_rn(p1, d2, x1);
  const float2 n0 = __ffma2_rn(f0, nr2, p0), n1 = __ffma2_rn(f1, nr2, p1);
  return __byte_perm(cvt2<FMT>(n0.x, n0.y), cvt2<FMT>(n1.x, n1.y), 0x5410) ^ 0x80808080u;
}

// eight bf16 (16 bytes) -> eight codes (8 bytes), fast path
template <int FMT>
__device__ __forceinline__ uint2 quant8_fast(uint4 v, float d, float r) {
  return make_uint2(quant4_fast<FMT>(v.x, v.y, d, r), quant4_fast<FMT>(v.z, v.w, d, r));
}

// sixteen bf16 (two 16-byte pieces) -> sixteen codes (16 bytes), fast path
template <int FMT>
__device__ __forceinline__ uint4 quant16_fast(uint4 a, uint4 b, float d, float r) {
  return make_uint4(quant4_fast<FMT>(a.x, a.y, d, r), quant4_fast<FMT>(a.z, a.w, d, r),
                    quant4_fast<FMT>(b.x, b.y, d, r), quant4_fast<FMT>(b.z, b.w, d, r));
}

// eight bf16 -> eight codes with IEEE divisions (groups with tiny, infinite or NaN amax).
// d == 0 is a zero scale met by delayed scaling (an all-zero amax history while the tensor is
// not zero): every code is the zero with the element's sign, as for an all-zero group.
template <int FMT>
__device__ __noinline__ uint2 quant8_slow(uint4 v, float d) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (d == 0.0f) {
    const uint32_t lo = ((w[0] >> 8) & 0x80u) | ((w[0] >> 16) & 0x8000u) | ((w[1] << 8) & 0x800000u) | (w[1] & 0x80000000u);
    const uint32_t hi = ((w[2] >> 8) & 0x80u) | ((w[2] >> 16) & 0x8000u) | ((w[3] << 8) & 0x800000u) | (w[3] & 0x80000000u);
    return make_uint2(lo, hi);
  }
  uint32_t c[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t a = cvt2<FMT>(__fdiv_rn(bf16_lo(w[2 * i]), d), __fdiv_rn(bf16_hi(w[2 * i]), d));
    const uint32_t b = cvt2<FMT>(__fdiv_rn(bf16_lo(w[2 * i + 1]), d), __fdiv_rn(bf16_hi(w[2 * i + 1]), d));
    c[i] = __byte_perm(a, b, 0x5410);
  }
  return make_uint2(c[0], c[1]);
}

// eight bf16 -> eight codes for a group of the slow path without a division (no call, for kernels
// whose register budget a call would break).  A scale from a tiny amax (d < 2^-60) is scaled
// with the elements by 2^100: both products are exact and normal, so x / d = (x 2^100) /
// (d 2^100) and Markstein's step on the scaled pair is RN(x / d).  d = +inf gives x * 0 (the
// signed zero for finite x, NaN for +-inf or NaN x) and d = NaN gives NaN, as x / d does.  The
// scale of delayed scaling (d = 0) is not handled here.
template <int FMT>
__device__ __forceinline__ uint2 quant8_nodiv(uint4 v, float d) {
  const bool tiny = d < 0x1.0p-60f;
  const bool inf = d == __int_as_float(0x7F800000);
  const float xs = tiny ? 0x1.0p100f : 1.0f;
  const float ds = tiny ? d * 0x1.0p100f : d;
  const float rs = inf ? 0.0f : __frcp_rn(ds);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x0 = bf16_lo(w[i]) * xs, x1 = bf16_hi(w[i]) * xs;
    const float q0 = inf ? x0 * 0.0f : markstein_div(x0, ds, rs);
    const float q1 = inf ? x1 * 0.0f : markstein_div(x1, ds, rs);
    c[i] = cvt2<FMT>(q0, q1);
  }
  return make_uint2(__byte_perm(c[0], c[1], 0x5410), __byte_perm(c[2], c[3], 0x5410));
}

template <int FMT>
__device__ __forceinline__ uint2 quant8(uint4 v, const GroupScale& g) {
  return g.fast ? quant8_fast<FMT>(v, g.d, g.r) : quant8_slow<FMT>(v, g.d);
}

// ---------------------------------------------------------------- delayed scaling, counts

// Scale of a delayed-scaling group from the largest amax in its history (>= 0 or NaN).  A zero
// history gives s = 0 with d = 0, which quant8_slow turns into sign-only codes.
template <int FMT>
__device__ __forceinline__ GroupScale make_delayed_scale(float hmax) {
  if (hmax == 0.0f) {
    GroupScale g;
    g.s = 0.0f;
    g.d = 0.0f;
    g.r = 0.0f;
    g.fast = false;
    return g;
  }
  return make_group_scale<FMT>(hmax);
}

// Counts of one chunk of eight bf16 and their codes: `sat` += elements whose quotient rounds
// above FMAX on the grid continued past it (ties to even: E4M3 |q| > 464, the tie going to 448;
// E5M2 |q| >= 61440, the tie going to 65536); `und` += elements with x != 0 (NaN excluded)
// whose code is +-0.
template <int FMT>
__device__ __forceinline__ void count8(uint4 v, uint2 codes, const GroupScale& g, uint32_t& sat, uint32_t& und) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float x = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
    const uint32_t code = ((i < 4 ? codes.x : codes.y) >> (8 * (i & 3))) & 0xFFu;
    if (g.d != 0.0f) {
      const float a = fabsf(g.fast ? markstein_div(x, g.d, g.r) : __fdiv_rn(x, g.d));
      sat += (FMT == kE4M3) ? (a > 464.0f) : (a >= 61440.0f);
    }
    und += (x == x && x != 0.0f && (code & 0x7Fu) == 0u);
  }
}

}  // namespace fp8q
