// Fused amax -> scale -> cast kernels for every scale granularity (sm_100a).
//
// Method: wangyu.me "大语言模型量化技术（五）：FP8", sections "什么是 FP8 量化" (s = amax/448,
// x/s, round to the nearest E4M3 value, saturate), "权重量化：128x128 分块 FP8" (one scale per
// 128x128 block, stored fp32 as [ceil(N/128)][ceil(K/128)]) and "激活动态量化" (one scale per
// token and 128-column group, computed at run time).  KV-cache granularities: pwwt.cn
// "从权重到激活：FP8 量化到底动了哪些东西", sections 1 and 3 (separate K/V scales, per head,
// per head x 128 tokens); api.makesence.top "LLM推理量化:FP8 versus INT8", section 二 (E5M2
// KV cache).
//
// All kernels are HBM-bound streams: 16-byte loads that bypass L1, group reductions in
// registers and warp shuffles, and the cast done on the registers already loaded, so a
// one-pass granularity reads each element once.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "fp8q_device.cuh"
#include "internal.h"

namespace fp8q {

int device_sm_count() {
  static int cache[128] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  f.s = s;
  f.m = (uint32_t)(((1ull << 32) * ((1ull << s) - d)) / d + 1);
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (uint32_t)(((uint64_t)__umulhi(n, f.m) + n) >> f.s);
}

// ============================================================================ 1 x 128 groups
//
// A warp quantizes four groups at a time: rows 4q .. 4q+3 of one 128-column group.  Eight
// lanes own one group, each lane 16 elements in two 16-byte pieces 64 columns apart, so each
// load instruction reads four fully used 128-byte lines.  The group amax is reduced across
// the eight lanes with three xor-shuffles.  The scales of consecutive rows of one group are
// contiguous in memory, so the four scales of a warp form one 16-byte run.

template <int FMT, int UNROLL>
__global__ void __launch_bounds__(256) k_quant_1x128(const uint16_t* __restrict__ x, uint8_t* __restrict__ codes,
                                                     float* __restrict__ scales, int64_t rows, int64_t cols,
                                                     uint32_t nrq, uint32_t units) {
  const uint32_t lane = threadIdx.x & 31u, sub = lane >> 3, l8 = lane & 7u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t u0 = warp; u0 < units; u0 += nwarps * UNROLL) {
    uint4 a[UNROLL], b[UNROLL];
    int64_t row[UNROLL], col[UNROLL];
    bool rv[UNROLL], v0[UNROLL], v1[UNROLL];
#pragma unroll
    for (int j = 0; j < UNROLL; ++j) {
      const uint32_t u = u0 + j * nwarps;
      const bool live = u < units;                     // warp-uniform
      const uint32_t g = live ? u / nrq : 0u;
      const uint32_t rq = live ? u - g * nrq : 0u;
      row[j] = (int64_t)rq * 4 + sub;
      col[j] = (int64_t)g * 128 + l8 * 8;
      rv[j] = live && row[j] < rows;
      v0[j] = rv[j] && col[j] < cols;
      v1[j] = rv[j] && col[j] + 64 < cols;
      const uint16_t* p = x + row[j] * cols + col[j];
      a[j] = v0[j] ? ld_stream_v4(p) : make_uint4(0u, 0u, 0u, 0u);
      b[j] = v1[j] ? ld_stream_v4(p + 64) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < UNROLL; ++j) {
      uint32_t m = absmax_v4(absmax_v4(0u, a[j]), b[j]);
      m = umax16x2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = umax16x2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      m = umax16x2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
      const GroupScale gs = make_group_scale<FMT>(packed_amax_to_f32(m));
      uint8_t* cp = codes + row[j] * cols + col[j];
      if (v0[j]) st_stream_v2(cp, quant8<FMT>(a[j], gs));
      if (v1[j]) st_stream_v2(cp + 64, quant8<FMT>(b[j], gs));
      if (l8 == 0 && rv[j]) scales[(col[j] >> 7) * rows + row[j]] = gs.s;
    }
  }
}

template <int FMT>
static cudaError_t launch_1x128_fmt(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes, float* scales,
                                    cudaStream_t st) {
  const int64_t ngc = (cols + 127) / 128, nrq = (rows + 3) / 4;
  const int64_t units = ngc * nrq;
  if (units == 0) return cudaSuccess;
  constexpr int kUnroll = 2;
  static int occ = 0;
  if (occ == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_quant_1x128<FMT, kUnroll>, 256, 0) != cudaSuccess ||
        occ <= 0)
      occ = 4;
  }
  const int64_t need = (units + 8 * kUnroll - 1) / (8 * kUnroll);   // 8 warps per block
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)device_sm_count() * occ));
  k_quant_1x128<FMT, kUnroll><<<grid, 256, 0, st>>>(x, codes, scales, rows, cols, (uint32_t)nrq, (uint32_t)units);
  return cudaGetLastError();
}

cudaError_t launch_quant_1x128(const uint16_t* x, int64_t rows, int64_t cols, int fmt, uint8_t* codes,
                               float* scales, cudaStream_t st) {
  return fmt == kE4M3 ? launch_1x128_fmt<kE4M3>(x, rows, cols, codes, scales, st)
                      : launch_1x128_fmt<kE5M2>(x, rows, cols, codes, scales, st);
}

// ============================================================================ 128-row tiles
//
// One CTA of 256 threads quantizes one tile of 128 rows x gw columns: 128 x 128 weight
// blocks (gw = 128, row stride = cols) and 128-token x head_dim KV blocks (gw = head_dim,
// row stride = heads * head_dim).  The whole tile (32 KB for 128 x 128) sits in registers,
// eight 16-byte pieces per thread, so the amax and the cast see each element exactly once.
// A warp loads two 256-byte row segments per instruction.  The CTA loops over tiles; several
// CTAs per SM keep loads of one tile in flight while another reduces and stores.

template <int FMT, int CPR_T, int MAXC>
__global__ void __launch_bounds__(256) k_quant_tiles(const uint16_t* __restrict__ x0, const uint16_t* __restrict__ x1,
                                                     uint8_t* __restrict__ c0, uint8_t* __restrict__ c1,
                                                     float* __restrict__ s0, float* __restrict__ s1, int64_t rows,
                                                     int64_t cols, int64_t ld, int gw, int nbr, int nbc,
                                                     int ntiles) {
  __shared__ uint32_t red[8];
  const int cpr = CPR_T > 0 ? CPR_T : gw / 8;   // 16-byte pieces per tile row
  const int nchunks = 128 * cpr;
  const int per_tensor = nbr * nbc;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
    const int tens = t / per_tensor;
    const int rem = t - tens * per_tensor;
    const int bi = rem / nbc, bj = rem - bi * nbc;
    const uint16_t* x = tens ? x1 : x0;
    uint8_t* c = tens ? c1 : c0;
    uint4 v[MAXC];
    int64_t off[MAXC];
    bool ok[MAXC];
    uint32_t m = 0;
#pragma unroll
    for (int k = 0; k < MAXC; ++k) {
      const int i = threadIdx.x + 256 * k;
      const int r = i / cpr, cc = i - r * cpr;
      const int64_t row = (int64_t)bi * 128 + r;
      const int64_t col = (int64_t)bj * gw + cc * 8;
      ok[k] = i < nchunks && row < rows && col < cols && cc * 8 < gw;
      off[k] = row * ld + col;
      v[k] = ok[k] ? ld_stream_v4(x + off[k]) : make_uint4(0u, 0u, 0u, 0u);
      m = absmax_v4(m, v[k]);
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) m = umax16x2(m, __shfl_xor_sync(0xFFFFFFFFu, m, d));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    uint32_t mm = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) mm = umax16x2(mm, red[w]);
    const GroupScale gs = make_group_scale<FMT>(packed_amax_to_f32(mm));
    if (threadIdx.x == 0) (tens ? s1 : s0)[bi * nbc + bj] = gs.s;
#pragma unroll
    for (int k = 0; k < MAXC; ++k)
      if (ok[k]) st_stream_v2(c + off[k], quant8<FMT>(v[k], gs));
    __syncthreads();   // red[] is rewritten by the next tile
  }
}

template <int FMT, int CPR_T, int MAXC>
static cudaError_t launch_tiles_impl(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                                     float* s1, int ntens, int64_t rows, int64_t cols, int64_t ld, int gw,
                                     cudaStream_t st) {
  const int nbr = (int)((rows + 127) / 128);
  const int nbc = (int)((cols + gw - 1) / gw);
  const int64_t ntiles = (int64_t)ntens * nbr * nbc;
  if (ntiles == 0) return cudaSuccess;
  static int occ = 0;
  if (occ == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_quant_tiles<FMT, CPR_T, MAXC>, 256, 0) !=
            cudaSuccess ||
        occ <= 0)
      occ = 2;
  }
  const int grid = (int)std::min<int64_t>(ntiles, (int64_t)device_sm_count() * occ);
  k_quant_tiles<FMT, CPR_T, MAXC><<<grid, 256, 0, st>>>(x0, x1, c0, c1, s0, s1, rows, cols, ld, gw, nbr, nbc,
                                                         (int)ntiles);
  return cudaGetLastError();
}

template <int FMT>
static cudaError_t launch_tiles_fmt(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                                    float* s1, int ntens, int64_t rows, int64_t cols, int64_t ld, int gw,
                                    cudaStream_t st) {
  if (gw == 128) return launch_tiles_impl<FMT, 16, 8>(x0, x1, c0, c1, s0, s1, ntens, rows, cols, ld, gw, st);
  if (gw <= 128) return launch_tiles_impl<FMT, 0, 8>(x0, x1, c0, c1, s0, s1, ntens, rows, cols, ld, gw, st);
  return launch_tiles_impl<FMT, 0, 16>(x0, x1, c0, c1, s0, s1, ntens, rows, cols, ld, gw, st);
}

cudaError_t launch_quant_tiles(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                               float* s1, int ntens, int64_t rows, int64_t cols, int64_t ld, int gw, int fmt,
                               cudaStream_t st) {
  return fmt == kE4M3 ? launch_tiles_fmt<kE4M3>(x0, x1, c0, c1, s0, s1, ntens, rows, cols, ld, gw, st)
                      : launch_tiles_fmt<kE5M2>(x0, x1, c0, c1, s0, s1, ntens, rows, cols, ld, gw, st);
}

// ============================================================================ two passes
//
// Per-tensor and per-head scales need the amax of a group that spans the whole tensor (or
// all tokens of a head) before its first element can be cast, so they take two kernels.
// Pass 1: CTA b reduces a contiguous range of 16-byte pieces into per-group maxima (shared
// memory atomics on the 16-bit magnitude patterns) and writes them to partials[b][group].
// Pass 2: each CTA folds the partials into the group scales, CTA 0 stores them, and the CTA
// casts the same range it covered in pass 1, walking it backwards so that the tail it read
// last, which is the part most likely still in L2, is consumed first.

constexpr int kTwoPassThreads = 256;
constexpr int kTwoPassUnroll = 8;

size_t two_pass_workspace_bytes(int ntens, int64_t heads) {
  return (size_t)kMaxPartials * (size_t)ntens * (size_t)heads * sizeof(float);
}

struct TwoPassShape {
  const uint16_t* x0;
  const uint16_t* x1;
  uint8_t* c0;
  uint8_t* c1;
  float* s0;
  float* s1;
  uint32_t chunks;      // 16-byte pieces per tensor
  FastDiv cpr;          // pieces per row
  FastDiv cpg;          // pieces per head
  uint32_t heads;
  uint32_t ngroups;     // ntens * heads
  uint32_t per_cta;     // pieces per CTA range (multiple of the thread count)
  uint32_t total;       // ntens * chunks
};

__device__ __forceinline__ uint32_t group_of(const TwoPassShape& sh, uint32_t i, uint32_t* tens, uint32_t* w) {
  const uint32_t t = i >= sh.chunks ? 1u : 0u;
  const uint32_t wi = i - t * sh.chunks;
  *tens = t;
  *w = wi;
  if (sh.heads == 1) return t;
  const uint32_t col_piece = wi - fdiv(wi, sh.cpr) * sh.cpr.d;
  return t * sh.heads + fdiv(col_piece, sh.cpg);
}

__global__ void __launch_bounds__(kTwoPassThreads) k_two_pass_amax(TwoPassShape sh, float* __restrict__ partials) {
  __shared__ uint32_t smax[256];
  for (uint32_t g = threadIdx.x; g < sh.ngroups; g += kTwoPassThreads) smax[g] = 0u;
  __syncthreads();
  const uint32_t beg = blockIdx.x * sh.per_cta;
  const uint32_t end = min(sh.total, beg + sh.per_cta);
  uint32_t cur = 0xFFFFFFFFu, m = 0u;
  for (uint32_t i0 = beg + threadIdx.x; i0 < end; i0 += kTwoPassThreads * kTwoPassUnroll) {
    uint4 v[kTwoPassUnroll];
#pragma unroll
    for (int k = 0; k < kTwoPassUnroll; ++k) {
      const uint32_t i = i0 + k * kTwoPassThreads;
      uint32_t t = 0, w = 0;
      if (i < end) group_of(sh, i, &t, &w);
      v[k] = i < end ? ld_stream_v4((t ? sh.x1 : sh.x0) + (size_t)w * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kTwoPassUnroll; ++k) {
      const uint32_t i = i0 + k * kTwoPassThreads;
      if (i >= end) break;
      uint32_t t, w;
      const uint32_t g = group_of(sh, i, &t, &w);
      if (g != cur) {
        if (cur != 0xFFFFFFFFu) atomicMax(&smax[cur], max(m & 0xFFFFu, m >> 16));
        cur = g;
        m = 0u;
      }
      m = absmax_v4(m, v[k]);
    }
  }
  if (cur != 0xFFFFFFFFu) atomicMax(&smax[cur], max(m & 0xFFFFu, m >> 16));
  __syncthreads();
  for (uint32_t g = threadIdx.x; g < sh.ngroups; g += kTwoPassThreads)
    partials[(size_t)blockIdx.x * sh.ngroups + g] = __uint_as_float(smax[g] << 16);
}

template <int FMT>
__global__ void __launch_bounds__(kTwoPassThreads) k_two_pass_cast(TwoPassShape sh, const float* __restrict__ partials,
                                                                 int nparts) {
  __shared__ uint32_t sred[256];
  __shared__ GroupScale sg[256];
  for (uint32_t g = threadIdx.x; g < sh.ngroups; g += kTwoPassThreads) sred[g] = 0u;
  __syncthreads();
  // fold partials: amax values are non-negative floats (or NaN), whose bit patterns order
  // like their values with NaN on top, so an integer max is exact
  const uint32_t nitems = (uint32_t)nparts * sh.ngroups;
  for (uint32_t it = threadIdx.x; it < nitems; it += kTwoPassThreads) {
    const uint32_t g = it % sh.ngroups;
    atomicMax(&sred[g], __float_as_uint(partials[it]));
  }
  __syncthreads();
  for (uint32_t g = threadIdx.x; g < sh.ngroups; g += kTwoPassThreads) {
    sg[g] = make_group_scale<FMT>(__uint_as_float(sred[g]));
    if (blockIdx.x == 0) {
      const uint32_t t = g / sh.heads;
      (t ? sh.s1 : sh.s0)[g - t * sh.heads] = sg[g].s;
    }
  }
  __syncthreads();
  const uint32_t beg = blockIdx.x * sh.per_cta;
  const uint32_t end = min(sh.total, beg + sh.per_cta);
  if (beg >= end) return;
  // walk the range backwards in steps of the CTA width
  const uint32_t span = end - beg;
  const uint32_t nsteps = (span + kTwoPassThreads - 1) / kTwoPassThreads;
  for (int64_t step = (int64_t)nsteps - 1; step >= 0; step -= 4) {
    uint4 v[4];
    uint32_t ii[4], tt[4], ww[4], gg[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t sidx = step - k;
      const uint32_t i = sidx >= 0 ? beg + (uint32_t)sidx * kTwoPassThreads + threadIdx.x : end;
      ii[k] = i;
      tt[k] = 0;
      ww[k] = 0;
      gg[k] = i < end ? group_of(sh, i, &tt[k], &ww[k]) : 0u;
      v[k] = i < end ? ld_stream_v4((tt[k] ? sh.x1 : sh.x0) + (size_t)ww[k] * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (ii[k] < end) st_stream_v2((tt[k] ? sh.c1 : sh.c0) + (size_t)ww[k] * 8, quant8<FMT>(v[k], sg[gg[k]]));
  }
}

cudaError_t launch_quant_two_pass(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                                  float* s1, int ntens, int64_t rows, int64_t heads, int64_t head_dim, int fmt,
                                  float* ws, cudaStream_t st) {
  TwoPassShape sh;
  sh.x0 = x0;
  sh.x1 = ntens > 1 ? x1 : x0;
  sh.c0 = c0;
  sh.c1 = ntens > 1 ? c1 : c0;
  sh.s0 = s0;
  sh.s1 = ntens > 1 ? s1 : s0;
  const int64_t cpr = heads * head_dim / 8;
  sh.chunks = (uint32_t)(rows * cpr);
  sh.cpr = make_fastdiv((uint32_t)std::max<int64_t>(cpr, 1));
  sh.cpg = make_fastdiv((uint32_t)std::max<int64_t>(head_dim / 8, 1));
  sh.heads = (uint32_t)heads;
  sh.ngroups = (uint32_t)(ntens * heads);
  sh.total = (uint32_t)ntens * sh.chunks;
  const int sms = device_sm_count();
  // pass-1 CTAs: two per SM for large tensors, fewer for small ones (at least 8 KB each)
  const int64_t want = std::min<int64_t>((int64_t)2 * sms, kMaxPartials);
  const int64_t min_per = 512;   // pieces (8 KB of bf16)
  int64_t nparts = std::max<int64_t>(1, std::min<int64_t>(want, ((int64_t)sh.total + min_per - 1) / min_per));
  int64_t per = ((int64_t)sh.total + nparts - 1) / nparts;
  per = std::max<int64_t>(kTwoPassThreads, (per + kTwoPassThreads - 1) / kTwoPassThreads * kTwoPassThreads);
  nparts = std::max<int64_t>(1, ((int64_t)sh.total + per - 1) / per);
  sh.per_cta = (uint32_t)per;
  k_two_pass_amax<<<(int)nparts, kTwoPassThreads, 0, st>>>(sh, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (fmt == kE4M3)
    k_two_pass_cast<kE4M3><<<(int)nparts, kTwoPassThreads, 0, st>>>(sh, ws, (int)nparts);
  else
    k_two_pass_cast<kE5M2><<<(int)nparts, kTwoPassThreads, 0, st>>>(sh, ws, (int)nparts);
  return cudaGetLastError();
}

}  // namespace fp8q
