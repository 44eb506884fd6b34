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
// Structure (all kernels): a persistent CTA of nine warps.  Warp 8 is the producer: one lane
// streams 2-D TMA boxes of the bf16 input into a ring of shared-memory stages (mbarrier
// full/empty pipeline).  Warps 0-7 consume: each thread reads its 16-byte pieces of a stage,
// frees the stage, reduces the group amax (warp shuffles, plus a named barrier when a group
// spans the whole box), computes the scale and writes the FP8 codes straight to global memory.
// Loads stay in flight several stages ahead regardless of the consumers' progress.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "fp8q_device.cuh"
#include "internal.h"
#include "sm100.cuh"

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

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kConsumers + 32;          // + the producer warp
constexpr int kMaxStages = 8;
constexpr uint32_t kStageBudget = 96 * 1024;        // ring bytes per CTA (two CTAs per SM)

// Producer side of the ring: issue TMA box loads for this CTA's items in `item_at(k)` order,
// each into the next stage once the consumers have freed it; finally wait until every issued
// copy has landed (they have, unless the consumers gave up), so no copy outlives the CTA.
template <class ItemFn, class IssueFn>
__device__ __forceinline__ void run_producer(uint64_t* full, uint64_t* empty, int S, uint32_t nk, uint32_t bytes,
                                             uint32_t* err, ItemFn item_at, IssueFn issue) {
  int s = 0;
  uint32_t ph = 0, k = 0;
  for (; k < nk; ++k) {
    if (k >= (uint32_t)S && !mbar_wait(&empty[s], ph ^ 1u, err)) break;
    mbar_arrive_expect_tx(&full[s], bytes);
    issue(item_at(k), s, &full[s]);
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
  }
  const uint32_t last = k;
  for (uint32_t j = 0; j < (uint32_t)S && j < last; ++j) {
    const uint32_t kk = last - 1 - j;
    mbar_wait(&full[kk % S], (kk / S) & 1u, err);
  }
}

// number of items of this CTA under a grid-stride assignment
__device__ __forceinline__ uint32_t items_of_cta(uint32_t nitems) {
  return nitems > blockIdx.x ? (nitems - blockIdx.x + gridDim.x - 1) / gridDim.x : 0u;
}

static uint32_t ring_stages(uint32_t stage_bytes) {
  return std::max<uint32_t>(2, std::min<uint32_t>(kMaxStages, kStageBudget / stage_bytes));
}

static size_t ring_smem(uint32_t stages, uint32_t stage_bytes) {
  return 1024 + (size_t)stages * stage_bytes + 2 * kMaxStages * sizeof(uint64_t);   // + alignment slack
}

// dynamic shared memory starts after the static arrays; TMA boxes land on 1024-byte boundaries
__device__ __forceinline__ uint8_t* ring_base(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return raw + (((a + 1023u) & ~1023u) - a);
}

template <class K>
static int grid_for(K kernel, size_t smem, uint32_t nitems) {
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kThreads, smem) != cudaSuccess || occ <= 0)
    occ = 1;
  return (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)nitems, (int64_t)device_sm_count() * occ));
}

// ============================================================================ 1 x 128 groups
//
// Box = 64 rows x 128 columns (16 KB): 64 groups.  Four consecutive threads own one group
// (32 elements each, four 16-byte pieces), reduce it with two xor-shuffles, and store 32 codes.
// The 64 scales of a box are 64 consecutive rows of one group column: one 256-byte run.

constexpr uint32_t kGroupBoxRows = 128;      // box: 128 rows x 128 columns (32 KB)
constexpr int kGroupRowsPerThread = kGroupBoxRows / 64;   // rows each of a row's four threads takes
constexpr uint32_t kGroupStage = kGroupBoxRows * 128 * 2;

struct GroupParams {
  uint8_t* codes;
  float* scales;
  uint8_t* mx_scales;  // MX: power-of-two exponents (k + 127), row-major [rows][cols / 32] or blocked
  int mx_blocked;      // MX: 1 = the blocked layout (one 512-byte chunk per 128 x 128 box)
  int64_t rows, cols;
  uint32_t nitems;
  FastDiv ngc;        // 128-column groups per row
  int stages;
  int wide_stores;    // cols % 16 == 0: rows start 16-byte aligned, 16-byte code stores
  uint32_t* err;
};

// The exponent k of an MX group's scale 2^k: the smallest k with amax <= FMAX * 2^k, clamped at
// -127; 128 for a NaN or infinite amax.  FMAX = 1.75 * 2^E (E = 8 for E4M3, 15 for E5M2), so for a
// normal amax = M * 2^e: k = e - E, plus one when M > 1.75 (mantissa field above 0x600000).
template <int FMT>
__device__ __forceinline__ int mx_exponent(float amax) {
  constexpr int kEmaxF = FMT == kE4M3 ? 8 : 15;
  const uint32_t b = __float_as_uint(amax);
  const int e = (int)(b >> 23);
  if (e == 255) return 128;
  if (e == 0) return -127;                    // zero or subnormal: below FMAX * 2^-127
  return max(-127, e - 127 - kEmaxF + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0));
}

// eight bf16 times the power of two `mul` (exact) -> eight codes
template <int FMT>
__device__ __forceinline__ uint2 mx_quant8(uint4 v, float mul) {
  const float2 m2 = make_float2(mul, mul);
  const float2 a = __fmul2_rn(make_float2(bf16_lo(v.x), bf16_hi(v.x)), m2);
  const float2 b = __fmul2_rn(make_float2(bf16_lo(v.y), bf16_hi(v.y)), m2);
  const float2 c = __fmul2_rn(make_float2(bf16_lo(v.z), bf16_hi(v.z)), m2);
  const float2 d = __fmul2_rn(make_float2(bf16_lo(v.w), bf16_hi(v.w)), m2);
  return make_uint2(__byte_perm(cvt2<FMT>(a.x, a.y), cvt2<FMT>(b.x, b.y), 0x5410),
                    __byte_perm(cvt2<FMT>(c.x, c.y), cvt2<FMT>(d.x, d.y), 0x5410));
}

// MX = false: 1x128 groups with fp32 scales.  MX = true: MXFP8, 1x32 groups with power-of-two
// scales (one group per thread: thread q of a row's four takes columns [32q, 32q + 32) of the box).
template <int FMT, bool MX>
__global__ void __launch_bounds__(kThreads, 2) k_group128(const __grid_constant__ CUtensorMap tx, GroupParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = ring_base(smem_raw);
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * kGroupStage);
  uint64_t* empty = full + kMaxStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  const uint32_t nk = items_of_cta(p.nitems);
  if (warp == kConsumerWarps && lane == 0 && nk > 0) {
    // warm L2 with this CTA's first boxes while the previous grid on the stream finishes
    tma_prefetch_desc(&tx);
    for (uint32_t k = 0; k < nk && k < (uint32_t)S; ++k) {
      const uint32_t i = blockIdx.x + k * gridDim.x, rb = fdiv(i, p.ngc), g = i - rb * p.ngc.d;
      tma_prefetch_l2_2d(&tx, (int32_t)(g * 128), (int32_t)(rb * kGroupBoxRows));
    }
  }
  __syncthreads();
  allow_dependent_launch();
  grid_dependency_wait();
  if (warp == kConsumerWarps) {
    if (lane == 0 && nk > 0) {
      run_producer(
          full, empty, S, nk, kGroupStage, p.err, [&](uint32_t k) { return blockIdx.x + k * gridDim.x; },
          [&](uint32_t i, int s, uint64_t* bar) {
            const uint32_t rb = fdiv(i, p.ngc), g = i - rb * p.ngc.d;
            tma_load_2d(smem + s * kGroupStage, &tx, (int32_t)(g * 128), (int32_t)(rb * kGroupBoxRows), bar);
          });
    }
    return;
  }
  if constexpr (MX) {
    const int t = threadIdx.x, grp = t >> 2, q = t & 3;
    const uint32_t soff = grp * 256 + q * 64;
    const int64_t ngroups = p.cols / 32;
    int s = 0;
    uint32_t ph = 0;
    for (uint32_t k = 0; k < nk; ++k) {
      const uint32_t i = blockIdx.x + k * gridDim.x;
      if (!mbar_wait(&full[s], ph, p.err)) break;
      uint4 v[kGroupRowsPerThread][4];
      uint32_t m[kGroupRowsPerThread];
#pragma unroll
      for (int h = 0; h < kGroupRowsPerThread; ++h) {
        const uint8_t* src = smem + s * kGroupStage + soff + h * 64 * 256;
        v[h][0] = ld_shared_v4(src);
        v[h][1] = ld_shared_v4(src + 16);
        v[h][2] = ld_shared_v4(src + 32);
        v[h][3] = ld_shared_v4(src + 48);
        m[h] = absmax_v4(absmax_v4(absmax_v4(absmax_v4(0u, v[h][0]), v[h][1]), v[h][2]), v[h][3]);
      }
      release_stage(&empty[s], lane);   // the amax consumed every load
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
      const uint32_t rb = fdiv(i, p.ngc), g = i - rb * p.ngc.d;
#pragma unroll
      for (int h = 0; h < kGroupRowsPerThread; ++h) {
        const int e = mx_exponent<FMT>(packed_amax_to_f32(m[h]));
        const float mul = e == 128 ? __uint_as_float(0x7FC00000u) : __uint_as_float((uint32_t)(127 - e) << 23);
        const int64_t row = (int64_t)rb * kGroupBoxRows + grp + h * 64;
        const int64_t col0 = (int64_t)g * 128 + q * 32;
        if (p.mx_blocked) {
          // the box's 128 rows x 4 groups are one 512-byte chunk: row r of the box at byte
          // 16 (r % 32) + 4 (r / 32), group q beside it; rows and groups past the edge read zeros
          // (the TMA fill), so they store byte 0
          const int r = grp + h * 64;
          p.mx_scales[((int64_t)rb * p.ngc.d + g) * 512 + (r & 31) * 16 + (r >> 5) * 4 + q] = (uint8_t)(e + 127);
        }
        if (row >= p.rows || col0 >= p.cols) continue;
        uint8_t* dst = p.codes + row * p.cols + col0;
        const uint2 c0 = mx_quant8<FMT>(v[h][0], mul), c1 = mx_quant8<FMT>(v[h][1], mul),
                    c2 = mx_quant8<FMT>(v[h][2], mul), c3 = mx_quant8<FMT>(v[h][3], mul);
        st_stream_v4(dst, make_uint4(c0.x, c0.y, c1.x, c1.y));
        st_stream_v4(dst + 16, make_uint4(c2.x, c2.y, c3.x, c3.y));
        if (!p.mx_blocked) p.mx_scales[row * ngroups + g * 4 + q] = (uint8_t)(e + 127);
      }
    }
    return;
  }
  // thread (grp, q) owns chunk pairs q and q + 4 of box row grp: 32 elements, two 16-byte stores
  const int t = threadIdx.x, grp = t >> 2, q = t & 3;
  const uint32_t soff = grp * 256 + q * 32;
  int s = 0;
  uint32_t ph = 0;
  for (uint32_t k = 0; k < nk; ++k) {
    const uint32_t i = blockIdx.x + k * gridDim.x;
    if (!mbar_wait(&full[s], ph, p.err)) break;
    uint4 v[kGroupRowsPerThread][4];
    uint32_t m[kGroupRowsPerThread];
#pragma unroll
    for (int h = 0; h < kGroupRowsPerThread; ++h) {
      const uint8_t* src = smem + s * kGroupStage + soff + h * 64 * 256;
      v[h][0] = ld_shared_v4(src);
      v[h][1] = ld_shared_v4(src + 16);
      v[h][2] = ld_shared_v4(src + 128);
      v[h][3] = ld_shared_v4(src + 144);
      m[h] = absmax_v4(absmax_v4(absmax_v4(absmax_v4(0u, v[h][0]), v[h][1]), v[h][2]), v[h][3]);
    }
    release_stage(&empty[s], lane);   // the amax consumed every load
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
    const uint32_t rb = fdiv(i, p.ngc), g = i - rb * p.ngc.d;
#pragma unroll
    for (int h = 0; h < kGroupRowsPerThread; ++h) {
      uint32_t mh = absmax2(m[h], __shfl_xor_sync(0xFFFFFFFFu, m[h], 1));
      mh = absmax2(mh, __shfl_xor_sync(0xFFFFFFFFu, mh, 2));
      const GroupScale gs = make_group_scale<FMT>(packed_amax_to_f32(mh));
      const int64_t row = (int64_t)rb * kGroupBoxRows + grp + h * 64;
      if (row >= p.rows) continue;
      const int64_t col0 = (int64_t)g * 128 + q * 16, col1 = col0 + 64;
      uint8_t* dst = p.codes + row * p.cols;
      if (gs.fast && p.wide_stores && (int64_t)g * 128 + 128 <= p.cols) {
        st_stream_v4(dst + col0, quant16_fast<FMT>(v[h][0], v[h][1], gs.d, gs.r));
        st_stream_v4(dst + col1, quant16_fast<FMT>(v[h][2], v[h][3], gs.d, gs.r));
      } else {
        if (col0 < p.cols) st_stream_v2(dst + col0, quant8<FMT>(v[h][0], gs));
        if (col0 + 8 < p.cols) st_stream_v2(dst + col0 + 8, quant8<FMT>(v[h][1], gs));
        if (col1 < p.cols) st_stream_v2(dst + col1, quant8<FMT>(v[h][2], gs));
        if (col1 + 8 < p.cols) st_stream_v2(dst + col1 + 8, quant8<FMT>(v[h][3], gs));
      }
      if (q == 0) p.scales[(int64_t)g * p.rows + row] = gs.s;
    }
  }
}

template <int FMT, bool MX>
static cudaError_t launch_group128_fmt(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes,
                                       float* scales, uint8_t* mx_scales, int mx_blocked, cudaStream_t st) {
  const int64_t ngc = (cols + 127) / 128, nrb = (rows + kGroupBoxRows - 1) / kGroupBoxRows;
  const int64_t nitems = ngc * nrb;
  if (nitems == 0) return cudaSuccess;
  CUtensorMap map;
  std::memset(&map, 0, sizeof(map));
  if (!make_tmap_2d(&map, 2, x, (uint64_t)cols, (uint64_t)rows, (uint64_t)cols * 2, 128, kGroupBoxRows, 0))
    return cudaErrorInvalidValue;
  GroupParams p;
  p.codes = codes;
  p.scales = scales;
  p.mx_scales = mx_scales;
  p.mx_blocked = mx_blocked;
  p.rows = rows;
  p.cols = cols;
  p.nitems = (uint32_t)nitems;
  p.ngc = make_fastdiv((uint32_t)ngc);
  p.stages = (int)ring_stages(kGroupStage);
  p.wide_stores = cols % 16 == 0;
  p.err = device_error_word();
  const size_t smem = ring_smem(p.stages, kGroupStage);
  const cudaError_t ea = ensure_dynamic_smem((const void*)k_group128<FMT, MX>, smem);
  if (ea != cudaSuccess) return ea;
  const int grid = grid_for(k_group128<FMT, MX>, smem, p.nitems);
  return launch_pdl(k_group128<FMT, MX>, dim3(grid), dim3(kThreads), smem, st, map, p);
}

cudaError_t launch_quant_1x128(const uint16_t* x, int64_t rows, int64_t cols, int fmt, uint8_t* codes,
                               float* scales, cudaStream_t st) {
  return fmt == kE4M3 ? launch_group128_fmt<kE4M3, false>(x, rows, cols, codes, scales, nullptr, 0, st)
                      : launch_group128_fmt<kE5M2, false>(x, rows, cols, codes, scales, nullptr, 0, st);
}

cudaError_t launch_quant_mx(const uint16_t* x, int64_t rows, int64_t cols, int fmt, uint8_t* codes, uint8_t* scales,
                            int blocked, cudaStream_t st) {
  return fmt == kE4M3 ? launch_group128_fmt<kE4M3, true>(x, rows, cols, codes, nullptr, scales, blocked, st)
                      : launch_group128_fmt<kE5M2, true>(x, rows, cols, codes, nullptr, scales, blocked, st);
}

// ============================================================================ 128-row tiles
//
// Box = 128 rows x bc columns of a [rows][ld] bf16 matrix (bc = 128 for weight blocks and
// per-tensor passes, bc = head_dim for the KV cache).  Thread t owns the 16-byte pieces
// t, t + 256, ... of the box (a warp reads 512 contiguous bytes of shared memory).
//   kOnePass: the box is one scale group (128x128 weight block, 128-token x head KV block):
//             amax over the CTA (shuffles + named barrier), scale, cast, store.
//   kAmax:    pass 1 of per-tensor / per-head: fold the box amax into this CTA's running
//             maximum for the box's group; write them out at the end.
//   kCast:    pass 2: fold all CTAs' partial maxima into the group scales, then cast every
//             box, walking the boxes in the reverse of pass 1's order so the boxes pass 1
//             read last, the likeliest to still be in L2, come first.

constexpr int kOnePass = 0;
constexpr int kAmax = 1;
constexpr int kCast = 2;
constexpr int kDelayed = 3;   // delayed scaling: cast with scales from an amax history, and
                              // record this call's per-CTA maxima like kAmax
constexpr int kMaxGroups = 256;

struct TileParams {
  uint8_t* c0;
  uint8_t* c1;
  float* s0;
  float* s1;
  float* partials;       // kAmax: written [grid][ngroups]; kCast: read [nparts][ngroups]
  int nparts;
  int64_t rows, cols, ld;
  int bc, cpr;           // box columns, 16-byte pieces per box row
  FastDiv nbc;           // boxes across
  FastDiv per_tensor;    // boxes per tensor
  uint32_t nitems;
  int head_groups;       // kAmax / kCast: the group follows the box column (one per head)
  int heads;             // groups per tensor
  int ngroups;
  int stages;
  uint32_t stage_bytes;
  const float* h0;                 // kDelayed: amax histories [hlen][heads] of tensors 0 and 1
  const float* h1;
  int hlen;
  unsigned long long* counters;    // kCast / kDelayed, optional: [2] saturated, underflowed (added to)
  uint32_t* err;
};

struct TileItem {
  uint32_t tens, bi, bj;
};

__device__ __forceinline__ TileItem tile_item(uint32_t i, const TileParams& p) {
  TileItem it;
  it.tens = fdiv(i, p.per_tensor);
  const uint32_t rem = i - it.tens * p.per_tensor.d;
  it.bi = fdiv(rem, p.nbc);
  it.bj = rem - it.bi * p.nbc.d;
  return it;
}

template <int MODE>
__device__ __forceinline__ uint32_t tile_item_index(uint32_t k, uint32_t nitems) {
  const uint32_t fwd = blockIdx.x + k * gridDim.x;
  return MODE == kCast ? nitems - 1 - fwd : fwd;
}

template <int FMT, int MODE, int CPR, int MAXC>
__global__ void __launch_bounds__(kThreads, 2) k_tile128(const __grid_constant__ CUtensorMap t0,
                                                          const __grid_constant__ CUtensorMap t1, TileParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = ring_base(smem_raw);
  __shared__ uint32_t red[2][kConsumerWarps];
  constexpr bool kRecordsAmax = MODE == kAmax || MODE == kDelayed;
  constexpr bool kUsesTable = MODE == kCast || MODE == kDelayed;
  constexpr bool kCanCount = MODE == kCast || MODE == kDelayed;
  __shared__ uint32_t wmax[kRecordsAmax ? kConsumerWarps : 1][kRecordsAmax ? kMaxGroups : 1];
  __shared__ uint32_t fold[MODE == kCast ? kMaxGroups : 1];
  __shared__ GroupScale table[kUsesTable ? kMaxGroups : 1];
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * p.stage_bytes);
  uint64_t* empty = full + kMaxStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  const uint32_t nk = items_of_cta(p.nitems);
  if (warp == kConsumerWarps && lane == 0 && nk > 0) {
    // warm L2 with this CTA's first boxes while the previous grid on the stream finishes
    tma_prefetch_desc(&t0);
    tma_prefetch_desc(&t1);
    for (uint32_t k = 0; k < nk && k < (uint32_t)S; ++k) {
      const TileItem it = tile_item(tile_item_index<MODE>(k, p.nitems), p);
      tma_prefetch_l2_2d(it.tens ? &t1 : &t0, (int32_t)(it.bj * p.bc), (int32_t)(it.bi * 128));
    }
  }
  __syncthreads();
  allow_dependent_launch();
  grid_dependency_wait();
  if (warp == kConsumerWarps) {
    if (lane == 0 && nk > 0) {
      run_producer(
          full, empty, S, nk, p.stage_bytes, p.err, [&](uint32_t k) { return tile_item_index<MODE>(k, p.nitems); },
          [&](uint32_t i, int s, uint64_t* bar) {
            const TileItem it = tile_item(i, p);
            tma_load_2d(smem + s * p.stage_bytes, it.tens ? &t1 : &t0, (int32_t)(it.bj * p.bc),
                        (int32_t)(it.bi * 128), bar);
          });
    }
    return;
  }
  const int t = threadIdx.x;
  const int cpr = CPR > 0 ? CPR : p.cpr;
  const int nchunks = 128 * cpr;

  if (kRecordsAmax) {
    for (int g = lane; g < kMaxGroups; g += 32) wmax[warp][g] = 0u;
    __syncwarp();
  }
  if (MODE == kDelayed) {
    // the scale of each group comes from the largest amax of its history (entries >= 0 or NaN,
    // which order like their bit patterns; NaN stays)
    for (int g = t; g < p.ngroups; g += kConsumers) {
      const int tens = g / p.heads, gl = g - tens * p.heads;
      const float* h = tens ? p.h1 : p.h0;
      uint32_t hm = 0u;
      for (int j = 0; j < p.hlen; ++j) hm = max(hm, __float_as_uint(h[(size_t)j * p.heads + gl]));
      table[g] = make_delayed_scale<FMT>(__uint_as_float(hm));
      if (blockIdx.x == 0) (tens ? p.s1 : p.s0)[gl] = table[g].s;
    }
    named_barrier(1, kConsumers);
  }
  if (MODE == kCast) {
    // fold the partial maxima: non-negative floats (or NaN) order like their bit patterns
    for (int g = t; g < p.ngroups; g += kConsumers) fold[g] = 0u;
    named_barrier(1, kConsumers);
    const int nitems_p = p.nparts * p.ngroups;
    for (int it = t; it < nitems_p; it += kConsumers)
      atomicMax(&fold[it % p.ngroups], __float_as_uint(p.partials[it]));
    named_barrier(1, kConsumers);
    for (int g = t; g < p.ngroups; g += kConsumers) {
      table[g] = make_group_scale<FMT>(__uint_as_float(fold[g]));
      if (blockIdx.x == 0) {
        const int tens = g / p.heads;
        (tens ? p.s1 : p.s0)[g - tens * p.heads] = table[g].s;
      }
    }
    named_barrier(1, kConsumers);
  }

  // CPR > 0: thread t owns chunk pairs t + 256 * jp (32 smem bytes each; pair q of the box sits
  // at row q / PPR, 16-column block q % PPR); interior boxes with a fast scale take 16-byte
  // stores with no per-chunk checks.  CPR == 0 (unusual head sizes): single chunks, all checked.
  constexpr int PPR = CPR / 2;
  constexpr int MAXP = CPR > 0 ? CPR / 4 : 1;
  constexpr int ROWSTEP = CPR > 0 ? kConsumers / PPR : 1;
  const int r0 = CPR > 0 ? t / PPR : 0, cp = CPR > 0 ? t % PPR : 0;
  const bool wide = (p.ld % 16) == 0;
  const bool count = kCanCount && p.counters != nullptr;
  uint32_t n_sat = 0, n_und = 0;
  int s = 0;
  uint32_t ph = 0;
  for (uint32_t k = 0; k < nk; ++k) {
    const uint32_t i = tile_item_index<MODE>(k, p.nitems);
    if (!mbar_wait(&full[s], ph, p.err)) break;
    const uint8_t* stage = smem + s * p.stage_bytes;
    uint4 va[CPR > 0 ? MAXP : MAXC], vb[CPR > 0 ? MAXP : 1];
    uint32_t m = 0u;
    if constexpr (CPR > 0) {
#pragma unroll
      for (int jp = 0; jp < MAXP; ++jp) {
        const uint8_t* src = stage + (t + kConsumers * jp) * 32;
        va[jp] = ld_shared_v4(src);
        vb[jp] = ld_shared_v4(src + 16);
        if (MODE != kCast) m = absmax_v4(absmax_v4(m, va[jp]), vb[jp]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < MAXC; ++j) {
        const int c = t + kConsumers * j;
        va[j] = c < nchunks ? ld_shared_v4(stage + c * 16) : make_uint4(0u, 0u, 0u, 0u);
        if (MODE != kCast) m = absmax_v4(m, va[j]);
      }
    }
    // the amax consumed every load; the cast pass releases the stage after the cast instead
    uint64_t* release = &empty[s];
    if (MODE != kCast) release_stage(release, lane);
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
    const TileItem it = tile_item(i, p);
    if (MODE != kCast) {
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) m = absmax2(m, __shfl_xor_sync(0xFFFFFFFFu, m, d));
    }
    if (kRecordsAmax) {
      if (lane == 0) {
        const int g = (int)it.tens * p.heads + (p.head_groups ? (int)it.bj : 0);
        const uint32_t a = __float_as_uint(packed_amax_to_f32(m));
        wmax[warp][g] = max(wmax[warp][g], a);
      }
      if (MODE == kAmax) continue;
    }
    GroupScale gs;
    if (MODE == kOnePass) {
      if (lane == 0) red[k & 1][warp] = m;
      named_barrier(1, kConsumers);
      uint32_t mm = red[k & 1][0];
#pragma unroll
      for (int w = 1; w < kConsumerWarps; ++w) mm = absmax2(mm, red[k & 1][w]);
      gs = make_group_scale<FMT>(packed_amax_to_f32(mm));
      if (t == 0) (it.tens ? p.s1 : p.s0)[it.bi * p.nbc.d + it.bj] = gs.s;
    } else {
      gs = table[(int)it.tens * p.heads + (p.head_groups ? (int)it.bj : 0)];
    }
    uint8_t* codes = it.tens ? p.c1 : p.c0;
    const int64_t row_base = (int64_t)it.bi * 128, col_base = (int64_t)it.bj * p.bc;
    if constexpr (CPR > 0) {
      const bool interior = row_base + 128 <= p.rows && col_base + p.bc <= p.cols;
      if (gs.fast && interior && wide) {
        uint8_t* dst = codes + (row_base + r0) * p.ld + col_base + cp * 16;
        const int64_t step = (int64_t)ROWSTEP * p.ld;
#pragma unroll
        for (int jp = 0; jp < MAXP; ++jp) {
          const uint4 q = quant16_fast<FMT>(va[jp], vb[jp], gs.d, gs.r);
          st_stream_v4(dst + jp * step, q);
          if (count) {
            count8<FMT>(va[jp], make_uint2(q.x, q.y), gs, n_sat, n_und);
            count8<FMT>(vb[jp], make_uint2(q.z, q.w), gs, n_sat, n_und);
          }
        }
      } else {
#pragma unroll
        for (int jp = 0; jp < MAXP; ++jp) {
          const int64_t row = row_base + r0 + jp * ROWSTEP;
          const int64_t col = col_base + cp * 16;
          uint8_t* dst = codes + row * p.ld + col;
          if (row < p.rows && col < p.cols) {
            const uint2 q = quant8<FMT>(va[jp], gs);
            st_stream_v2(dst, q);
            if (count) count8<FMT>(va[jp], q, gs, n_sat, n_und);
          }
          if (row < p.rows && col + 8 < p.cols) {
            const uint2 q = quant8<FMT>(vb[jp], gs);
            st_stream_v2(dst + 8, q);
            if (count) count8<FMT>(vb[jp], q, gs, n_sat, n_und);
          }
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < MAXC; ++j) {
        const int c = t + kConsumers * j;
        const int r = c / cpr, cc = c - r * cpr;
        const int64_t row = row_base + r;
        const int64_t col = col_base + cc * 8;
        const uint2 q = quant8<FMT>(va[j], gs);
        if (c < nchunks && row < p.rows && col < p.cols) {
          st_stream_v2(codes + row * p.ld + col, q);
          if (count) count8<FMT>(va[j], q, gs, n_sat, n_und);
        }
      }
    }
    if (MODE == kCast) release_stage(release, lane);
  }
  if (count) {
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
      n_sat += __shfl_xor_sync(0xFFFFFFFFu, n_sat, d);
      n_und += __shfl_xor_sync(0xFFFFFFFFu, n_und, d);
    }
    if (lane == 0) {
      if (n_sat) atomicAdd(p.counters, (unsigned long long)n_sat);
      if (n_und) atomicAdd(p.counters + 1, (unsigned long long)n_und);
    }
  }
  if (kRecordsAmax) {
    named_barrier(1, kConsumers);
    for (int g = t; g < p.ngroups; g += kConsumers) {
      uint32_t mx = wmax[0][g];
#pragma unroll
      for (int w = 1; w < kConsumerWarps; ++w) mx = max(mx, wmax[w][g]);
      p.partials[(size_t)blockIdx.x * p.ngroups + g] = __uint_as_float(mx);
    }
  }
}

template <int FMT, int MODE, int CPR, int MAXC>
static cudaError_t launch_tile_impl(const CUtensorMap& m0, const CUtensorMap& m1, TileParams& p, int max_grid,
                                    cudaStream_t st, int* grid_used) {
  const size_t smem = ring_smem(p.stages, p.stage_bytes);
  const cudaError_t ea = ensure_dynamic_smem((const void*)k_tile128<FMT, MODE, CPR, MAXC>, smem);
  if (ea != cudaSuccess) return ea;
  int grid = grid_for(k_tile128<FMT, MODE, CPR, MAXC>, smem, std::max<uint32_t>(p.nitems, 1));
  if (max_grid > 0) grid = std::min(grid, max_grid);
  if (grid_used) *grid_used = grid;
  return launch_pdl(k_tile128<FMT, MODE, CPR, MAXC>, dim3(grid), dim3(kThreads), smem, st, m0, m1, p);
}

template <int FMT, int MODE>
static cudaError_t launch_tile_fmt(const CUtensorMap& m0, const CUtensorMap& m1, TileParams& p, int max_grid,
                                   cudaStream_t st, int* grid_used) {
  if (p.bc == 128) return launch_tile_impl<FMT, MODE, 16, 8>(m0, m1, p, max_grid, st, grid_used);
  if (p.bc == 64) return launch_tile_impl<FMT, MODE, 8, 4>(m0, m1, p, max_grid, st, grid_used);
  if (p.bc == 256) return launch_tile_impl<FMT, MODE, 32, 16>(m0, m1, p, max_grid, st, grid_used);
  if (p.bc < 128) return launch_tile_impl<FMT, MODE, 0, 8>(m0, m1, p, max_grid, st, grid_used);
  return launch_tile_impl<FMT, MODE, 0, 16>(m0, m1, p, max_grid, st, grid_used);
}

template <int MODE>
static cudaError_t launch_tile(int fmt, const CUtensorMap& m0, const CUtensorMap& m1, TileParams& p, int max_grid,
                               cudaStream_t st, int* grid_used = nullptr) {
  return fmt == kE4M3 ? launch_tile_fmt<kE4M3, MODE>(m0, m1, p, max_grid, st, grid_used)
                      : launch_tile_fmt<kE5M2, MODE>(m0, m1, p, max_grid, st, grid_used);
}

// common set-up of a tile launch over ntens tensors of [rows][cols] (row stride ld) with
// boxes of 128 x bc
static bool tile_setup(TileParams& p, CUtensorMap& m0, CUtensorMap& m1, const uint16_t* x0, const uint16_t* x1,
                       int ntens, int64_t rows, int64_t cols, int64_t ld, int bc) {
  std::memset(&m0, 0, sizeof(m0));
  std::memset(&m1, 0, sizeof(m1));
  p.rows = rows;
  p.cols = cols;
  p.ld = ld;
  p.bc = bc;
  p.cpr = bc / 8;
  const int64_t nbr = (rows + 127) / 128, nbc = (cols + bc - 1) / bc;
  p.nbc = make_fastdiv((uint32_t)std::max<int64_t>(nbc, 1));
  p.per_tensor = make_fastdiv((uint32_t)std::max<int64_t>(nbr * nbc, 1));
  p.nitems = (uint32_t)(ntens * nbr * nbc);
  p.stage_bytes = (uint32_t)(128 * bc * 2);
  p.stages = (int)ring_stages(p.stage_bytes);
  p.err = device_error_word();
  p.partials = nullptr;
  p.nparts = 0;
  p.h0 = p.h1 = nullptr;
  p.hlen = 0;
  p.counters = nullptr;
  p.head_groups = 0;
  p.heads = 1;
  p.ngroups = ntens;
  if (p.nitems == 0) return true;
  if (!make_tmap_2d(&m0, 2, x0, (uint64_t)cols, (uint64_t)rows, (uint64_t)ld * 2, (uint32_t)bc, 128, 0)) return false;
  if (!make_tmap_2d(&m1, 2, ntens > 1 ? x1 : x0, (uint64_t)cols, (uint64_t)rows, (uint64_t)ld * 2, (uint32_t)bc, 128,
                    0))
    return false;
  return true;
}

cudaError_t launch_quant_tiles(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                               float* s1, int ntens, int64_t rows, int64_t cols, int64_t ld, int gw, int fmt,
                               cudaStream_t st) {
  TileParams p;
  CUtensorMap m0, m1;
  if (!tile_setup(p, m0, m1, x0, x1, ntens, rows, cols, ld, gw)) return cudaErrorInvalidValue;
  if (p.nitems == 0) return cudaSuccess;
  p.c0 = c0;
  p.c1 = ntens > 1 ? c1 : c0;
  p.s0 = s0;
  p.s1 = ntens > 1 ? s1 : s0;
  return launch_tile<kOnePass>(fmt, m0, m1, p, 0, st);
}

// ============================================================================ two passes
//
// Per-tensor and per-head scales need the amax of a group spanning a whole tensor (or all
// tokens of a head) before any of its elements can be cast: pass 1 (kAmax) writes per-CTA
// partial maxima to the workspace, pass 2 (kCast) folds them and casts.

size_t two_pass_workspace_bytes(int ntens, int64_t heads) {
  return (size_t)kMaxPartials * (size_t)ntens * (size_t)std::max<int64_t>(heads, 1) * sizeof(float);
}

// shared set-up of the two-pass and delayed launches: boxes of 128 x 128 over
// [rows][heads * head_dim] for per-tensor groups, 128 tokens x head_dim per (tensor, head)
static bool group_setup(TileParams& p, CUtensorMap& m0, CUtensorMap& m1, const uint16_t* x0, const uint16_t* x1,
                        uint8_t* c0, uint8_t* c1, float* s0, float* s1, int ntens, int64_t rows, int64_t heads,
                        int64_t head_dim, float* ws) {
  const int64_t cols = heads * head_dim;
  const bool per_head = heads > 1;
  const int bc = per_head ? (int)head_dim : 128;
  if (ntens * (per_head ? heads : 1) > kMaxGroups) return false;
  if (!tile_setup(p, m0, m1, x0, x1, ntens, rows, cols, cols, bc)) return false;
  p.c0 = c0;
  p.c1 = ntens > 1 ? c1 : c0;
  p.s0 = s0;
  p.s1 = ntens > 1 ? s1 : s0;
  p.head_groups = per_head ? 1 : 0;
  p.heads = per_head ? (int)heads : 1;
  p.ngroups = ntens * p.heads;
  p.partials = ws;
  return true;
}

// the two passes; *nparts receives the number of partial rows pass 1 wrote (0 for empty input)
static cudaError_t two_pass(TileParams& p, const CUtensorMap& m0, const CUtensorMap& m1, int fmt, cudaStream_t st,
                            int* nparts) {
  if (p.nitems == 0) {
    // empty tensors: amax = 0 for every group, so pass 2 alone writes s = 0
    p.nparts = 0;
    *nparts = 0;
    return launch_tile<kCast>(fmt, m0, m1, p, 1, st);
  }
  const int grid1 = (int)std::min<int64_t>((int64_t)p.nitems, std::min<int64_t>(kMaxPartials, 2 * device_sm_count()));
  p.nparts = 0;
  int written = 0;
  cudaError_t e = launch_tile<kAmax>(fmt, m0, m1, p, grid1, st, &written);
  if (e != cudaSuccess) return e;
  p.nparts = written;   // partial rows pass 1 wrote (its grid size)
  *nparts = written;
  return launch_tile<kCast>(fmt, m0, m1, p, written, st);
}

cudaError_t launch_quant_two_pass(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                                  float* s1, int ntens, int64_t rows, int64_t heads, int64_t head_dim, int fmt,
                                  float* ws, cudaStream_t st) {
  TileParams p;
  CUtensorMap m0, m1;
  if (!group_setup(p, m0, m1, x0, x1, c0, c1, s0, s1, ntens, rows, heads, head_dim, ws)) return cudaErrorInvalidValue;
  int nparts = 0;
  return two_pass(p, m0, m1, fmt, st, &nparts);
}

// ============================================================================ delayed scaling
//
// Step 0 has no history: the two passes above (the group's own amax).  Step t >= 1: one pass
// (kDelayed) casting with s = RN(max(history) / FMAX) while it records per-CTA maxima.  Either
// way k_history_update then folds the recorded maxima into history slot t mod hlen.

__global__ void __launch_bounds__(256) k_history_update(const float* partials, int nparts, int ngroups, int heads,
                                                        float* h0, float* h1, int64_t slot) {
  allow_dependent_launch();
  grid_dependency_wait();
  // one warp per group: lanes stride over the CTAs' partial maxima (independent loads), then a
  // shuffle reduction; amax values are >= 0 or NaN and order like their bit patterns
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int g = warp; g < ngroups; g += nwarps) {
    uint32_t m = 0u;
    for (int c = lane; c < nparts; c += 32) m = max(m, __float_as_uint(partials[(size_t)c * ngroups + g]));
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, d));
    if (lane == 0) {
      const int tens = g / heads, gl = g - tens * heads;
      (tens ? h1 : h0)[slot * heads + gl] = __uint_as_float(m);
    }
  }
}

cudaError_t launch_quant_delayed(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                                 float* s1, int ntens, int64_t rows, int64_t heads, int64_t head_dim, int fmt,
                                 float* h0, float* h1, int64_t hlen, int64_t step, unsigned long long* counters,
                                 float* ws, cudaStream_t st) {
  TileParams p;
  CUtensorMap m0, m1;
  if (!group_setup(p, m0, m1, x0, x1, c0, c1, s0, s1, ntens, rows, heads, head_dim, ws)) return cudaErrorInvalidValue;
  p.counters = counters;
  p.h0 = h0;
  p.h1 = ntens > 1 ? h1 : h0;
  p.hlen = (int)hlen;
  int nparts = 0;
  cudaError_t e;
  if (step == 0) {
    e = two_pass(p, m0, m1, fmt, st, &nparts);
  } else {
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>((int64_t)p.nitems, std::min<int64_t>(kMaxPartials, 2 * device_sm_count())));
    e = launch_tile<kDelayed>(fmt, m0, m1, p, grid, st, &nparts);
  }
  if (e != cudaSuccess) return e;
  return launch_pdl(k_history_update, dim3(1), dim3(256), 0, st, (const float*)ws, nparts, p.ngroups, p.heads, h0,
                    ntens > 1 ? h1 : h0, step % hlen);
}


// ============================================================================ several tensors, one launch
//
// Up to kMaxJobs tensors, each quantized in 1x128 groups or 128x128 blocks, in one persistent
// launch: every tensor is cut into 128 x 128 bf16 boxes (the 32 KB stages above), the boxes of
// all tensors form one item list split over the CTAs with the grid stride, so one ring, one ramp
// and one tail serve them all, and the work divides evenly however the tensors' box counts fall.
// A box is consumed as its tensor's granularity requires, with the arithmetic of k_group128
// (per-row amax, four threads per row) or of k_tile128's one-pass mode (CTA-wide amax): the
// codes and scales are those of separate calls.

struct ManyJob {
  uint8_t* codes;
  float* scales;
  int64_t rows, cols;
  uint32_t first;    // first item of this tensor in the combined list
  FastDiv nbc;       // 128-column boxes across
  int block;         // 1: 128x128 blocks; 0: 1x128 groups
  int wide;          // cols % 16 == 0: 16-byte code stores
};

struct ManyMaps {
  CUtensorMap m[kMaxManyJobs];
};

struct ManyParams {
  ManyJob job[kMaxManyJobs];
  int njobs;
  uint32_t nitems;
  int stages;
  uint32_t* err;
};

__device__ __forceinline__ int many_job_of(uint32_t i, const ManyParams& p) {
  int j = 0;
  while (j + 1 < p.njobs && i >= p.job[j + 1].first) ++j;
  return j;
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 2) k_quant_many(const __grid_constant__ ManyMaps maps,
                                                             const __grid_constant__ ManyParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = ring_base(smem_raw);
  __shared__ uint32_t red[2][kConsumerWarps];
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * kGroupStage);
  uint64_t* empty = full + kMaxStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  const uint32_t nk = items_of_cta(p.nitems);
  if (warp == kConsumerWarps && lane == 0 && nk > 0) {
    // warm L2 with this CTA's first boxes while the previous grid on the stream finishes
    for (int j = 0; j < p.njobs; ++j)
      if (p.job[j].rows > 0 && p.job[j].cols > 0) tma_prefetch_desc(&maps.m[j]);
    for (uint32_t k = 0; k < nk && k < (uint32_t)S; ++k) {
      const uint32_t i = blockIdx.x + k * gridDim.x;
      const int j = many_job_of(i, p);
      const uint32_t local = i - p.job[j].first, rb = fdiv(local, p.job[j].nbc), g = local - rb * p.job[j].nbc.d;
      tma_prefetch_l2_2d(&maps.m[j], (int32_t)(g * 128), (int32_t)(rb * 128));
    }
  }
  __syncthreads();
  allow_dependent_launch();
  grid_dependency_wait();
  if (warp == kConsumerWarps) {
    if (lane == 0 && nk > 0) {
      run_producer(
          full, empty, S, nk, kGroupStage, p.err, [&](uint32_t k) { return blockIdx.x + k * gridDim.x; },
          [&](uint32_t i, int s, uint64_t* bar) {
            const int j = many_job_of(i, p);
            const uint32_t local = i - p.job[j].first, rb = fdiv(local, p.job[j].nbc), g = local - rb * p.job[j].nbc.d;
            tma_load_2d(smem + s * kGroupStage, &maps.m[j], (int32_t)(g * 128), (int32_t)(rb * 128), bar);
          });
    }
    return;
  }
  const int t = threadIdx.x;
  int s = 0;
  uint32_t ph = 0, nblock = 0;   // nblock: 128x128 items so far (their reduction slots alternate)
  for (uint32_t k = 0; k < nk; ++k) {
    const uint32_t i = blockIdx.x + k * gridDim.x;
    const ManyJob& J = p.job[many_job_of(i, p)];
    const uint32_t local = i - J.first, rb = fdiv(local, J.nbc), g = local - rb * J.nbc.d;
    if (!mbar_wait(&full[s], ph, p.err)) break;
    const uint8_t* stage = smem + s * kGroupStage;
    if (J.block) {
      // 128x128 block (k_tile128 one-pass, 16-byte pieces per row CPR = 16): thread t owns the
      // 32-byte chunk pairs t + 256 jp, i.e. rows t / 8 + 32 jp, 16-column block t % 8
      uint4 va[4], vb[4];
      uint32_t m = 0u;
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {
        const uint8_t* src = stage + (t + kConsumers * jp) * 32;
        va[jp] = ld_shared_v4(src);
        vb[jp] = ld_shared_v4(src + 16);
        m = absmax_v4(absmax_v4(m, va[jp]), vb[jp]);
      }
      release_stage(&empty[s], lane);
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) m = absmax2(m, __shfl_xor_sync(0xFFFFFFFFu, m, d));
      const uint32_t slot = nblock++ & 1u;
      if (lane == 0) red[slot][warp] = m;
      named_barrier(1, kConsumers);
      uint32_t mm = red[slot][0];
#pragma unroll
      for (int w = 1; w < kConsumerWarps; ++w) mm = absmax2(mm, red[slot][w]);
      const GroupScale gs = make_group_scale<FMT>(packed_amax_to_f32(mm));
      if (t == 0) J.scales[(size_t)rb * J.nbc.d + g] = gs.s;
      const int r0 = t >> 3, cp = t & 7;
      const int64_t row_base = (int64_t)rb * 128, col_base = (int64_t)g * 128;
      if (gs.fast && J.wide && row_base + 128 <= J.rows && col_base + 128 <= J.cols) {
        uint8_t* dst = J.codes + (row_base + r0) * J.cols + col_base + cp * 16;
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) st_stream_v4(dst + jp * 32 * J.cols, quant16_fast<FMT>(va[jp], vb[jp], gs.d, gs.r));
      } else {
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) {
          const int64_t row = row_base + r0 + jp * 32, col = col_base + cp * 16;
          uint8_t* dst = J.codes + row * J.cols + col;
          if (row < J.rows && col < J.cols) st_stream_v2(dst, quant8<FMT>(va[jp], gs));
          if (row < J.rows && col + 8 < J.cols) st_stream_v2(dst + 8, quant8<FMT>(vb[jp], gs));
        }
      }
    } else {
      // 1x128 groups (k_group128): thread (grp, q) owns chunk pairs q and q + 4 of box rows grp
      // and grp + 64
      const int grp = t >> 2, q = t & 3;
      const uint32_t soff = grp * 256 + q * 32;
      uint4 v[kGroupRowsPerThread][4];
      uint32_t m[kGroupRowsPerThread];
#pragma unroll
      for (int h = 0; h < kGroupRowsPerThread; ++h) {
        const uint8_t* src = stage + soff + h * 64 * 256;
        v[h][0] = ld_shared_v4(src);
        v[h][1] = ld_shared_v4(src + 16);
        v[h][2] = ld_shared_v4(src + 128);
        v[h][3] = ld_shared_v4(src + 144);
        m[h] = absmax_v4(absmax_v4(absmax_v4(absmax_v4(0u, v[h][0]), v[h][1]), v[h][2]), v[h][3]);
      }
      release_stage(&empty[s], lane);
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
#pragma unroll
      for (int h = 0; h < kGroupRowsPerThread; ++h) {
        uint32_t mh = absmax2(m[h], __shfl_xor_sync(0xFFFFFFFFu, m[h], 1));
        mh = absmax2(mh, __shfl_xor_sync(0xFFFFFFFFu, mh, 2));
        const GroupScale gs = make_group_scale<FMT>(packed_amax_to_f32(mh));
        const int64_t row = (int64_t)rb * kGroupBoxRows + grp + h * 64;
        if (row >= J.rows) continue;
        const int64_t col0 = (int64_t)g * 128 + q * 16, col1 = col0 + 64;
        uint8_t* dst = J.codes + row * J.cols;
        if (gs.fast && J.wide && (int64_t)g * 128 + 128 <= J.cols) {
          st_stream_v4(dst + col0, quant16_fast<FMT>(v[h][0], v[h][1], gs.d, gs.r));
          st_stream_v4(dst + col1, quant16_fast<FMT>(v[h][2], v[h][3], gs.d, gs.r));
        } else {
          if (col0 < J.cols) st_stream_v2(dst + col0, quant8<FMT>(v[h][0], gs));
          if (col0 + 8 < J.cols) st_stream_v2(dst + col0 + 8, quant8<FMT>(v[h][1], gs));
          if (col1 < J.cols) st_stream_v2(dst + col1, quant8<FMT>(v[h][2], gs));
          if (col1 + 8 < J.cols) st_stream_v2(dst + col1 + 8, quant8<FMT>(v[h][3], gs));
        }
        if (q == 0) J.scales[(int64_t)g * J.rows + row] = gs.s;
      }
    }
  }
}

template <int FMT>
static cudaError_t launch_many_fmt(const ManyMaps& maps, const ManyParams& p, cudaStream_t st) {
  const size_t smem = ring_smem(p.stages, kGroupStage);
  const cudaError_t ea = ensure_dynamic_smem((const void*)k_quant_many<FMT>, smem);
  if (ea != cudaSuccess) return ea;
  const int grid = grid_for(k_quant_many<FMT>, smem, p.nitems);
  return launch_pdl(k_quant_many<FMT>, dim3(grid), dim3(kThreads), smem, st, maps, p);
}

cudaError_t launch_quant_many(const QuantJob* jobs, int n, int fmt, cudaStream_t st) {
  if (n < 1 || n > kMaxManyJobs) return cudaErrorInvalidValue;
  ManyMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  ManyParams p;
  std::memset(&p, 0, sizeof(p));
  uint64_t items = 0;
  for (int j = 0; j < n; ++j) {
    const QuantJob& q = jobs[j];
    ManyJob& J = p.job[j];
    J.codes = q.codes;
    J.scales = q.scales;
    J.rows = q.rows;
    J.cols = q.cols;
    J.block = q.block;
    J.wide = q.cols % 16 == 0;
    const int64_t nbr = (q.rows + 127) / 128, nbc = (q.cols + 127) / 128;
    J.nbc = make_fastdiv((uint32_t)std::max<int64_t>(nbc, 1));
    J.first = (uint32_t)items;
    items += (uint64_t)(nbr * nbc);
    if (items >= (1ull << 32)) return cudaErrorInvalidValue;
    if (nbr * nbc > 0 &&
        !make_tmap_2d(&maps.m[j], 2, q.x, (uint64_t)q.cols, (uint64_t)q.rows, (uint64_t)q.cols * 2, 128, 128, 0))
      return cudaErrorInvalidValue;
  }
  if (items == 0) return cudaSuccess;
  p.njobs = n;
  p.nitems = (uint32_t)items;
  p.stages = (int)ring_stages(kGroupStage);
  p.err = device_error_word();
  return fmt == kE4M3 ? launch_many_fmt<kE4M3>(maps, p, st) : launch_many_fmt<kE5M2>(maps, p, st);
}

}  // namespace fp8q
