// Block-scaled FP8 GEMM on the fifth-generation tensor cores (sm_100a: tcgen05 + TMEM, fed by TMA).
//
// Method: wangyu.me "大语言模型量化技术（五）：FP8", sections "激活动态量化" (the product splits into
// 128-wide K blocks, y = sum_j s_x,j s_w,j (x_hat^(j) W_hat^(j))) and "FP8 矩阵乘" (each block
// product on the FP8 tensor cores with fp32 accumulation; the scales multiplied back as the
// partial results are accumulated).  With 1x128 activation scales the activation scale varies
// along K too, so it sits inside the sum: C[m][n] = sum_kb sA[kb][m] * sB[n/128][kb] * P_kb[m][n].
//
// One persistent CTA per SM walks output tiles of 128 x 256 (m fastest, so concurrent CTAs share
// B tiles and the A panel stays in L2):
//   warp 0      TMA producer: A box 128 x 128 and B box 256 x 128 (E4M3 bytes, 128-byte
//               swizzle) per K block into a 4-stage shared-memory ring.
//   warp 1      allocates all 512 TMEM columns; lane 0 issues four tcgen05.mma (M128 N256 K32,
//               kind::f8f6f4, fp32 accumulate) per K block.
//   warp 2      block-scaled path: copies each K block's A row scales and B scales (cp.async)
//               into an 8-slot shared-memory ring for the epilogue.
//   warp 3      idle (completes warpgroup 0, which hands its registers to the epilogue).
//   warps 4-11  promotion / epilogue.  Block-scaled: each K block's partial P_kb goes to one of
//               two 256-column TMEM buffers; while the tensor cores fill the other buffer, each
//               thread loads its row's 128 columns (tcgen05.ld) and accumulates
//               acc += (sA * sB) * P_kb in fp32 registers; at the end of the tile the
//               accumulators are rounded to bf16 and stored.  Per-tensor scales: the MMAs
//               accumulate all of K in TMEM (two buffers alternate between tiles) and the
//               epilogue scales once.
// Every mbarrier wait is bounded (see sm100.cuh): on a timeout the kernel records an error in
// the device error word and winds down instead of hanging.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "fp8q_device.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tcgen05.cuh"

namespace fp8q {

namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int kStages = 4;
constexpr uint32_t kStageA = BM * BK;             // 16 KB of E4M3
constexpr uint32_t kStageB = BN * BK;             // 32 KB
constexpr uint32_t kStageBytes = kStageA + kStageB;
constexpr int kEpiWarps = 8;
constexpr int kFirstEpiWarp = 4;                  // warpgroup 0: producer, MMA, two idle warps
constexpr int kThreads = 128 + 32 * kEpiWarps;    // three warpgroups
constexpr uint32_t kTmemCols = 512;               // two 128 x 256 fp32 accumulators

// Register split.  The kernel is launched with kLaunchRegs registers per thread (enforced by the
// build, which checks ptxas' report): 384 x 168 = 64512.  Warpgroup 0 gives registers back and
// the two epilogue warpgroups take them: 128 x 40 + 256 x 232 = 64512, the launch's total, so
// setmaxnreg.inc always finds its registers.  Per SM sub-partition (one warp of each warpgroup):
// 40 + 232 + 232 = 504 registers x 32 lanes = 16128 <= 16384.
constexpr int kScaleSlots = 8;                    // scale ring depth (K blocks)
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 40;
constexpr int kEpilogueRegs = 232;
static_assert(128 * kProducerRegs + 256 * kEpilogueRegs == kThreads * kLaunchRegs, "register split must add up");

// kind::f8f6f4 instruction descriptor: D fp32, A = B = E4M3, both K-major, N = 256, M = 128
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

struct Params {
  int M, N, K;
  int num_kb;
  int m_tiles, n_tiles, tiles;
  int group_m;        // tile walk band height (tile_walk)
  const float* sA;
  const float* sB;
  int gA_group;       // 1: sA is [K/128][M]; 0: one scale
  int gB_block;       // 1: sB is [N/128][K/128]; 0: one scale
  const uint8_t* Bp;  // packed B tiles (16 KB each, tile (nb, kb) at nb * num_kb + kb), or null: B via TMA
  uint16_t* C;
  uint8_t* q_codes;   // non-null: the output is quantized (E4M3, 1x128 groups) instead of stored as bf16
  float* q_scales;    // [N/128][M]
  // non-null: a first phase quantizes these bf16 activations [M][K] into the A codes and 1x128
  // scales the GEMM then reads (xq_codes / sA), behind a grid barrier on gbar (cooperative launch)
  const uint16_t* xq;
  uint8_t* xq_codes;
  uint32_t* gbar;     // [0] arrivals (zero between calls), [1] generation
  uint32_t* err;
};

// The 1x128 E4M3 quantizer on one 128-column row segment of C held by one thread; pair(i) gives
// the segment's bf16 pair i (0..63), the values a bf16 C would store: the group's amax, its
// scale, the codes and the scale, with the arithmetic of the stand-alone quantizer, so the
// result equals quantizing the bf16 C in a second pass.
template <class PairFn>
__device__ __forceinline__ void store_row_e4m3(PairFn pair, uint8_t* codes_row, float* scale) {
  uint32_t m = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = absmax_v4(m, make_uint4(pair(4 * i), pair(4 * i + 1), pair(4 * i + 2), pair(4 * i + 3)));
  const GroupScale gs = make_group_scale<kE4M3>(packed_amax_to_f32(m));
  if (gs.fast) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {   // 32 codes per 32-byte store
      const uint4 q0 = quant16_fast<kE4M3>(make_uint4(pair(16 * c), pair(16 * c + 1), pair(16 * c + 2), pair(16 * c + 3)),
                                           make_uint4(pair(16 * c + 4), pair(16 * c + 5), pair(16 * c + 6), pair(16 * c + 7)),
                                           gs.d, gs.r);
      const uint4 q1 =
          quant16_fast<kE4M3>(make_uint4(pair(16 * c + 8), pair(16 * c + 9), pair(16 * c + 10), pair(16 * c + 11)),
                              make_uint4(pair(16 * c + 12), pair(16 * c + 13), pair(16 * c + 14), pair(16 * c + 15)),
                              gs.d, gs.r);
      st_stream_v8(codes_row + 32 * c, q0, q1);
    }
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c)
      st_stream_v2(codes_row + 8 * c, quant8<kE4M3>(make_uint4(pair(4 * c), pair(4 * c + 1), pair(4 * c + 2), pair(4 * c + 3)), gs));
  }
  *scale = gs.s;
}

constexpr int kPhaseDepth = 16;

// First phase of the fused linear layer: every warp of the grid quantizes 1x128 groups of the
// bf16 activations (group g = row g / nkb, K block g % nkb) with the arithmetic of the stand-alone
// 1x128 kernel; then the grid meets at a barrier (all CTAs are resident: the kernel is launched
// cooperatively) so no A tile is loaded before every code and scale is written.  Returns false
// if the barrier's wait gave up (error word set).
__device__ __forceinline__ bool quantize_phase(const uint16_t* __restrict__ xq, uint8_t* __restrict__ xq_codes,
                                             float* __restrict__ sA, uint32_t M, uint32_t K, uint32_t* gbar,
                                             uint32_t* err) {
  __shared__ uint32_t s_flag_bar;
  const uint32_t nkb = K / 128u;
  const uint32_t groups = M * nkb;   // < 2^31 (checked by the launcher)
  // a half-warp per group, a lane per 16 bytes (8 elements): every load and store of a warp is
  // 512 contiguous bytes of two groups of one row.  A warp's work item is a run of up to
  // 2 * kPhaseDepth groups of one row, all loaded before the first is quantized.
  const uint32_t lane = threadIdx.x & 31u, half = lane >> 4, hl = lane & 15u;
  const uint32_t warps = gridDim.x * (blockDim.x >> 5);
  const uint32_t runs = (nkb + 2u * kPhaseDepth - 1u) / (2u * kPhaseDepth);   // runs per row
  const uint32_t items = M * runs;
  for (uint32_t item = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); item < items; item += warps) {
    const uint32_t m = item / runs, kb0 = (item - m * runs) * (2u * kPhaseDepth) + half;
    const uint16_t* row = xq + (size_t)m * K + hl * 8;
    uint8_t* crow = xq_codes + (size_t)m * K + hl * 8;
    uint4 v[kPhaseDepth];
#pragma unroll
    for (int u = 0; u < kPhaseDepth; ++u) {
      const uint32_t kb = kb0 + 2u * u;
      v[u] = kb < nkb ? ld_stream_v4(row + (size_t)kb * 128) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kPhaseDepth; ++u) {
      const uint32_t kb = kb0 + 2u * u;
      uint32_t mx = absmax_v4(0u, v[u]);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) mx = absmax2(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
      const GroupScale gs = make_group_scale<kE4M3>(packed_amax_to_f32(mx));
      const uint2 q = gs.fast ? quant8_fast<kE4M3>(v[u], gs.d, gs.r) : quant8_nodiv<kE4M3>(v[u], gs.d);
      if (kb < nkb) {
        st_v2(crow + (size_t)kb * 128, q);
        if (hl == 0) sA[(size_t)kb * M + m] = gs.s;
      }
    }
  }
  // the codes and scales written above must be visible to every CTA's TMA loads and scale copies
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __threadfence();
  __syncthreads();
  bool ok = true;
  if (threadIdx.x == 0) {
    uint32_t gen0;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(gen0) : "l"(gbar + 1) : "memory");
    __threadfence();                                   // the generation is read before arriving
    const uint32_t old = atomicAdd(gbar, 1u);
    if (old >= gridDim.x) {
      raise_device_error(err, kErrWorkspaceDirty);     // arrivals left from a call that did not finish
      ok = false;
    } else if (old == gridDim.x - 1) {
      gbar[0] = 0;                                     // the last to arrive resets the count
      __threadfence();
      atomicAdd(gbar + 1, 1u);                         // and releases the others
    } else {
      const uint64_t t0 = globaltimer_ns();
      for (;;) {
        uint32_t gen;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(gen) : "l"(gbar + 1) : "memory");
        if (gen != gen0) break;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          raise_device_error(err, kErrWaitTimeout);
          ok = false;
          break;
        }
        __nanosleep(256);
      }
    }
    __threadfence();
    s_flag_bar = ok ? 1u : 0u;
  }
  __syncthreads();
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return s_flag_bar != 0;
}

__device__ __forceinline__ void tile_coords(int t, const Params& p, int* m0, int* n0) {
  int mt, nt;
  tile_walk(t, p.m_tiles, p.n_tiles, p.group_m, &mt, &nt);
  *m0 = mt * BM;
  *n0 = nt * BN;
}

// QPHASE: the fused linear layer's instantiation, whose first phase quantizes the activations
// (quantize_phase); a separate kernel so the phase's registers do not weigh on the others
template <bool PROMOTE, bool QPHASE = false>
__global__ void __launch_bounds__(kThreads, 1) k_gemm(const __grid_constant__ CUtensorMap tA,
                                                      const __grid_constant__ CUtensorMap tB, Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // scale ring (block-scaled path): slot r holds the 128 row scales of A and the two column-half
  // scales of B for one (tile, K block) pair, written by warp 2 and read by the epilogue
  __shared__ float sc_a[PROMOTE ? kScaleSlots : 1][BM];
  __shared__ float sc_b[PROMOTE ? kScaleSlots : 1][4];
  __shared__ uint64_t sc_full[kScaleSlots], sc_empty[kScaleSlots];
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  uint8_t* sm_a = smem;                                   // kStages x 16 KB
  uint8_t* sm_b = smem + kStages * kStageA;               // kStages x 32 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;                      // [2]
  uint64_t* tempty = tfull + 2;                           // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    for (int r = 0; r < kScaleSlots; ++r) {
      mbar_init(&sc_full[r], 32);            // one arrival per lane of warp 2, on copy completion
      mbar_init(&sc_empty[r], kEpiWarps);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  allow_dependent_launch();
  grid_dependency_wait();
  bool phase_ok = true;
  if constexpr (QPHASE)
    phase_ok = quantize_phase(p.xq, p.xq_codes, const_cast<float*>(p.sA), (uint32_t)p.M, (uint32_t)p.K, p.gbar, p.err);
  const int my_tiles = !phase_ok             ? 0
                       : p.tiles > (int)blockIdx.x ? (p.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                                                   : 0;

  if (warp < kFirstEpiWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && my_tiles > 0) {
      tma_prefetch_desc(&tA);
      if (!p.Bp) tma_prefetch_desc(&tB);
      int s = 0;
      uint32_t ph = 0;
      uint32_t it = 0;
      bool ok = true;
      for (int k = 0; k < my_tiles && ok; ++k) {
        int m0, n0;
        tile_coords((int)blockIdx.x + k * (int)gridDim.x, p, &m0, &n0);
        // packed B: one bulk copy per 128-row half inside N (a half past N is not loaded; its
        // accumulator columns are never stored)
        const int halves = p.Bp ? min(2, (p.N - n0) / 128) : 0;
        const uint8_t* bp = p.Bp ? p.Bp + (size_t)(n0 / 128) * p.num_kb * 16384u : nullptr;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          if (it >= (uint32_t)kStages && !mbar_wait(&empty[s], ph ^ 1u, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], p.Bp ? kStageA + 16384u * halves : kStageBytes);
          tma_load_2d(sm_a + s * kStageA, &tA, kb * BK, m0, &full[s]);
          if (p.Bp) {
            for (int h = 0; h < halves; ++h)
              bulk_load(sm_b + s * kStageB + h * 16384u, bp + ((size_t)h * p.num_kb + kb) * 16384u, 16384u, &full[s]);
          } else {
            tma_load_2d(sm_b + s * kStageB, &tB, kb * BK, n0, &full[s]);
          }
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // drain: every issued copy must land before the CTA may exit
      for (uint32_t j = 0; j < (uint32_t)kStages && j < it; ++j) {
        const uint32_t kk = it - 1 - j;
        mbar_wait(&full[kk % kStages], (kk / kStages) & 1u, p.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && my_tiles > 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t acc_use = 0;       // TMEM buffer uses so far (K blocks when promoting, tiles otherwise)
      bool ok = true;
      for (int k = 0; k < my_tiles && ok; ++k) {
        for (int kb = 0; kb < p.num_kb; ++kb) {
          const bool new_acc = PROMOTE || kb == 0;
          const uint32_t buf = acc_use & 1u;
          if (new_acc && acc_use >= 2) {
            // wait until the epilogue has drained this buffer's previous use
            if (!mbar_wait(&tempty[buf], ((acc_use >> 1) - 1) & 1u, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (!mbar_wait(&full[s], ph, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tmem_d = tmem_base + buf * BN;
          const uint64_t adesc = umma_desc_sw128(smem_u32(sm_a + s * kStageA));
          const uint64_t bdesc = umma_desc_sw128(smem_u32(sm_b + s * kStageB));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint32_t accumulate = (kk > 0 || (!PROMOTE && kb > 0)) ? 1u : 0u;
            umma_f8(tmem_d, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), kIdesc, accumulate);
          }
          umma_commit(&empty[s]);                                    // frees the smem stage
          if (PROMOTE || kb == p.num_kb - 1) {
            umma_commit(&tfull[buf]);                                // partial / tile ready
            ++acc_use;
          }
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // all issued MMAs must complete before TMEM is released
      if (acc_use > 0) mbar_wait(&tfull[(acc_use - 1) & 1u], ((acc_use - 1) >> 1) & 1u, p.err);
    }
  } else if (warp == 2 && PROMOTE) {
    // ------------------------------------------------------------ scale producer
    // For every (tile, K block) pair, lane l copies A's row scales 4l .. 4l+3 of the tile (zero
    // beyond M) and lanes 0-1 B's scales of the two 128-column halves, all with cp.async, then
    // every lane arrives on the slot's barrier once its copies have landed.
    const int nkb = p.num_kb;
    int r = 0;
    uint32_t ph = 0, g = 0;
    bool ok = true;
    for (int k = 0; k < my_tiles && ok; ++k) {
      int m0, n0;
      tile_coords((int)blockIdx.x + k * (int)gridDim.x, p, &m0, &n0);
      for (int kb = 0; kb < nkb; ++kb, ++g) {
        if (g >= (uint32_t)kScaleSlots && !mbar_wait(&sc_empty[r], ph ^ 1u, p.err)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = lane * 4 + i, m = m0 + row;
          const float* src = p.gA_group ? p.sA + (size_t)kb * p.M + (m < p.M ? m : 0) : p.sA;
          const uint32_t nbytes = (p.gA_group && m >= p.M) ? 0u : 4u;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(&sc_a[r][row])), "l"(src),
                       "r"(nbytes)
                       : "memory");
        }
        if (lane < 2) {
          const int ncol0 = n0 + lane * 128;
          const float* src = p.gB_block ? p.sB + (size_t)((ncol0 < p.N ? ncol0 : 0) >> 7) * nkb + kb : p.sB;
          const uint32_t nbytes = (p.gB_block && ncol0 >= p.N) ? 0u : 4u;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(&sc_b[r][lane])), "l"(src),
                       "r"(nbytes)
                       : "memory");
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&sc_full[r]))
                     : "memory");
        if (++r == kScaleSlots) {
          r = 0;
          ph ^= 1u;
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpilogueRegs));
    // ------------------------------------------------------------ promotion / epilogue
    const int ew = warp - kFirstEpiWarp;     // 0..7
    const int quarter = warp & 3;            // TMEM lane quarter this warp may access
    const int half = ew >> 2;                // column half: 128 columns each
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    uint32_t acc_use = 0;
    if (PROMOTE) {
      // Scales come from the ring filled by warp 2: one wait, two shared loads per K block.
      const int nkb = p.num_kb;
      const int total = my_tiles * nkb;
      int r = 0;
      uint32_t sph = 0;
      float2 acc[64];
      int kb = 0, k = 0;
      for (int g = 0; g < total; ++g) {
        if (kb == 0) {
#pragma unroll
          for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
        }
        if (!mbar_wait(&sc_full[r], sph, p.err)) break;
        const float mult = sc_a[r][row_in_tile] * sc_b[r][half];
        const int r_used = r;
        if (++r == kScaleSlots) {
          r = 0;
          sph ^= 1u;
        }
        const float2 mult2 = make_float2(mult, mult);
        const uint32_t buf = acc_use & 1u;
        if (!mbar_wait(&tfull[buf], (acc_use >> 1) & 1u, p.err)) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_addr + buf * BN + half * 128;
#pragma unroll
        for (int c = 0; c < 4; c += 2) {
          uint32_t v[32], w[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_ld32(taddr + c * 32 + 32, w);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            acc[c * 16 + i] =
                __ffma2_rn(mult2, make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), acc[c * 16 + i]);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            acc[c * 16 + 16 + i] = __ffma2_rn(
                mult2, make_float2(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1])), acc[c * 16 + 16 + i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tempty[buf]);          // TMEM buffer drained
          mbar_arrive(&sc_empty[r_used]);     // scale slot read (the loads were consumed above)
        }
        ++acc_use;
        if (++kb == nkb) {
          // tile done: round to bf16 and store this thread's row segment (256 bytes)
          int m0, n0;
          tile_coords((int)blockIdx.x + k * (int)gridDim.x, p, &m0, &n0);
          const int m = m0 + row_in_tile;
          const int ncol0 = n0 + half * 128;
          if (m < p.M && ncol0 < p.N) {
            if (p.q_codes) {
              store_row_e4m3([&](int i) { return f32x2_to_bf16x2(acc[i].x, acc[i].y); },
                             p.q_codes + (size_t)m * p.N + ncol0, p.q_scales + (size_t)(ncol0 >> 7) * p.M + m);
            } else {
              uint16_t* dst = p.C + (size_t)m * p.N + ncol0;
#pragma unroll
              for (int c = 0; c < 8; ++c) {   // 32-byte stores: every store fills whole sectors
                uint4 lo, hi;
                lo.x = f32x2_to_bf16x2(acc[c * 8 + 0].x, acc[c * 8 + 0].y);
                lo.y = f32x2_to_bf16x2(acc[c * 8 + 1].x, acc[c * 8 + 1].y);
                lo.z = f32x2_to_bf16x2(acc[c * 8 + 2].x, acc[c * 8 + 2].y);
                lo.w = f32x2_to_bf16x2(acc[c * 8 + 3].x, acc[c * 8 + 3].y);
                hi.x = f32x2_to_bf16x2(acc[c * 8 + 4].x, acc[c * 8 + 4].y);
                hi.y = f32x2_to_bf16x2(acc[c * 8 + 5].x, acc[c * 8 + 5].y);
                hi.z = f32x2_to_bf16x2(acc[c * 8 + 6].x, acc[c * 8 + 6].y);
                hi.w = f32x2_to_bf16x2(acc[c * 8 + 7].x, acc[c * 8 + 7].y);
                st_stream_v8(dst + c * 16, lo, hi);
              }
            }
          }
          kb = 0;
          ++k;
        }
      }
    } else {
      for (int k = 0; k < my_tiles; ++k) {
        int m0, n0;
        tile_coords((int)blockIdx.x + k * (int)gridDim.x, p, &m0, &n0);
        const int m = m0 + row_in_tile;
        const int ncol0 = n0 + half * 128;
        const uint32_t buf = acc_use & 1u;
        if (!mbar_wait(&tfull[buf], (acc_use >> 1) & 1u, p.err)) break;
        tc_fence_after();
        const float mult = __ldg(p.sA) * __ldg(p.sB);
        const uint32_t taddr = tmem_base + lane_addr + buf * BN + half * 128;
        uint32_t out[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            out[c * 16 + i] = f32x2_to_bf16x2(__fmul_rn(mult, __uint_as_float(v[2 * i])),
                                              __fmul_rn(mult, __uint_as_float(v[2 * i + 1])));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        ++acc_use;
        if (m < p.M && ncol0 < p.N) {
          if (p.q_codes) {
            store_row_e4m3([&](int i) { return out[i]; }, p.q_codes + (size_t)m * p.N + ncol0,
                           p.q_scales + (size_t)(ncol0 >> 7) * p.M + m);
          } else {
            uint16_t* dst = p.C + (size_t)m * p.N + ncol0;
#pragma unroll
            for (int c = 0; c < 8; ++c)   // 32-byte stores: every store fills whole sectors
              st_stream_v8(dst + c * 16, make_uint4(out[c * 8], out[c * 8 + 1], out[c * 8 + 2], out[c * 8 + 3]),
                           make_uint4(out[c * 8 + 4], out[c * 8 + 5], out[c * 8 + 6], out[c * 8 + 7]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + (2 * kStages + 4) * sizeof(uint64_t) + 16;


// ============================================================================ decode shapes
//
// For M <= 64 (decode) the tile walk above would leave most SMs idle and waste the MMA's
// 128-row side on padding.  Here the operands swap roles: the weights' 128-row tile is the
// MMA's M side and the tokens (M rounded up to 16) its N side, so each MMA computes
// P^T[n][m] for 128 weight rows.  The (weight tile, K block) units are split evenly and
// contiguously over all CTAs (a CTA's range may cross tile boundaries); each CTA promotes its
// units per K block (acc[m] += sB[tile][kb] * sA[kb][m] * P^T[n][m], thread = weight row n).
// A tile that lies wholly in one CTA's range is rounded to bf16 and stored directly.  A tile
// shared by several CTAs is finished without any CTA waiting for another, so the result does
// not depend on which CTAs are resident at the same time.  Every later contributor (for which
// the tile is the first segment of its range, done early in its run) writes its fp32 partial to
// the workspace and counts itself in on the tile's counter.  The CTA that started the tile (for
// which it is the last segment) polls that counter while its units stream:
//   - when every later contributor is in by the time its own promotion of the tile ends, its
//     promotion warps add the other partials to their own and store the tile;
//   - otherwise it publishes its partial too and counts itself in, and whichever contributor
//     counts in last (the atomic add that completes the count) sums every partial and stores
//     the tile with its bookkeeping warp.
// Both ways add the partials in ascending CTA order starting from the first contributor's, so
// the output is the same bits whichever CTA finishes.  The finisher resets the tile's counter,
// so every completed call leaves the counters zero; the partial slots are scratch.
//   warp 0 TMA producer, warp 1 MMA issuer (four TMEM buffers), warp 2 scale producer,
//   warps 3-6 promotion, warp 7 split-tile bookkeeping.
namespace dec {

constexpr int BM = 128;                 // weight rows per tile (the MMA's M)
constexpr int kThreads = 32 * 8;
constexpr int kTBuf = 4;                // TMEM buffers of kMaxMp columns
constexpr int kMaxMp = 64;
constexpr uint32_t kTmemCols = kTBuf * kMaxMp;
constexpr int kScaleSlots = 8;
// At 64 tokens the scale warp forms each unit's products RN(sA[m] * sB) once for the CTA (from
// raw scales staged by cp.async kRawLag units ahead) and the promotion only loads them: there the
// promotion's instructions are the bound (70B shapes: 56.6 -> 53.7 us).  With fewer tokens the
// per-thread products are cheaper than the staging, whose per-unit wait then paces the kernel
// (measured slower at 16, 32 and 48 tokens).
constexpr int kProdMinMp = 64;
constexpr int kRawLag = 8;
constexpr uint32_t kStageW = BM * BK;   // 16 KB of weight codes
constexpr int kMaxStages = 10;
// At 16 tokens a CTA fits in half an SM (at most 128 registers a thread, five stages within
// kHalfSmStageBytes), so the next call's CTAs become resident while this call's still run: their
// set-up and L2 prefetch of their first weight tiles overlap this call's tail, and they start
// streaming as soon as the grid dependency resolves (measured about 1 % faster, 8B M=16).  At 32
// tokens the four stages that fit were measured slower (19.0 against 17.3 us), and at 64 the
// promotion's registers (64 accumulators and two 64-column partials) need the whole file.
__host__ __device__ constexpr int ctas_per_sm(int mp) { return mp <= 16 ? 2 : 1; }
constexpr uint32_t kHalfSmStageBytes = 96u * 1024u;
constexpr uint32_t kFullSmStageBytes = 200u * 1024u;

// The workspace: per-tile counters in a fixed region at its start, then the partial slots.  Only
// the counters carry state between calls (zero on entry, reset by every call that completes);
// the slots are scratch, written by each contributor before anyone reads them.  The fixed
// region keeps one call's slots clear of another shape's counters when calls of different
// shapes share a workspace.
constexpr size_t kCounterRegionBytes = 65536;   // 16384 tiles: N <= 2,097,152

struct Params {
  int M, N, K, nkb;
  uint32_t W;         // units: N / 128 tiles x nkb K blocks
  int G;              // CTAs
  int maxseg;         // most tile segments any CTA touches
  const float* sA;
  const float* sB;
  int gA_group, gB_block;
  uint32_t* counters; // [N / 128]: segments counted in per tile; zero between calls (null: none shared)
  float* partials;    // [G][maxseg][Mp][128], scratch
  uint16_t* C;
  int stages;
  uint32_t stage_bytes;
  const uint8_t* Bp;  // packed weight tiles (tile t, K block kb at t * nkb + kb), or null: TMA
  uint32_t* err;
};

// first unit of CTA c when W units are split over G CTAs (W * G < 2^32, checked by the planner)
__host__ __device__ __forceinline__ uint32_t range_lo(uint32_t c, uint32_t W, uint32_t G) { return (c * W) / G; }

// A range's first segment adds to a tile that a lower CTA started when the range does not begin
// on a tile boundary; its last segment starts a tile that a higher CTA ends when the range holds
// that tile's first unit but not its last.  (The split-tile hand-off relies on these being the
// only shared segments of a range; fp8q_check_decode_split verifies it.)
__host__ __device__ __forceinline__ bool first_seg_adds_to_lower(uint32_t lo, uint32_t nkb) { return lo % nkb != 0; }
__host__ __device__ __forceinline__ bool last_seg_finishes_shared(uint32_t lo, uint32_t hi, uint32_t nkb) {
  return (lo <= ((hi - 1) / nkb) * nkb) && hi % nkb != 0;
}

// CTAs for `tiles` weight tiles of nkb units on `sms` SMs.  When whole tiles keep at least three
// quarters of the SMs busy, each CTA takes exactly one tile and no tile is shared (the split-tile
// hand-off measured 3.8 us of a 16.5 us call at the 8B shape, 112 tiles); otherwise the units are
// spread evenly over all SMs, ranges crossing tile boundaries.
__host__ __device__ __forceinline__ uint32_t decode_ctas(uint32_t tiles, uint32_t nkb, uint32_t sms) {
  if (tiles <= sms && 4u * tiles >= 3u * sms) return tiles;
  const uint32_t W = tiles * nkb;
  return W < sms ? W : sms;
}

// the CTA whose range holds unit u
__host__ __device__ __forceinline__ uint32_t cta_of(uint32_t u, uint32_t W, uint32_t G) {
  uint32_t c = (u * G) / W;
  while (c > 0 && range_lo(c, W, G) > u) --c;
  while (c + 1 < G && range_lo(c + 1, W, G) <= u) ++c;
  return c;
}

// The bookkeeping warp's decision (s_fin) for the tile a CTA started and a higher CTA ends.
constexpr uint32_t kFinSkip = 0;      // nothing more here: a workspace error, or another CTA finishes
constexpr uint32_t kFinHere = 1;      // every later contributor is in: the promotion warps finish it
constexpr uint32_t kFinPublish = 2;   // publish this CTA's partial and count it in
// how long the starting CTA keeps polling once its own part of the tile is done, before it
// publishes its partial instead (a bounded optimisation, not a dependency)
constexpr uint64_t kFinGraceNs = 3000;

// CTA c's partial of tile t: [MP][128] fp32, rows contiguous (slot t - c's first tile of c's maxseg)
__device__ __forceinline__ float* partial_slot(const Params& p, int mp, uint32_t c, uint32_t t) {
  const uint32_t t_first = range_lo(c, p.W, p.G) / (uint32_t)p.nkb;
  return p.partials + ((size_t)(c * (uint32_t)p.maxseg + (t - t_first)) * mp) * BM;
}

// One warp finishes tile t once every contributor c_first..c_last has published its partial:
// lane l owns rows 4l..4l+3; the partials are added in ascending CTA order starting from
// c_first's (the order the promotion warps use when c_first finishes the tile itself), rounded
// to bf16 and stored; then the tile's counter is reset (the partial slots are scratch).
template <int MP>
__device__ __forceinline__ void finish_tile_warp(const Params& p, uint32_t t, uint32_t c_first, uint32_t c_last,
                                              int lane) {
  constexpr int kChunk = ctas_per_sm(MP) == 2 ? 4 : 16;   // float4 registers: 8 kChunk
  const int r0 = lane * 4;
  for (int m0 = 0; m0 < MP; m0 += kChunk) {
    float4 sum[kChunk];
    const float* first = partial_slot(p, MP, c_first, t) + (size_t)m0 * BM + r0;
#pragma unroll
    for (int j = 0; j < kChunk; ++j) sum[j] = __ldcg(reinterpret_cast<const float4*>(first + (size_t)j * BM));
#pragma unroll 1
    for (uint32_t c = c_first + 1; c <= c_last; ++c) {
      const float* src = partial_slot(p, MP, c, t) + (size_t)m0 * BM + r0;
      float4 part[kChunk];
#pragma unroll
      for (int j = 0; j < kChunk; ++j) part[j] = __ldcg(reinterpret_cast<const float4*>(src + (size_t)j * BM));
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        sum[j].x += part[j].x;
        sum[j].y += part[j].y;
        sum[j].z += part[j].z;
        sum[j].w += part[j].w;
      }
    }
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      const int m = m0 + j;
      if (m < p.M) {
        const uint2 v = make_uint2(f32x2_to_bf16x2(sum[j].x, sum[j].y), f32x2_to_bf16x2(sum[j].z, sum[j].w));
        *reinterpret_cast<uint2*>(p.C + (size_t)m * p.N + (size_t)t * BM + r0) = v;
      }
    }
  }
  __syncwarp();
  if (lane == 0) p.counters[t] = 0;
}

template <int MP>
__global__ void __launch_bounds__(kThreads, ctas_per_sm(MP)) k_decode_mma(const __grid_constant__ CUtensorMap tW,
                                                             const __grid_constant__ CUtensorMap tX, Params p) {
  constexpr uint32_t kIdescD = (1u << 4) | ((uint32_t)(MP >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  constexpr bool kProd = MP >= kProdMinMp;
  __shared__ __align__(16) float sc_a[kScaleSlots][MP];   // sA[m], or RN(sA[m] * sB) when kProd
  __shared__ float sc_b[kScaleSlots];
  __shared__ __align__(16) float raw_a[kProd ? kRawLag + 1 : 1][MP];
  __shared__ float raw_b[kProd ? kRawLag + 1 : 1][32];
  __shared__ uint64_t bars[2 * kMaxStages + 2 * kTBuf + 2 * kScaleSlots + 4];
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t s_fin;   // the bookkeeping warp's decision for the tile this CTA started
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  const int S = p.stages;
  uint64_t* full = bars;
  uint64_t* empty = bars + kMaxStages;
  uint64_t* tfull = bars + 2 * kMaxStages;
  uint64_t* tempty = tfull + kTBuf;
  uint64_t* sfull = tempty + kTBuf;
  uint64_t* sempty = sfull + kScaleSlots;
  uint64_t* seg_written = sempty + kScaleSlots;   // first segment: the promotion warps' partials are out
  uint64_t* at_end = seg_written + 1;             // last segment: the promotion warps have its partial
  uint64_t* fin_ready = at_end + 1;               // last segment: s_fin is set
  uint64_t* seg_pub = fin_ready + 1;              // last segment: its partial is published
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lo = range_lo(blockIdx.x, p.W, p.G), hi = range_lo(blockIdx.x + 1, p.W, p.G);
  const uint32_t n_units = hi - lo;
  const int nkb = p.nkb;
  if (warp == 2 && lane == 0 && n_units > 0) {
    // the weights are read once: start their first tiles towards L2 before waiting on the
    // previous grid (a prefetch only warms L2, which stays coherent with any later write); the
    // scale warp is idle until then, so thread 0's barrier set-up does not wait behind it
    if (!p.Bp) tma_prefetch_desc(&tW);
    tma_prefetch_desc(&tX);
    for (uint32_t i = 0; i < n_units && i < (uint32_t)S; ++i) {
      const uint32_t u = lo + i, t = u / nkb;
      if (p.Bp)
        bulk_prefetch_l2(p.Bp + (size_t)u * kStageW, kStageW);
      else
        tma_prefetch_l2_2d(&tW, (int32_t)((u - t * nkb) * BK), (int32_t)(t * BM));
    }
  }
  if (threadIdx.x == 0) {
    mbar_init(seg_written, 4);
    mbar_init(at_end, 4);
    mbar_init(fin_ready, 1);
    mbar_init(seg_pub, 4);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < kTBuf; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    for (int r = 0; r < kScaleSlots; ++r) {
      mbar_init(&sfull[r], 32);
      mbar_init(&sempty[r], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  allow_dependent_launch();
  grid_dependency_wait();

  if (warp == 0) {
    if (lane == 0 && n_units > 0) {
      int s = 0;
      uint32_t ph = 0, i = 0;
      for (; i < n_units; ++i) {
        const uint32_t u = lo + i, t = u / nkb, kb = u - t * nkb;
        if (i >= (uint32_t)S && !mbar_wait(&empty[s], ph ^ 1u, p.err)) break;
        uint8_t* st = smem + s * p.stage_bytes;
        mbar_arrive_expect_tx(&full[s], p.stage_bytes);
        if (p.Bp)
          bulk_load(st, p.Bp + (size_t)u * kStageW, kStageW, &full[s]);   // unit u = tile t, K block kb
        else
          tma_load_2d(st, &tW, (int32_t)(kb * BK), (int32_t)(t * BM), &full[s]);
        tma_load_2d(st + kStageW, &tX, (int32_t)(kb * BK), 0, &full[s]);
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
      for (uint32_t j = 0; j < (uint32_t)S && j < i; ++j) {
        const uint32_t kk = i - 1 - j;
        mbar_wait(&full[kk % S], (kk / S) & 1u, p.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n_units > 0) {
      int s = 0;
      uint32_t ph = 0, i = 0;
      for (; i < n_units; ++i) {
        const uint32_t buf = i % kTBuf;
        if (i >= (uint32_t)kTBuf) {
          if (!mbar_wait(&tempty[buf], ((i / kTBuf) - 1) & 1u, p.err)) break;
          tc_fence_after();
        }
        if (!mbar_wait(&full[s], ph, p.err)) break;
        tc_fence_after();
        const uint8_t* st = smem + s * p.stage_bytes;
        const uint64_t adesc = umma_desc_sw128(smem_u32(st));
        const uint64_t bdesc = umma_desc_sw128(smem_u32(st + kStageW));
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk)
          umma_f8(tmem_base + buf * kMaxMp, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), kIdescD,
                  kk > 0 ? 1u : 0u);
        umma_commit(&empty[s]);
        umma_commit(&tfull[buf]);
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (i > 0) mbar_wait(&tfull[(i - 1) % kTBuf], ((i - 1) / kTBuf) & 1u, p.err);
    }
  } else if (warp == 2) {
    if constexpr (kProd) {
      // scale producer, product form: each unit's activation scales (zero beyond M) and weight
      // scale are copied with cp.async into a staging ring; kRawLag units later, when they have
      // landed, each lane forms the products RN(sA[m] * sB) of its two tokens once for the CTA
      // (the roundings the promotion would make) and publishes them in the ring
      uint32_t r = 0, ph = 0;
      const int m0 = lane * 2;
      for (uint32_t i = 0; i < n_units + kRawLag; ++i) {
        if (i < n_units) {
          const uint32_t u = lo + i, t = u / nkb, kb = u - t * nkb, rs = i % (kRawLag + 1);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int m = m0 + h;
            if (m < MP) {
              const float* src = p.gA_group ? p.sA + (size_t)kb * p.M + (m < p.M ? m : 0) : p.sA;
              const uint32_t nbytes = (p.gA_group && m >= p.M) ? 0u : 4u;
              asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(&raw_a[rs][m])), "l"(src),
                           "r"(nbytes)
                           : "memory");
            }
          }
          const float* srcb = p.gB_block ? p.sB + (size_t)t * nkb + kb : p.sB;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(&raw_b[rs][lane])), "l"(srcb)
                       : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (i < (uint32_t)kRawLag) continue;
        // this lane's copies for unit j have landed once at most kRawLag later groups are pending
        const uint32_t j = i - kRawLag, rs = j % (kRawLag + 1);
        asm volatile("cp.async.wait_group %0;" ::"n"(kRawLag) : "memory");
        if (j >= (uint32_t)kScaleSlots && !mbar_wait(&sempty[r], ph ^ 1u, p.err)) break;
        if (m0 < MP) {
          const float sb = raw_b[rs][lane];
          const float2 c = __fmul2_rn(make_float2(raw_a[rs][m0], raw_a[rs][m0 + 1]), make_float2(sb, sb));
          *reinterpret_cast<float2*>(&sc_a[r][m0]) = c;
        }
        mbar_arrive(&sfull[r]);   // release: this lane's products
        if (++r == kScaleSlots) {
          r = 0;
          ph ^= 1u;
        }
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
      // scale producer: the K block's activation scales (one per token, zero beyond M) and the
      // tile's weight scale, copied with cp.async into a ring slot
      uint32_t r = 0, ph = 0;
      for (uint32_t i = 0; i < n_units; ++i) {
        const uint32_t u = lo + i, t = u / nkb, kb = u - t * nkb;
        if (i >= (uint32_t)kScaleSlots && !mbar_wait(&sempty[r], ph ^ 1u, p.err)) break;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int m = lane * 2 + h;
          if (m < MP) {
            const float* src = p.gA_group ? p.sA + (size_t)kb * p.M + (m < p.M ? m : 0) : p.sA;
            const uint32_t nbytes = (p.gA_group && m >= p.M) ? 0u : 4u;
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(&sc_a[r][m])), "l"(src),
                         "r"(nbytes)
                         : "memory");
          }
        }
        if (lane == 0) {
          const float* src = p.gB_block ? p.sB + (size_t)t * nkb + kb : p.sB;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(&sc_b[r])), "l"(src) : "memory");
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&sfull[r])) : "memory");
        if (++r == kScaleSlots) {
          r = 0;
          ph ^= 1u;
        }
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
  } else if (warp == 7) {
    // split-tile bookkeeping.  A CTA's range holds at most one segment of a tile a lower CTA
    // started (its first: the partial is counted in here) and at most one segment of a tile it
    // starts but a higher CTA ends (its last: the decision below).  No step waits for another CTA.
    if (n_units > 0) {
      const uint32_t t0 = lo / nkb, t1 = (hi - 1) / nkb;
      if (first_seg_adds_to_lower(lo, nkb)) {
        const uint32_t c_first = cta_of(t0 * nkb, p.W, p.G), c_last = cta_of(t0 * nkb + nkb - 1, p.W, p.G);
        uint32_t last = 0;
        // the promotion warps hand their partial writes over through the mbarrier (release /
        // acquire at CTA scope); this gpu-scope fence then orders all of them (cumulatively)
        // before the count
        if (lane == 0 && mbar_wait(seg_written, 0, p.err)) {
          __threadfence();
          const uint32_t old = atomicAdd(p.counters + t0, 1u);
          if (old > c_last - c_first) {
            // a workspace that was not zero: report it and mark the counter (its top bit stays
            // set however the other adds interleave), so no contributor takes it for complete
            raise_device_error(p.err, kErrWorkspaceDirty);
            atomicOr(p.counters + t0, 0x80000000u);
          } else {
            last = old == c_last - c_first;   // every other contributor, the starter included, is in
          }
        }
        if (__shfl_sync(0xffffffffu, last, 0)) {
          __threadfence();
          finish_tile_warp<MP>(p, t0, c_first, c_last, lane);
        }
      }
      if (last_seg_finishes_shared(lo, hi, nkb)) {
        const uint32_t c_last = cta_of(t1 * nkb + nkb - 1, p.W, p.G);
        const uint32_t need = c_last - blockIdx.x;   // later contributors
        uint32_t dec = kFinSkip;
        if (lane == 0) {
          // polled while this CTA's units stream (the later contributors count in early in their
          // runs); the poll ends when they are all in, or kFinGraceNs after this CTA's own
          // promotion of the tile is done, whichever comes first.  The grace only saves the
          // publish-and-reduce round trips when a contributor is about to count in (a middle CTA
          // ends its run when this one does); nothing depends on another CTA being resident.
          const uint64_t t_start = globaltimer_ns();
          uint64_t t_end = 0;
          for (;;) {
            uint32_t v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p.counters + t1) : "memory");
            if (v == need) {
              p.counters[t1] = 0;   // nobody else touches it in this call: leave it zero
              dec = kFinHere;
              break;
            }
            if (v > need) {
              raise_device_error(p.err, kErrWorkspaceDirty);
              break;
            }
            if (t_end == 0 && mbar_test(at_end, 0)) t_end = globaltimer_ns();
            if (t_end != 0 && globaltimer_ns() - t_end > kFinGraceNs) {
              dec = kFinPublish;
              break;
            }
            if (globaltimer_ns() - t_start > kWaitLimitNs) {
              raise_device_error(p.err, kErrWaitTimeout);
              break;
            }
            __nanosleep(128);
          }
          s_fin = dec;
          mbar_arrive(fin_ready);
        }
        if (__shfl_sync(0xffffffffu, dec, 0) == kFinPublish) {
          uint32_t last = 0;
          if (lane == 0 && mbar_wait(seg_pub, 0, p.err)) {
            __threadfence();
            const uint32_t old = atomicAdd(p.counters + t1, 1u);
            if (old > need) {
              raise_device_error(p.err, kErrWorkspaceDirty);
              atomicOr(p.counters + t1, 0x80000000u);
            } else {
              last = old == need;   // the later contributors came in meanwhile
            }
          }
          if (__shfl_sync(0xffffffffu, last, 0)) {
            __threadfence();
            finish_tile_warp<MP>(p, t1, blockIdx.x, c_last, lane);
          }
        }
      }
    }
  } else {
    // promotion: thread = weight row (TMEM lane) of the tile, MP accumulators (one per token)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    float acc[MP];
#pragma unroll
    for (int m = 0; m < MP; ++m) acc[m] = 0.0f;
    uint32_t r = 0, sph = 0;
    const uint32_t first_tile = lo / nkb;
    // Units are taken in pairs when the next unit belongs to the same tile: one round of waits,
    // both partials loaded before one tcgen05.wait, applied in unit order (the same fp32 sums as
    // one at a time), both buffers and scale slots released together.
    auto ld_partial = [&](uint32_t buf, uint32_t (&v)[MP]) {
#pragma unroll
      for (int c = 0; c < MP / 16; ++c) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15}, [%16];"
            : "=r"(v[c * 16 + 0]), "=r"(v[c * 16 + 1]), "=r"(v[c * 16 + 2]), "=r"(v[c * 16 + 3]),
              "=r"(v[c * 16 + 4]), "=r"(v[c * 16 + 5]), "=r"(v[c * 16 + 6]), "=r"(v[c * 16 + 7]),
              "=r"(v[c * 16 + 8]), "=r"(v[c * 16 + 9]), "=r"(v[c * 16 + 10]), "=r"(v[c * 16 + 11]),
              "=r"(v[c * 16 + 12]), "=r"(v[c * 16 + 13]), "=r"(v[c * 16 + 14]), "=r"(v[c * 16 + 15])
            : "r"(tmem_base + lane_addr + buf * kMaxMp + c * 16));
      }
    };
    for (uint32_t i = 0; i < n_units;) {
      const uint32_t u0 = lo + i, t = u0 / nkb;
      const bool pair = i + 1 < n_units && (u0 + 1) % nkb != 0;   // unit i + 1 is in tile t too
      const uint32_t buf0 = i % kTBuf, buf1 = (i + 1) % kTBuf;
      const uint32_t r0 = r, ph0 = sph;
      const uint32_t r1 = r0 + 1 == (uint32_t)kScaleSlots ? 0u : r0 + 1;
      const uint32_t ph1 = r0 + 1 == (uint32_t)kScaleSlots ? sph ^ 1u : sph;
      if (!mbar_wait(&sfull[r0], ph0, p.err)) break;
      if (!mbar_wait(&tfull[buf0], (i / kTBuf) & 1u, p.err)) break;
      if (pair && !mbar_wait(&sfull[r1], ph1, p.err)) break;
      if (pair && !mbar_wait(&tfull[buf1], ((i + 1) / kTBuf) & 1u, p.err)) break;
      tc_fence_after();
      uint32_t v0[MP], v1[MP];
      ld_partial(buf0, v0);
      if (pair) ld_partial(buf1, v1);
      tmem_ld_wait();
      // acc[m] += RN(sA[m] * sB) * P[m] on packed pairs (two independent roundings each: the
      // same values as one element at a time)
      auto promote = [&](uint32_t rs, const uint32_t (&v)[MP]) {
        const float sb = kProd ? 1.0f : sc_b[rs];
        const float2 sb2 = make_float2(sb, sb);
#pragma unroll
        for (int m = 0; m < MP; m += 4) {
          const float4 a4 = *reinterpret_cast<const float4*>(&sc_a[rs][m]);
          const float2 c01 = kProd ? make_float2(a4.x, a4.y) : __fmul2_rn(make_float2(a4.x, a4.y), sb2);
          const float2 c23 = kProd ? make_float2(a4.z, a4.w) : __fmul2_rn(make_float2(a4.z, a4.w), sb2);
          const float2 s01 = __ffma2_rn(c01, make_float2(__uint_as_float(v[m]), __uint_as_float(v[m + 1])),
                                        make_float2(acc[m], acc[m + 1]));
          const float2 s23 = __ffma2_rn(c23, make_float2(__uint_as_float(v[m + 2]), __uint_as_float(v[m + 3])),
                                        make_float2(acc[m + 2], acc[m + 3]));
          acc[m] = s01.x;
          acc[m + 1] = s01.y;
          acc[m + 2] = s23.x;
          acc[m + 3] = s23.y;
        }
      };
      promote(r0, v0);
      if (pair) promote(r1, v1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[buf0]);
        mbar_arrive(&sempty[r0]);
        if (pair) {
          mbar_arrive(&tempty[buf1]);
          mbar_arrive(&sempty[r1]);
        }
      }
      const uint32_t used = pair ? 2u : 1u;
      r += used;
      if (r >= (uint32_t)kScaleSlots) {
        r -= kScaleSlots;
        sph ^= 1u;
      }
      i += used;
      const uint32_t u = u0 + used - 1;   // the last unit taken
      if (u + 1 == hi || (u + 1) % nkb == 0) {
        // this CTA's segment of tile t ends
        const uint32_t c_first = cta_of(t * nkb, p.W, p.G), c_last = cta_of(t * nkb + nkb - 1, p.W, p.G);
        bool finish = c_first == c_last;   // the whole tile is this CTA's
        if (!finish && blockIdx.x != c_first) {
          // a lower CTA started the tile: publish this row's partial ([m][row] layout, coalesced
          // over rows) and hand it to the reducer warp, which counts it in; nothing to wait for
          float* dst = p.partials + ((size_t)(blockIdx.x * p.maxseg + (t - first_tile)) * MP) * BM + row;
#pragma unroll
          for (int m = 0; m < MP; ++m) dst[(size_t)m * BM] = acc[m];
          __syncwarp();
          if (lane == 0) mbar_arrive(seg_written);
        } else if (!finish) {
          // this CTA started the tile and a higher one ends it (always this CTA's last segment):
          // the bookkeeping warp decides, without waiting for the other CTAs, whether they are
          // all in.  If so, add their partials to this row in ascending CTA order (the order the
          // bookkeeping warp of whichever CTA finishes uses too); if not, publish
          // this row's partial for the CTA that counts in last.
          __syncwarp();
          if (lane == 0) mbar_arrive(at_end);
          if (!mbar_wait(fin_ready, 0, p.err)) break;
          const uint32_t dec = s_fin;
          finish = dec == kFinHere;
          if (dec == kFinPublish) {
            float* dst = p.partials + ((size_t)(blockIdx.x * p.maxseg + (t - first_tile)) * MP) * BM + row;
#pragma unroll
            for (int m = 0; m < MP; ++m) dst[(size_t)m * BM] = acc[m];
            __syncwarp();
            if (lane == 0) mbar_arrive(seg_pub);
          }
          if (finish) {
            __threadfence();
#pragma unroll 1
            for (uint32_t c = c_first + 1; c <= c_last; ++c) {
              const uint32_t clo = range_lo(c, p.W, p.G);
              float* src = p.partials + ((size_t)(c * (uint32_t)p.maxseg + (t - clo / nkb)) * MP) * BM + row;
#pragma unroll
              for (int m0 = 0; m0 < MP; m0 += 16) {
                float part[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) part[j] = __ldcg(src + (size_t)(m0 + j) * BM);
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[m0 + j] += part[j];
              }
            }
          }
        }
        if (finish) {
          uint16_t* out = p.C + (size_t)t * BM + row;
          const size_t ldc = (size_t)p.N;
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            if (m < p.M) *out = (uint16_t)(f32x2_to_bf16x2(acc[m], 0.0f) & 0xFFFFu);
            out += ldc;
          }
        }
#pragma unroll
        for (int m = 0; m < MP; ++m) acc[m] = 0.0f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace dec
}  // namespace gemm

namespace {

// decode plan: CTAs, segments per CTA and workspace bytes for M <= 64
struct DecodePlan {
  int mp = 0, G = 0, maxseg = 0;
  uint32_t W = 0;
  size_t ws_bytes = 0, counter_bytes = 0;
};

DecodePlan decode_plan_uncached(int64_t M, int64_t N, int64_t K) {
  DecodePlan d;
  if (M <= 0 || M > gemm::dec::kMaxMp || N % 128 != 0 || K % 128 != 0 || N == 0 || K == 0) return d;
  d.mp = (int)((M + 15) / 16 * 16);
  const int64_t nkb = K / 128, tiles = N / 128;
  if ((uint64_t)tiles * nkb * (uint64_t)std::max(1, device_sm_count()) >= (1ull << 32) ||
      tiles > (int64_t)(gemm::dec::kCounterRegionBytes / sizeof(uint32_t))) {
    d.mp = 0;   // not a decode shape: the prefill kernel takes it
    return d;
  }
  d.W = (uint32_t)(tiles * nkb);
  d.G = (int)gemm::dec::decode_ctas((uint32_t)tiles, (uint32_t)nkb, (uint32_t)std::max(1, device_sm_count()));
  for (int c = 0; c < d.G; ++c) {
    const uint32_t lo = gemm::dec::range_lo(c, d.W, d.G), hi = gemm::dec::range_lo(c + 1, d.W, d.G);
    if (hi > lo) d.maxseg = std::max<int>(d.maxseg, (int)((hi - 1) / nkb - lo / nkb + 1));
  }
  if ((uint64_t)d.G * nkb == d.W) return d;   // one whole tile per CTA: nothing shared, no workspace
  d.counter_bytes = gemm::dec::kCounterRegionBytes;
  d.ws_bytes = d.counter_bytes + (size_t)d.G * d.maxseg * d.mp * gemm::dec::BM * sizeof(float);
  return d;
}

// The plan walks every CTA's range; a decode step asks for the same few shapes on every call
// (once for the workspace size, once to launch), so the last plan is kept per host thread.
DecodePlan decode_plan(int64_t M, int64_t N, int64_t K) {
  struct Entry {
    int64_t M = -1, N = -1, K = -1;
    int sms = -1;
    DecodePlan plan;
  };
  thread_local Entry last;
  const int sms = device_sm_count();
  if (last.M != M || last.N != N || last.K != K || last.sms != sms) {
    last.plan = decode_plan_uncached(M, N, K);
    last.M = M;
    last.N = N;
    last.K = K;
    last.sms = sms;
  }
  return last.plan;
}

template <int MP>
cudaError_t launch_decode(const CUtensorMap& mW, const CUtensorMap& mX, gemm::dec::Params& p, cudaStream_t st) {
  using namespace gemm::dec;
  const size_t smem = 1024 + (size_t)p.stages * p.stage_bytes;
  const cudaError_t ea = ensure_dynamic_smem((const void*)k_decode_mma<MP>, smem);
  if (ea != cudaSuccess) return ea;
  // a programmatic dependent of what precedes it on the stream: its set-up (and the L2 prefetch
  // of the first weight tiles) overlaps that grid's tail; griddepcontrol.wait orders every
  // load and store of operands, scales, workspace and output after it
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_decode_mma<MP>, mW, mX, p);
}

cudaError_t launch_decode_gemm(const DecodePlan& plan, const uint8_t* A, const float* sA, int gA, const uint8_t* B,
                               bool b_packed, const float* sB, int gB, int64_t M, int64_t N, int64_t K, uint16_t* C,
                               void* ws, size_t ws_bytes, cudaStream_t st) {
  using namespace gemm::dec;
  using gemm::BK;
  if (plan.ws_bytes > 0 && (!ws || ws_bytes < plan.ws_bytes)) return cudaErrorInvalidValue;
  CUtensorMap mW, mX;
  std::memset(&mW, 0, sizeof(mW));
  std::memset(&mX, 0, sizeof(mX));
  if (!b_packed && !make_tmap_2d(&mW, 1, B, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BM, 1))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&mX, 1, A, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, (uint32_t)plan.mp, 1))
    return cudaErrorInvalidValue;
  gemm::dec::Params d;
  d.M = (int)M;
  d.N = (int)N;
  d.K = (int)K;
  d.nkb = (int)(K / BK);
  d.W = plan.W;
  d.G = plan.G;
  d.maxseg = plan.maxseg;
  d.sA = sA;
  d.sB = sB;
  d.gA_group = gA == 1;
  d.gB_block = gB == 2;
  d.counters = plan.ws_bytes > 0 ? static_cast<uint32_t*>(ws) : nullptr;
  d.partials = plan.ws_bytes > 0 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + plan.counter_bytes) : nullptr;
  d.C = C;
  d.stage_bytes = kStageW + (uint32_t)plan.mp * BK;
  // half-SM CTAs only when every SM has one: with one whole tile per CTA on fewer CTAs than SMs
  // the scheduler could put two on one SM, so those take a full SM's stages
  const bool whole_tiles = (uint32_t)plan.G * (uint32_t)(K / BK) == plan.W;
  const uint32_t budget = (ctas_per_sm(plan.mp) == 2 && !whole_tiles) ? kHalfSmStageBytes : kFullSmStageBytes;
  d.stages = (int)std::max<uint32_t>(2, std::min<uint32_t>(kMaxStages, budget / d.stage_bytes));
  d.Bp = b_packed ? B : nullptr;
  d.err = device_error_word();
  switch (plan.mp) {
    case 16: return launch_decode<16>(mW, mX, d, st);
    case 32: return launch_decode<32>(mW, mX, d, st);
    case 48: return launch_decode<48>(mW, mX, d, st);
    default: return launch_decode<64>(mW, mX, d, st);
  }
}

}  // namespace

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) { return decode_plan(M, N, K).ws_bytes; }

// The invariants of the decode kernel's split-tile hand-off, checked on the host with the
// kernel's own range functions (see fp8q_check_decode_split in fp8q.h for the list).
int check_decode_split(int64_t M, int64_t N, int64_t K, int sms) {
  using gemm::dec::cta_of;
  using gemm::dec::range_lo;
  if (M <= 0 || M > gemm::dec::kMaxMp || N <= 0 || K <= 0 || N % 128 != 0 || K % 128 != 0 || sms <= 0) return -1;
  if (N / 128 > (int64_t)(gemm::dec::kCounterRegionBytes / sizeof(uint32_t))) return -1;
  const uint32_t nkb = (uint32_t)(K / 128), tiles = (uint32_t)(N / 128);
  if ((uint64_t)tiles * nkb * (uint64_t)sms >= (1ull << 32)) return -1;
  const uint32_t W = tiles * nkb, G = gemm::dec::decode_ctas(tiles, nkb, (uint32_t)sms);
  int maxseg = 0;
  for (uint32_t c = 0; c < G; ++c) {
    const uint32_t lo = range_lo(c, W, G), hi = range_lo(c + 1, W, G);
    if (hi <= lo) return 1;                                   // every CTA has work
    maxseg = std::max<int>(maxseg, (int)((hi - 1) / nkb - lo / nkb + 1));
  }
  std::vector<uint32_t> later(tiles, 0), finishers(tiles, 0);
  for (uint32_t c = 0; c < G; ++c) {
    const uint32_t lo = range_lo(c, W, G), hi = range_lo(c + 1, W, G);
    const uint32_t t0 = lo / nkb, t1 = (hi - 1) / nkb;
    // the bookkeeping warp's view
    const bool red_later = gemm::dec::first_seg_adds_to_lower(lo, nkb);
    const bool red_fin = gemm::dec::last_seg_finishes_shared(lo, hi, nkb);
    // the promotion warps' view, segment by segment
    int n_later = 0, n_fin = 0;
    for (uint32_t t = t0; t <= t1; ++t) {
      const uint32_t c_first = cta_of(t * nkb, W, G), c_last = cta_of(t * nkb + nkb - 1, W, G);
      if (c_first > c || c_last < c) return 2;                // the range functions disagree
      if (c_first == c_last) continue;                        // whole tile: stored directly
      if (c != c_first) {
        ++n_later;
        if (t != t0 || !red_later) return 3;                  // only the first segment, seen by both
        if ((int)(t - t0) >= maxseg) return 4;                // its partial slot is in the workspace
        ++later[t];
      } else {
        ++n_fin;
        if (t != t1 || !red_fin) return 5;                    // only the last segment, seen by both
        if ((int)(t - t0) >= maxseg) return 4;                // the slot it may publish into exists
        ++finishers[t];
      }
    }
    if (n_later > 1 || n_fin > 1) return 6;
    if ((n_later == 1) != red_later || (n_fin == 1) != red_fin) return 7;
  }
  for (uint32_t t = 0; t < tiles; ++t) {
    const uint32_t c_first = cta_of(t * nkb, W, G), c_last = cta_of(t * nkb + nkb - 1, W, G);
    if (c_first == c_last) {
      if (later[t] != 0 || finishers[t] != 0) return 8;
    } else if (finishers[t] != 1 || later[t] != c_last - c_first) {
      return 9;                                               // one finisher, every other contributor counted once
    }
  }
  return 0;
}

// The prefill kernels' tile walk, checked on the host with the kernels' own functions: every tile
// of the M x N output visited once, every coordinate inside the matrix.
int check_tile_walk(int64_t M, int64_t N, int64_t K) {
  using namespace gemm;
  if (M <= 64 || N <= 0 || K <= 0 || N % 128 != 0 || K % 128 != 0) return -1;
  const int64_t m_tiles = (M + BM - 1) / BM, n_tiles = (N + BN - 1) / BN;
  if (m_tiles * n_tiles > (int64_t(1) << 26)) return -1;
  const int group_m = tile_group_m(M, K, (int)m_tiles);
  if (group_m < 1 || group_m > m_tiles) return 1;
  std::vector<uint8_t> seen((size_t)(m_tiles * n_tiles), 0);
  for (int t = 0; t < (int)(m_tiles * n_tiles); ++t) {
    int mt, nt;
    tile_walk(t, (int)m_tiles, (int)n_tiles, group_m, &mt, &nt);
    if (mt < 0 || mt >= m_tiles || nt < 0 || nt >= n_tiles) return 2;   // outside the matrix
    uint8_t& v = seen[(size_t)nt * m_tiles + mt];
    if (v) return 3;                                                      // visited twice
    v = 1;
  }
  return 0;   // tiles visited = tiles in the matrix, none twice: each exactly once
}

// the prefill kernel (M > 64): C in bf16, or (q_codes non-null) quantized to E4M3 1x128 groups
static cudaError_t launch_prefill(const uint8_t* A, const float* sA, int gA, const uint8_t* B, bool b_packed,
                                  const float* sB, int gB, int64_t M, int64_t N, int64_t K, uint16_t* C,
                                  uint8_t* q_codes, float* q_scales, cudaStream_t st) {
  using namespace gemm;
  CUtensorMap mA, mB;
  std::memset(&mA, 0, sizeof(mA));
  std::memset(&mB, 0, sizeof(mB));
  if (!make_tmap_2d(&mA, 1, A, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM, 1)) return cudaErrorInvalidValue;
  if (!b_packed && !make_tmap_2d(&mB, 1, B, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BN, 1))
    return cudaErrorInvalidValue;
  Params p{};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.num_kb = (int)(K / BK);
  p.m_tiles = (int)((M + BM - 1) / BM);
  p.n_tiles = (int)((N + BN - 1) / BN);
  p.tiles = p.m_tiles * p.n_tiles;
  p.group_m = tile_group_m(M, K, p.m_tiles);
  p.sA = sA;
  p.sB = sB;
  p.gA_group = gA == 1;
  p.gB_block = gB == 2;
  p.Bp = b_packed ? B : nullptr;
  p.C = C;
  p.q_codes = q_codes;
  p.q_scales = q_scales;
  p.err = device_error_word();
  const bool promote = p.gA_group || p.gB_block;
  const int grid = std::max(1, std::min(p.tiles, device_sm_count()));
  if (promote) {
    const cudaError_t ea = ensure_dynamic_smem((const void*)k_gemm<true>, kSmemBytes);
    if (ea != cudaSuccess) return ea;
    return launch_pdl(k_gemm<true>, dim3(grid), dim3(kThreads), kSmemBytes, st, mA, mB, p);
  } else {
    const cudaError_t ea = ensure_dynamic_smem((const void*)k_gemm<false>, kSmemBytes);
    if (ea != cudaSuccess) return ea;
    return launch_pdl(k_gemm<false>, dim3(grid), dim3(kThreads), kSmemBytes, st, mA, mB, p);
  }
}

cudaError_t launch_gemm(const uint8_t* A, const float* sA, int gA, const uint8_t* B, bool b_packed, const float* sB,
                        int gB, int64_t M, int64_t N, int64_t K, uint16_t* C, void* ws, size_t ws_bytes,
                        cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  const DecodePlan plan = decode_plan(M, N, K);
  if (plan.mp > 0) return launch_decode_gemm(plan, A, sA, gA, B, b_packed, sB, gB, M, N, K, C, ws, ws_bytes, st);
  return launch_prefill(A, sA, gA, B, b_packed, sB, gB, M, N, K, C, nullptr, nullptr, st);
}

cudaError_t launch_gemm_to_fp8(const uint8_t* A, const float* sA, int gA, const uint8_t* B, bool b_packed,
                               const float* sB, int gB, int64_t M, int64_t N, int64_t K, uint8_t* codes,
                               float* scales, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (decode_plan(M, N, K).mp > 0) return cudaErrorNotSupported;   // the decode kernel has no such epilogue
  return launch_prefill(A, sA, gA, B, b_packed, sB, gB, M, N, K, nullptr, codes, scales, st);
}

// Linear layer with dynamic activation quantization: C = GEMM(quantize_1x128_E4M3(X), B), as the
// 1x128 quantizer into act_ws followed by the block-scaled GEMM (two programmatic-dependent
// launches; for decode shapes the codes stay in L2 between them).  gemm_ws is the GEMM's own
// workspace (decode shapes), with its zero-fill rule.
size_t linear_act_workspace_bytes(int64_t M, int64_t K) {
  const size_t codes = ((size_t)M * (size_t)K + 255) / 256 * 256;
  return codes + (size_t)((K + 127) / 128) * (size_t)M * sizeof(float);
}

// The fused linear layer (prefill shapes): one cooperative launch of the block-scaled GEMM whose
// first phase quantizes X into act_ws (the two grid-barrier words in its first 256 bytes, then the
// codes, then the 1x128 scales),
// so the codes are read back from L2 by the second phase without a kernel boundary.
size_t linear_fused_workspace_bytes(int64_t M, int64_t K) {
  return (linear_act_workspace_bytes(M, K) + 255) / 256 * 256 + 256;
}

cudaError_t launch_linear_fused(const uint16_t* X, const uint8_t* B, const float* sB, int gB, int64_t M, int64_t N,
                                int64_t K, uint16_t* C, void* act_ws, cudaStream_t st) {
  using namespace gemm;
  if (M <= 64 || N == 0) return M <= 64 ? cudaErrorNotSupported : cudaSuccess;
  if (M * (K / BK) >= (int64_t(1) << 31)) return cudaErrorNotSupported;   // the phase's group index
  // the barrier words first, at a place that does not depend on the shape, so one buffer serves
  // calls of any shape; then the codes and the scales
  uint32_t* gbar = static_cast<uint32_t*>(act_ws);
  uint8_t* codes = static_cast<uint8_t*>(act_ws) + 256;
  float* scales = reinterpret_cast<float*>(codes + ((size_t)M * (size_t)K + 255) / 256 * 256);
  CUtensorMap mA, mB;
  std::memset(&mA, 0, sizeof(mA));
  std::memset(&mB, 0, sizeof(mB));
  if (!make_tmap_2d(&mA, 1, codes, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM, 1)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&mB, 1, B, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BN, 1)) return cudaErrorInvalidValue;
  Params p{};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.num_kb = (int)(K / BK);
  p.m_tiles = (int)((M + BM - 1) / BM);
  p.n_tiles = (int)((N + BN - 1) / BN);
  p.tiles = p.m_tiles * p.n_tiles;
  p.group_m = tile_group_m(M, K, p.m_tiles);
  p.sA = scales;
  p.sB = sB;
  p.gA_group = 1;
  p.gB_block = gB == 2;
  p.C = C;
  p.xq = X;
  p.xq_codes = codes;
  p.gbar = gbar;
  p.err = device_error_word();
  const cudaError_t ea = ensure_dynamic_smem((const void*)k_gemm<true, true>, kSmemBytes);
  if (ea != cudaSuccess) return ea;
  // every CTA must be resident for the grid barrier: a cooperative launch guarantees it (one CTA
  // per SM here) or fails
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max(1, std::min(p.tiles, device_sm_count())));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_gemm<true, true>, mA, mB, p);
}

cudaError_t launch_linear(const uint16_t* X, const uint8_t* B, const float* sB, int gB, int64_t M, int64_t N,
                          int64_t K, uint16_t* C, void* act_ws, void* gemm_ws, size_t gemm_ws_bytes,
                          cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  uint8_t* codes = static_cast<uint8_t*>(act_ws);
  float* scales = reinterpret_cast<float*>(codes + ((size_t)M * (size_t)K + 255) / 256 * 256);
  const cudaError_t e = launch_quant_1x128(X, M, K, 0, codes, scales, st);
  if (e != cudaSuccess) return e;
  return launch_gemm(codes, scales, 1, B, false, sB, gB, M, N, K, C, gemm_ws, gemm_ws_bytes, st);
}

}  // namespace fp8q
