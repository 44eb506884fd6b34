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

#include "fp8q_device.cuh"
#include "internal.h"
#include "sm100.cuh"

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
  const float* sA;
  const float* sB;
  int gA_group;       // 1: sA is [K/128][M]; 0: one scale
  int gB_block;       // 1: sB is [N/128][K/128]; 0: one scale
  uint16_t* C;
  uint32_t* err;
};

// UMMA shared-memory descriptor for a K-major tile with 128-byte swizzle: rows of 128 bytes,
// 8-row groups 1024 bytes apart (stride byte offset), version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;                 // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;      // stride byte offset
  d |= (uint64_t)1 << 46;                 // descriptor version for sm_100
  d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void umma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive on `bar` once every tcgen05 operation this thread issued so far has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 32 columns of fp32 from TMEM: thread = lane, v[j] = column col + j
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tile_coords(int t, const Params& p, int* m0, int* n0) {
  const int mt = t % p.m_tiles, nt = t / p.m_tiles;
  *m0 = mt * BM;
  *n0 = nt * BN;
}

template <bool PROMOTE>
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
  const int my_tiles = p.tiles > (int)blockIdx.x ? (p.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  if (warp < kFirstEpiWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && my_tiles > 0) {
      tma_prefetch_desc(&tA);
      tma_prefetch_desc(&tB);
      int s = 0;
      uint32_t ph = 0;
      uint32_t it = 0;
      bool ok = true;
      for (int k = 0; k < my_tiles && ok; ++k) {
        int m0, n0;
        tile_coords((int)blockIdx.x + k * (int)gridDim.x, p, &m0, &n0);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          if (it >= (uint32_t)kStages && !mbar_wait(&empty[s], ph ^ 1u, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(sm_a + s * kStageA, &tA, kb * BK, m0, &full[s]);
          tma_load_2d(sm_b + s * kStageB, &tB, kb * BK, n0, &full[s]);
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
            uint16_t* dst = p.C + (size_t)m * p.N + ncol0;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              uint4 wv;
              wv.x = f32x2_to_bf16x2(acc[c * 4 + 0].x, acc[c * 4 + 0].y);
              wv.y = f32x2_to_bf16x2(acc[c * 4 + 1].x, acc[c * 4 + 1].y);
              wv.z = f32x2_to_bf16x2(acc[c * 4 + 2].x, acc[c * 4 + 2].y);
              wv.w = f32x2_to_bf16x2(acc[c * 4 + 3].x, acc[c * 4 + 3].y);
              st_stream_v4(dst + c * 8, wv);
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
          uint16_t* dst = p.C + (size_t)m * p.N + ncol0;
#pragma unroll
          for (int c = 0; c < 16; ++c)
            st_stream_v4(dst + c * 8, make_uint4(out[c * 4], out[c * 4 + 1], out[c * 4 + 2], out[c * 4 + 3]));
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

}  // namespace gemm

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

cudaError_t launch_gemm(const uint8_t* A, const float* sA, int gA, const uint8_t* B, const float* sB, int gB,
                        int64_t M, int64_t N, int64_t K, uint16_t* C, void*, size_t, cudaStream_t st) {
  using namespace gemm;
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap mA, mB;
  std::memset(&mA, 0, sizeof(mA));
  std::memset(&mB, 0, sizeof(mB));
  if (!make_tmap_2d(&mA, 1, A, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM, 1)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&mB, 1, B, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BN, 1)) return cudaErrorInvalidValue;
  Params p;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.num_kb = (int)(K / BK);
  p.m_tiles = (int)((M + BM - 1) / BM);
  p.n_tiles = (int)((N + BN - 1) / BN);
  p.tiles = p.m_tiles * p.n_tiles;
  p.sA = sA;
  p.sB = sB;
  p.gA_group = gA == 1;
  p.gB_block = gB == 2;
  p.C = C;
  p.err = device_error_word();
  const bool promote = p.gA_group || p.gB_block;
  const int grid = std::max(1, std::min(p.tiles, device_sm_count()));
  if (promote) {
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(k_gemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
      attr = true;
    }
    k_gemm<true><<<grid, kThreads, kSmemBytes, st>>>(mA, mB, p);
  } else {
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(k_gemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
      attr = true;
    }
    k_gemm<false><<<grid, kThreads, kSmemBytes, st>>>(mA, mB, p);
  }
  return cudaGetLastError();
}

}  // namespace fp8q
