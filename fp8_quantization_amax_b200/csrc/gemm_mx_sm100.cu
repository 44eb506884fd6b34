// MXFP8 GEMM on the tensor cores' block-scaled MMA (sm_100a: tcgen05.mma kind::mxf8f6f4).
//
// Method: api.makesence.top "LLM推理量化:FP8 versus INT8", the Microscaling passage (every 32
// consecutive elements along K share one power-of-two scale; native on Blackwell) and wangyu.me
// "大语言模型量化技术（五）：FP8", "FP8 矩阵乘" (FP8 products with fp32 accumulation, the scales
// multiplied back).  Here the tensor core applies the scales itself: each MMA of K = 32 reads
// one UE8M0 scale per row of A and per column of B from tensor memory, so the whole of K
// accumulates in TMEM and no promotion pass exists:
//     C[m][n] = bf16( sum_k decode(A[m][k]) 2^(sA[m][k/32]-127) decode(B[n][k]) 2^(sB[n][k/32]-127) )
//
// Scale input: the blocked layout (one 512-byte chunk per 128 rows x 128 K; chunk (rb, kb) at
// 512 (rb * K/128 + kb); in a chunk, byte 16 (r % 32) + 4 ((r % 128) / 32) + j holds the scale of
// row r and the j-th 32-column group).  A chunk is exactly what one tcgen05.cp 32x128b.warpx4
// moves into TMEM: 32 lanes x 16 bytes, replicated into the four lane quarters, so lane l holds
// the scales of rows l % 32 + 32 c in column c, one byte per 32-column group.
//
// One persistent CTA per SM walks output tiles of 128 x 256 (m fastest):
//   warp 0      producer: per K block of 128, the A box 128 x 128 and the B box 256 x 128
//               (128-byte swizzle, TMA) and the scale chunks of A (512 B) and of B's two
//               128-row halves (bulk copies) into a 4-stage shared-memory ring.
//   warp 1      allocates 512 TMEM columns: two 256-column accumulators that overlap by one
//               32-column chunk (columns 0..255 and 224..479), A scales 480..483, B scales
//               484..491; lane 0 copies each stage's scale chunks into TMEM (tcgen05.cp) and
//               issues four block-scaled MMAs (M128 N256 K32).  tcgen05 operations of one thread
//               run in issue order, so one set of scale columns serves every K block.
//   warps 2-3   idle (they complete warpgroup 0, which hands its registers to the epilogue).
//   warps 4-11  epilogue: TMEM -> registers -> bf16, release the accumulator, then store.  The
//               warps holding the shared chunk read it first and release it at once, so the
//               next tile's MMAs (into the other accumulator) wait only for that one load.
// Every mbarrier wait is bounded (sm100.cuh): on a timeout the kernel records an error in the
// device error word and winds down instead of hanging.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "fp8q_device.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tcgen05.cuh"

namespace fp8q {
namespace gemm {
namespace mx {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int kStages = 4;
constexpr uint32_t kStageA = BM * BK;                 // 16 KB of codes
constexpr uint32_t kStageB = BN * BK;                 // 32 KB
constexpr uint32_t kSfChunk = 512;                    // scales of 128 rows x 128 K
constexpr uint32_t kStageSf = kSfChunk * (1 + BN / 128);
constexpr int kEpiWarps = 8;
constexpr int kFirstEpiWarp = 4;
constexpr int kThreads = 128 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBuf1Col = 224;                    // second accumulator: shares columns 224..255
constexpr uint32_t kSfaCol = 480;                     // 4 columns: rows 32c .. 32c + 31 in column c
constexpr uint32_t kSfbCol = 484;                     // 8 columns for the tile's 256 B rows

// the same register split as the block-scaled GEMM (the build checks the launch count)
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 40;
constexpr int kEpilogueRegs = 232;
static_assert(128 * kProducerRegs + 256 * kEpilogueRegs == kThreads * kLaunchRegs, "register split must add up");

// kind::mxf8f6f4 block-scaled instruction descriptor: A / B formats (0 E4M3, 1 E5M2) at bits 7
// and 10, both K-major, N >> 3 at bit 17, UE8M0 scales (bit 23), M >> 4 at bit 24; the scale
// byte selectors of B (bits 4-5) and A (bits 29-30) are set per MMA.
__host__ __device__ constexpr uint32_t idesc_mx(int fa, int fb) {
  return ((uint32_t)fa << 7) | ((uint32_t)fb << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) |
         ((uint32_t)(BM >> 4) << 24);
}

struct Params {
  int M, N, K;
  int num_kb;
  int m_tiles, n_tiles, tiles;
  int group_m;          // tile walk band height (tile_walk)
  uint32_t idesc;
  const uint8_t* sfa;   // blocked, ceil(M / 128) x K / 128 chunks
  const uint8_t* sfb;   // blocked, N / 128 x K / 128 chunks
  uint16_t* C;
  uint32_t* err;
};

// shared-memory descriptor of one 512-byte scale chunk as the source of tcgen05.cp 32x128b:
// no swizzle, 16-byte rows, 8-row core matrices 128 bytes apart (stride byte offset), version 1
__device__ __forceinline__ uint64_t sf_chunk_desc(uint32_t smem_addr) {
  uint64_t d = (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(128u >> 4) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// 32 rows x 128 bits of shared memory -> TMEM columns taddr .. taddr + 3 of lanes 0-31, copied
// to the other three lane quarters as well
__device__ __forceinline__ void tmem_copy_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void umma_mx(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

// one 32-column chunk of this thread's accumulator row -> 16 packed bf16 pairs
template <int C>
__device__ __forceinline__ void epi_chunk(uint32_t taddr, uint32_t (&out)[64]) {
  uint32_t v[32];
  tmem_ld32(taddr + C * 32, v);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 16; ++i)
    out[C * 16 + i] = f32x2_to_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
}

__global__ void __launch_bounds__(kThreads, 1) k_gemm_mx(const __grid_constant__ CUtensorMap tA,
                                                         const __grid_constant__ CUtensorMap tB, Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  uint8_t* sm_a = smem;                                      // kStages x 16 KB
  uint8_t* sm_b = smem + kStages * kStageA;                  // kStages x 32 KB
  uint8_t* sm_sf = smem + kStages * (kStageA + kStageB);     // kStages x 1.5 KB (A, B half 0, B half 1)
  uint64_t* full = reinterpret_cast<uint64_t*>(sm_sf + kStages * kStageSf);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;                         // [2] per accumulator
  uint64_t* tempty = tfull + 2;                              // [2]
  uint64_t* ofree = tempty + 2;                              // shared chunk read, once per tile
  uint64_t* drain = ofree + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

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
    mbar_init(ofree, kEpiWarps / 2);
    mbar_init(drain, 1);
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
  const int my_tiles = p.tiles > (int)blockIdx.x ? (p.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  if (warp < kFirstEpiWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0 && my_tiles > 0) {
        tma_prefetch_desc(&tA);
        tma_prefetch_desc(&tB);
        int s = 0;
        uint32_t ph = 0, it = 0;
        bool ok = true;
        for (int k = 0; k < my_tiles && ok; ++k) {
          const int t = (int)blockIdx.x + k * (int)gridDim.x;
          int mt, nt;
          tile_walk(t, p.m_tiles, p.n_tiles, p.group_m, &mt, &nt);
          const int m0 = mt * BM, n0 = nt * BN;
          const int nhalves = min(2, (p.N - n0) / 128);    // N % 128 == 0: 1 or 2 valid B halves
          const uint8_t* sfa = p.sfa + (size_t)mt * p.num_kb * kSfChunk;
          const uint8_t* sfb = p.sfb + (size_t)(n0 / 128) * p.num_kb * kSfChunk;
          for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
            if (it >= (uint32_t)kStages && !mbar_wait(&empty[s], ph ^ 1u, p.err)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], kStageA + kStageB + kSfChunk * (1 + nhalves));
            tma_load_2d(sm_a + s * kStageA, &tA, kb * BK, m0, &full[s]);
            tma_load_2d(sm_b + s * kStageB, &tB, kb * BK, n0, &full[s]);
            uint8_t* sf = sm_sf + s * kStageSf;
            bulk_load(sf, sfa + (size_t)kb * kSfChunk, kSfChunk, &full[s]);
            for (int h = 0; h < nhalves; ++h)
              bulk_load(sf + (1 + h) * kSfChunk, sfb + ((size_t)h * p.num_kb + kb) * kSfChunk, kSfChunk, &full[s]);
            if (++s == kStages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        // drain: every issued copy lands before the CTA may exit
        for (uint32_t j = 0; j < (uint32_t)kStages && j < it; ++j) {
          const uint32_t kk = it - 1 - j;
          mbar_wait(&full[kk % kStages], (kk / kStages) & 1u, p.err);
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- scale copies + MMA issue
      if (lane == 0 && my_tiles > 0) {
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        const uint32_t tsfa = tmem_base + kSfaCol, tsfb = tmem_base + kSfbCol;
        for (int k = 0; k < my_tiles && ok; ++k) {
          const uint32_t buf = (uint32_t)k & 1u;
          // this accumulator's previous tile has been read out, and the previous tile (in the
          // other accumulator) has released the shared chunk
          if (k >= 2 && !mbar_wait(&tempty[buf], ((uint32_t)(k >> 1) - 1u) & 1u, p.err)) {
            ok = false;
            break;
          }
          if (k >= 1 && !mbar_wait(ofree, (uint32_t)(k - 1) & 1u, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tmem_d = tmem_base + (buf ? kBuf1Col : 0u);
          for (int kb = 0; kb < p.num_kb; ++kb) {
            if (!mbar_wait(&full[s], ph, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sf = smem_u32(sm_sf + s * kStageSf);
            tmem_copy_sf(tsfa, sf_chunk_desc(sf));
            tmem_copy_sf(tsfb, sf_chunk_desc(sf + kSfChunk));
            tmem_copy_sf(tsfb + 4, sf_chunk_desc(sf + 2 * kSfChunk));
            const uint64_t adesc = umma_desc_sw128(smem_u32(sm_a + s * kStageA));
            const uint64_t bdesc = umma_desc_sw128(smem_u32(sm_b + s * kStageB));
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk) {
              // scale byte kk of each TMEM word: the address' top two bits and the descriptor's
              // selectors name it
              const uint32_t sel = (uint32_t)kk;
              umma_mx(tmem_d, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2),
                      p.idesc | (sel << 4) | (sel << 29), tsfa | (sel << 30), tsfb | (sel << 30),
                      (kb > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&empty[s]);                       // frees the stage (codes and scales)
            if (kb == p.num_kb - 1) umma_commit(&tfull[buf]);   // tile accumulated
            if (++s == kStages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        // every tcgen05 operation issued above (on any path) completes before TMEM is released
        umma_commit(drain);
        mbar_wait(drain, 0u, p.err);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpilogueRegs));
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kFirstEpiWarp;
    const int quarter = warp & 3;            // TMEM lane quarter this warp may access
    const int half = ew >> 2;                // 128-column half of the tile
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16) + half * 128;
    for (int k = 0; k < my_tiles; ++k) {
      const int t = (int)blockIdx.x + k * (int)gridDim.x;
      int mt, nt;
      tile_walk(t, p.m_tiles, p.n_tiles, p.group_m, &mt, &nt);
      const int m = mt * BM + row_in_tile;
      const int ncol0 = nt * BN + half * 128;
      const uint32_t buf = (uint32_t)k & 1u;
      if (!mbar_wait(&tfull[buf], (uint32_t)(k >> 1) & 1u, p.err)) break;
      tc_fence_after();
      const uint32_t taddr = lane_base + (buf ? kBuf1Col : 0u);
      uint32_t out[64];
      // the shared chunk is accumulator 0's last (tile columns 224..255, held by half 1) and
      // accumulator 1's first (tile columns 0..31, half 0): its holders read it first
      const bool first_last = buf == 0 && half == 1;
      const bool holds_shared = first_last || (buf == 1 && half == 0);
      if (first_last) {
        epi_chunk<3>(taddr, out);
      } else {
        epi_chunk<0>(taddr, out);
      }
      if (holds_shared) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ofree);
      }
      if (first_last) {
        epi_chunk<0>(taddr, out);
        epi_chunk<1>(taddr, out);
        epi_chunk<2>(taddr, out);
      } else {
        epi_chunk<1>(taddr, out);
        epi_chunk<2>(taddr, out);
        epi_chunk<3>(taddr, out);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (m < p.M && ncol0 < p.N) {
        uint16_t* dst = p.C + (size_t)m * p.N + ncol0;
#pragma unroll
        for (int c = 0; c < 8; ++c)   // 32-byte stores: every store fills whole sectors
          st_stream_v8(dst + c * 16, make_uint4(out[c * 8], out[c * 8 + 1], out[c * 8 + 2], out[c * 8 + 3]),
                       make_uint4(out[c * 8 + 4], out[c * 8 + 5], out[c * 8 + 6], out[c * 8 + 7]));
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

constexpr size_t kSmemBytes = 1024 + kStages * (kStageA + kStageB + kStageSf) + (2 * kStages + 6) * sizeof(uint64_t) + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

}  // namespace mx
}  // namespace gemm

cudaError_t launch_gemm_mx(const uint8_t* A, const uint8_t* sfa, int fa, const uint8_t* B, const uint8_t* sfb, int fb,
                           int64_t M, int64_t N, int64_t K, uint16_t* C, cudaStream_t st) {
  using namespace gemm::mx;
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
  p.group_m = gemm::tile_group_m(M, K, p.m_tiles);
  p.idesc = idesc_mx(fa, fb);
  p.sfa = sfa;
  p.sfb = sfb;
  p.C = C;
  p.err = device_error_word();
  const int grid = std::max(1, std::min(p.tiles, device_sm_count()));
  const cudaError_t ea = ensure_dynamic_smem((const void*)k_gemm_mx, kSmemBytes);
  if (ea != cudaSuccess) return ea;
  return launch_pdl(k_gemm_mx, dim3(grid), dim3(kThreads), kSmemBytes, st, mA, mB, p);
}

}  // namespace fp8q
