// tcgen05 building blocks shared by the GEMM kernels (sm_100a): shared-memory operand
// descriptors, MMA issue and commit, TMEM loads and the tcgen05 fences.
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace fp8q {
namespace gemm {

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

// Persistent tile walk of the prefill GEMMs: tile index t -> (M tile, N tile).  Tiles go in
// bands of group_m M tiles; inside a band M varies fastest, then N.  The CTAs running at the same
// time (consecutive t) then share group_m A panels and about gridDim / group_m B panels, and both
// are read from HBM about once per band instead of the whole A once per N column.  With
// group_m = m_tiles this is the plain M-fastest walk (kept when all of A fits in L2).
__host__ __device__ __forceinline__ void tile_walk(int t, int m_tiles, int n_tiles, int group_m, int* mt, int* nt) {
  const int per_band = group_m * n_tiles;
  const int band = t / per_band;
  const int r = t - band * per_band;
  const int rows = min(group_m, m_tiles - band * group_m);   // the last band may be shorter
  *nt = r / rows;
  *mt = band * group_m + (r - *nt * rows);
}

// The band height for an M x K A operand of E4M3 codes: the M-fastest walk while A fits in L2
// next to the B panels in flight, else 16 M tiles (for G concurrent CTAs the panels per band
// are about 16 of A and G / 16 of B, the minimum of A + B bytes per wave near G = 148).
inline int tile_group_m(int64_t M, int64_t K, int m_tiles) {
  constexpr int64_t kAInL2 = 48ll << 20;
  if (M * K <= kAInL2) return m_tiles;
  return m_tiles < 16 ? m_tiles : 16;
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

// 32-byte and 8-byte stores with the default cache policy (data read again soon)
__device__ __forceinline__ void st_v8(void* p, uint4 a, uint4 b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
               "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}
__device__ __forceinline__ void st_v2(void* p, uint2 a) {
  asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(p), "r"(a.x), "r"(a.y) : "memory");
}

// one 32-byte streaming store (a whole sector; p 32-byte aligned)
__device__ __forceinline__ void st_stream_v8(void* p, uint4 a, uint4 b) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
               "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

}  // namespace gemm
}  // namespace fp8q
