// Packed B tiles for the GEMMs: each 128 x 128 tile of the codes becomes one contiguous 16 KB
// block laid out exactly as a 128-byte-swizzled TMA load would leave it in shared memory (row
// r at byte 128 r, its 16-byte piece j at position j XOR (r % 8)), so the GEMMs fetch a whole
// tile with one bulk copy instead of 128 row requests.  Tile (nb, kb) sits at 16384 (nb K/128 + kb).
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fp8q {
namespace {

// one thread per 16-byte piece; a warp reads 512 contiguous bytes of a row (four tiles' rows)
__global__ void k_pack_b_tiles(const uint4* __restrict__ b, uint4* __restrict__ out, int64_t K, uint32_t nkb,
                               int64_t pieces) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= pieces) return;
  const int64_t per_row = K / 16;
  const int64_t n = i / per_row;
  const int64_t j = i - n * per_row;            // piece along the row
  const int64_t kb = j >> 3, piece = j & 7;
  const int64_t r = n & 127, nb = n >> 7;
  const int64_t dst = ((nb * nkb + kb) * 16384 + r * 128 + ((piece ^ (r & 7)) << 4)) >> 4;
  out[dst] = __ldg(b + i);
}

}  // namespace

cudaError_t launch_pack_b_tiles(const uint8_t* B, int64_t N, int64_t K, uint8_t* packed, cudaStream_t st) {
  const int64_t pieces = N * K / 16;
  if (pieces == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (pieces + threads - 1) / threads;
  k_pack_b_tiles<<<(unsigned)blocks, threads, 0, st>>>(reinterpret_cast<const uint4*>(B), reinterpret_cast<uint4*>(packed),
                                                       K, (uint32_t)(K / 128), pieces);
  return cudaGetLastError();
}

}  // namespace fp8q
