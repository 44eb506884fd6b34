// Block-scaled FP8 GEMM on the fifth-generation tensor cores (tcgen05 + TMEM, fed by TMA).
// Placeholder until the tcgen05 kernel lands: reports "not supported".
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace fp8q {

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

cudaError_t launch_gemm(const uint8_t*, const float*, int, const uint8_t*, const float*, int, int64_t, int64_t,
                        int64_t, uint16_t*, void*, size_t, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace fp8q
