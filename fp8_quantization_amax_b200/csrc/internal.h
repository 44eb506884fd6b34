// Launchers shared between the C-ABI entry points and the kernel files.  Host-side only.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <utility>

namespace fp8q {

// Launch `kernel` as a programmatic dependent of the previous grid on `st`: it may begin while
// that grid finishes.  Every kernel launched this way calls grid_dependency_wait() (sm100.cuh)
// before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// number of SMs of the current device (queried once per device)
int device_sm_count();

// Raise `kernel`'s dynamic shared-memory limit on the current device to at least `bytes`, once
// per (kernel, device) and size (thread-safe); returns the error of cudaFuncSetAttribute, or
// cudaSuccess when an earlier call on this device already set a limit this large.
cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes);

// device address of the library's error word on the current device (kernels set bits in it
// when a bounded wait gives up); read_and_clear_device_error() synchronizes the device first
uint32_t* device_error_word();
uint32_t read_and_clear_device_error();

// 2-D TMA descriptor for a row-major [outer][inner] tensor of 1-, 2- or 4-byte elements with the
// given row stride; box = box_outer rows x box_inner elements
bool make_tmap_2d(CUtensorMap* map, int elem_bytes, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_128b);

// largest number of first-pass partial maxima any two-pass launch writes, per scale group
constexpr int kMaxPartials = 1024;

// 32-bit unsigned division by an invariant divisor (T. Granlund, P. Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994): q = (umulhi(n, m) + n) >> s.
struct FastDiv {
  uint32_t d, m, s;
};
FastDiv make_fastdiv(uint32_t d);

cudaError_t launch_encode(const float* q, int64_t n, int fmt, uint8_t* codes, cudaStream_t st);
cudaError_t launch_decode(const uint8_t* codes, int64_t n, int fmt, float* out, cudaStream_t st);

// one scale per (row, 128 consecutive columns); scales laid out [ceil(cols/128)][rows]
cudaError_t launch_quant_1x128(const uint16_t* x, int64_t rows, int64_t cols, int fmt, uint8_t* codes,
                               float* scales, cudaStream_t st);

// one scale per tile of 128 rows x gw columns of a [rows][ld] matrix (cols valid columns);
// up to two tensors in one launch; scales [ceil(rows/128)][nbc]
cudaError_t launch_quant_tiles(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                               float* s1, int ntens, int64_t rows, int64_t cols, int64_t ld, int gw, int fmt,
                               cudaStream_t st);

// two passes: amax per (tensor, head) over all rows, then the cast.  Each tensor is
// [rows][heads * head_dim]; per-tensor quantization is heads = 1, head_dim = cols.
size_t two_pass_workspace_bytes(int ntens, int64_t heads);
cudaError_t launch_quant_two_pass(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                                  float* s1, int ntens, int64_t rows, int64_t heads, int64_t head_dim, int fmt,
                                  float* ws, cudaStream_t st);

// delayed scaling over the same groups as launch_quant_two_pass: step 0 scales from the groups'
// own amax (two passes), step >= 1 from max(history) / FMAX in one pass; afterwards history
// slot step % hlen ([hlen][heads] per tensor) holds this call's amax.  counters (optional, [2])
// accumulate saturated and underflowed elements.
cudaError_t launch_quant_delayed(const uint16_t* x0, const uint16_t* x1, uint8_t* c0, uint8_t* c1, float* s0,
                                 float* s1, int ntens, int64_t rows, int64_t heads, int64_t head_dim, int fmt,
                                 float* h0, float* h1, int64_t hlen, int64_t step, unsigned long long* counters,
                                 float* ws, cudaStream_t st);

// several tensors, each in 1x128 groups (block = 0) or 128x128 blocks (block = 1), in one launch
constexpr int kMaxManyJobs = 8;
struct QuantJob {
  const uint16_t* x;
  int64_t rows, cols;
  int block;
  uint8_t* codes;
  float* scales;
};
cudaError_t launch_quant_many(const QuantJob* jobs, int n, int fmt, cudaStream_t st);

// MXFP8: 1x32 groups along rows (cols % 32 == 0), scales as byte exponents, row-major
// [rows][cols / 32] (blocked = 0) or in the blocked layout of the block-scaled MMA (blocked = 1:
// ceil(rows / 128) x ceil(cols / 128) chunks of 512 bytes)
cudaError_t launch_quant_mx(const uint16_t* x, int64_t rows, int64_t cols, int fmt, uint8_t* codes, uint8_t* scales,
                            int blocked, cudaStream_t st);

// y = bf16(decode(code) * s) under a granularity (0 tensor, 1 1x128, 2 128x128, 3 MX 1x32 with
// byte exponents passed through `scales`)
cudaError_t launch_dequant(const uint8_t* codes, const float* scales, int64_t rows, int64_t cols, int fmt,
                           int gran, uint16_t* y, cudaStream_t st);

// block-scaled / per-tensor FP8 GEMM on tcgen05
// (b_packed: B holds packed tiles, launch_pack_b_tiles, instead of row-major codes)
cudaError_t launch_gemm(const uint8_t* A, const float* sA, int gA, const uint8_t* B, bool b_packed, const float* sB,
                        int gB, int64_t M, int64_t N, int64_t K, uint16_t* C, void* ws, size_t ws_bytes,
                        cudaStream_t st);

// scale health: a 256-bucket histogram of scales by power of two (kind 0: fp32 scales by their
// exponent field; 1: MX bytes), added to hist; and the count of nonzero non-NaN inputs whose
// code is +-0, added to *count
cudaError_t launch_scale_histogram(const void* scales, int64_t n, int kind, uint32_t* hist, cudaStream_t st);
cudaError_t launch_count_underflow(const uint16_t* x, const uint8_t* codes, int64_t n, unsigned long long* count,
                                   cudaStream_t st);

// B codes [N][K] (N, K multiples of 128) -> packed 16 KB tiles in the 128-byte-swizzled image of
// a TMA load, tile (nb, kb) at 16384 (nb K/128 + kb)
cudaError_t launch_pack_b_tiles(const uint8_t* B, int64_t N, int64_t K, uint8_t* packed, cudaStream_t st);
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
// host-only consistency check of the decode split (fp8q_check_decode_split)
int check_decode_split(int64_t M, int64_t N, int64_t K, int sms);
// host-only check of the prefill GEMMs' tile walk (fp8q_check_tile_walk)
int check_tile_walk(int64_t M, int64_t N, int64_t K);

// the same GEMM (prefill shapes, M > 64) with C quantized in the epilogue to E4M3 1x128 groups:
// codes [M][N], scales [N/128][M]; cudaErrorNotSupported for decode shapes
cudaError_t launch_gemm_to_fp8(const uint8_t* A, const float* sA, int gA, const uint8_t* B, bool b_packed,
                               const float* sB, int gB, int64_t M, int64_t N, int64_t K, uint8_t* codes,
                               float* scales, cudaStream_t st);

// MXFP8 GEMM on the block-scaled MMA: A [M][K], B [N][K] codes (formats fa, fb), scales in the
// blocked layout; N % 128 == 0, K % 128 == 0
cudaError_t launch_gemm_mx(const uint8_t* A, const uint8_t* sfa, int fa, const uint8_t* B, const uint8_t* sfb, int fb,
                           int64_t M, int64_t N, int64_t K, uint16_t* C, cudaStream_t st);

// C = GEMM(quantize_1x128_E4M3(X), B) for bf16 X [M][K]: the 1x128 quantizer into act_ws
// (linear_act_workspace_bytes) and the block-scaled GEMM with gemm_ws
size_t linear_act_workspace_bytes(int64_t M, int64_t K);
cudaError_t launch_linear(const uint16_t* X, const uint8_t* B, const float* sB, int gB, int64_t M, int64_t N,
                          int64_t K, uint16_t* C, void* act_ws, void* gemm_ws, size_t gemm_ws_bytes,
                          cudaStream_t st);
// the same as one cooperative launch (M > 64): the quantizer as the GEMM kernel's first phase
size_t linear_fused_workspace_bytes(int64_t M, int64_t K);
cudaError_t launch_linear_fused(const uint16_t* X, const uint8_t* B, const float* sB, int gB, int64_t M, int64_t N,
                                int64_t K, uint16_t* C, void* act_ws, cudaStream_t st);

}  // namespace fp8q
