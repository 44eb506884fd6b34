// C-ABI entry points declared in include/fp8q.h: argument validation, sizes and dispatch.
// Every check happens on the host before anything is launched.
#include <cuda_runtime.h>

#include <cstdint>

#include "fp8q.h"
#include "internal.h"

namespace fp8q {
cudaError_t launch_selftest_wait(cudaStream_t st);
}

namespace {

constexpr int64_t kMaxElems = int64_t(1) << 33;   // 32-bit indexing of 16-byte pieces of two tensors
constexpr int64_t kMaxHistory = int64_t(1) << 20;   // amax history entries per group (the kernels index with int)

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool valid_fmt(int f) { return f == FP8Q_E4M3 || f == FP8Q_E5M2; }
bool valid_gran(int g) { return g == FP8Q_PER_TENSOR || g == FP8Q_GROUP_1x128 || g == FP8Q_BLOCK_128x128; }
bool valid_kv_gran(int g) {
  return g == FP8Q_KV_PER_TENSOR || g == FP8Q_KV_PER_HEAD || g == FP8Q_KV_PER_HEAD_TOK128;
}
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// rows * cols without overflow; -1 when it does not fit the library's indexing
int64_t checked_elems(int64_t a, int64_t b) {
  if (a < 0 || b < 0) return -1;
  if (a == 0 || b == 0) return 0;
  if (a > kMaxElems / b) return -1;
  return a * b;
}

fp8q_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA; }

}  // namespace

extern "C" {

const char* fp8q_status_string(fp8q_status status) {
  switch (status) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_INVALID_ARGUMENT: return "invalid argument";
    case FP8Q_ERR_UNSUPPORTED: return "unsupported";
    case FP8Q_ERR_WORKSPACE: return "workspace missing or too small";
    case FP8Q_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

int fp8q_version(void) { return 100; }

uint32_t fp8q_device_status(void) { return fp8q::read_and_clear_device_error(); }

fp8q_status fp8q_selftest_wait_timeout(fp8q_stream_t stream) {
  return from_cuda(fp8q::launch_selftest_wait((cudaStream_t)stream));
}

int fp8q_check_tile_walk(int64_t M, int64_t N, int64_t K) { return fp8q::check_tile_walk(M, N, K); }

int fp8q_check_decode_split(int64_t M, int64_t N, int64_t K, int sms) {
  return fp8q::check_decode_split(M, N, K, sms);
}

size_t fp8q_num_scales(int64_t rows, int64_t cols, fp8q_granularity g) {
  if (rows < 0 || cols < 0 || !valid_gran(g)) return 0;
  if (g == FP8Q_PER_TENSOR) return 1;
  if (g == FP8Q_GROUP_1x128) return (size_t)(cdiv(cols, 128) * rows);
  return (size_t)(cdiv(rows, 128) * cdiv(cols, 128));
}

size_t fp8q_workspace_bytes(int64_t rows, int64_t cols, fp8q_granularity g) {
  if (rows < 0 || cols < 0 || !valid_gran(g)) return 0;
  return g == FP8Q_PER_TENSOR ? fp8q::two_pass_workspace_bytes(1, 1) : 0;
}

size_t fp8q_kv_num_scales(int64_t tokens, int64_t heads, fp8q_kv_granularity g) {
  if (tokens < 0 || heads < 0 || !valid_kv_gran(g)) return 0;
  if (g == FP8Q_KV_PER_TENSOR) return 1;
  if (g == FP8Q_KV_PER_HEAD) return (size_t)heads;
  return (size_t)(cdiv(tokens, 128) * heads);
}

size_t fp8q_kv_workspace_bytes(int64_t tokens, int64_t heads, int64_t head_dim, fp8q_kv_granularity g) {
  if (tokens < 0 || heads < 0 || head_dim < 0 || !valid_kv_gran(g)) return 0;
  if (g == FP8Q_KV_PER_TENSOR) return fp8q::two_pass_workspace_bytes(2, 1);
  if (g == FP8Q_KV_PER_HEAD) return fp8q::two_pass_workspace_bytes(2, heads);
  return 0;
}

size_t fp8q_linear_act_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0 || K % 128 != 0 || checked_elems(M, K) < 0) return 0;
  return fp8q::linear_act_workspace_bytes(M, K);
}

size_t fp8q_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return fp8q::gemm_workspace_bytes(M, N, K);
}

fp8q_status fp8_encode(const float* q, int64_t n, fp8q_format f, uint8_t* codes, fp8q_stream_t stream) {
  if (n < 0 || n > kMaxElems || !valid_fmt(f)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n == 0) return FP8Q_OK;
  if (!q || !codes || !aligned(q, 16) || !aligned(codes, 16)) return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_encode(q, n, f, codes, (cudaStream_t)stream));
}

fp8q_status fp8_decode(const uint8_t* codes, int64_t n, fp8q_format f, float* out, fp8q_stream_t stream) {
  if (n < 0 || n > kMaxElems || !valid_fmt(f)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n == 0) return FP8Q_OK;
  if (!codes || !out || !aligned(codes, 16) || !aligned(out, 16)) return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_decode(codes, n, f, out, (cudaStream_t)stream));
}

fp8q_status fp8_quantize(const void* x, int64_t rows, int64_t cols, fp8q_format f, fp8q_granularity g,
                         uint8_t* codes, float* scales, void* ws, size_t ws_bytes, fp8q_stream_t stream) {
  const int64_t n = checked_elems(rows, cols);
  if (rows < 0 || cols < 0 || !valid_fmt(f) || !valid_gran(g) || cols % 8 != 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n < 0) return FP8Q_ERR_UNSUPPORTED;
  if (n > 0 && (!x || !codes || !aligned(x, 16) || !aligned(codes, 16))) return FP8Q_ERR_INVALID_ARGUMENT;
  if ((n > 0 || g == FP8Q_PER_TENSOR) && (!scales || !aligned(scales, 4))) return FP8Q_ERR_INVALID_ARGUMENT;
  const cudaStream_t st = (cudaStream_t)stream;
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  if (g == FP8Q_PER_TENSOR) {
    const size_t need = fp8q_workspace_bytes(rows, cols, g);
    if (!ws || ws_bytes < need || !aligned(ws, 4)) return FP8Q_ERR_WORKSPACE;
    return from_cuda(fp8q::launch_quant_two_pass(xs, nullptr, codes, nullptr, scales, nullptr, 1, rows, 1, cols, f,
                                                 static_cast<float*>(ws), st));
  }
  if (n == 0) return FP8Q_OK;
  if (g == FP8Q_GROUP_1x128) return from_cuda(fp8q::launch_quant_1x128(xs, rows, cols, f, codes, scales, st));
  return from_cuda(
      fp8q::launch_quant_tiles(xs, nullptr, codes, nullptr, scales, nullptr, 1, rows, cols, cols, 128, f, st));
}

fp8q_status fp8_quantize_many(const fp8q_quant_tensor* tensors, int n, fp8q_format f, fp8q_stream_t stream) {
  if (!tensors || n < 1 || n > fp8q::kMaxManyJobs || !valid_fmt(f)) return FP8Q_ERR_INVALID_ARGUMENT;
  fp8q::QuantJob jobs[fp8q::kMaxManyJobs];
  for (int j = 0; j < n; ++j) {
    const fp8q_quant_tensor& t = tensors[j];
    const int64_t e = checked_elems(t.rows, t.cols);
    if (t.rows < 0 || t.cols < 0 || !valid_gran(t.g) || t.cols % 8 != 0) return FP8Q_ERR_INVALID_ARGUMENT;
    if (t.g == FP8Q_PER_TENSOR) return FP8Q_ERR_UNSUPPORTED;
    if (e < 0) return FP8Q_ERR_UNSUPPORTED;
    if (e > 0 && (!t.x || !t.codes || !t.scales || !aligned(t.x, 16) || !aligned(t.codes, 16) ||
                  !aligned(t.scales, 4)))
      return FP8Q_ERR_INVALID_ARGUMENT;
    jobs[j].x = static_cast<const uint16_t*>(t.x);
    jobs[j].rows = t.rows;
    jobs[j].cols = t.cols;
    jobs[j].block = t.g == FP8Q_BLOCK_128x128 ? 1 : 0;
    jobs[j].codes = t.codes;
    jobs[j].scales = t.scales;
  }
  return from_cuda(fp8q::launch_quant_many(jobs, n, f, (cudaStream_t)stream));
}

fp8q_status fp8_quantize_mx(const void* x, int64_t rows, int64_t cols, fp8q_format f, uint8_t* codes,
                            uint8_t* scales, fp8q_stream_t stream) {
  const int64_t n = checked_elems(rows, cols);
  if (rows < 0 || cols < 0 || !valid_fmt(f) || cols % 32 != 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n < 0) return FP8Q_ERR_UNSUPPORTED;
  if (n == 0) return FP8Q_OK;
  if (!x || !codes || !scales || !aligned(x, 16) || !aligned(codes, 16)) return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_quant_mx(static_cast<const uint16_t*>(x), rows, cols, f, codes, scales, 0,
                                         (cudaStream_t)stream));
}

size_t fp8q_mx_blocked_scale_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return 0;
  return (size_t)(cdiv(rows, 128) * cdiv(cols, 128) * 512);
}

fp8q_status fp8_quantize_mx_blocked(const void* x, int64_t rows, int64_t cols, fp8q_format f, uint8_t* codes,
                                    uint8_t* scales, fp8q_stream_t stream) {
  const int64_t n = checked_elems(rows, cols);
  if (rows < 0 || cols < 0 || !valid_fmt(f) || cols % 32 != 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n < 0) return FP8Q_ERR_UNSUPPORTED;
  if (n == 0) return FP8Q_OK;
  if (!x || !codes || !scales || !aligned(x, 16) || !aligned(codes, 16)) return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_quant_mx(static_cast<const uint16_t*>(x), rows, cols, f, codes, scales, 1,
                                         (cudaStream_t)stream));
}

fp8q_status fp8_dequantize_mx(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, fp8q_format f,
                              void* y, fp8q_stream_t stream) {
  const int64_t n = checked_elems(rows, cols);
  if (rows < 0 || cols < 0 || !valid_fmt(f) || cols % 32 != 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n < 0) return FP8Q_ERR_UNSUPPORTED;
  if (n == 0) return FP8Q_OK;
  if (!codes || !scales || !y || !aligned(codes, 16) || !aligned(y, 16)) return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_dequant(codes, reinterpret_cast<const float*>(scales), rows, cols, f, 3,
                                        static_cast<uint16_t*>(y), (cudaStream_t)stream));
}

fp8q_status fp8_quantize_delayed(const void* x, int64_t rows, int64_t cols, fp8q_format f, float* amax_history,
                                 int64_t history_len, int64_t step, uint8_t* codes, float* scale,
                                 unsigned long long* counts, void* ws, size_t ws_bytes, fp8q_stream_t stream) {
  const int64_t n = checked_elems(rows, cols);
  if (rows < 0 || cols < 0 || !valid_fmt(f) || cols % 8 != 0 || history_len < 1 || step < 0)
    return FP8Q_ERR_INVALID_ARGUMENT;
  if (n < 0 || history_len > kMaxHistory) return FP8Q_ERR_UNSUPPORTED;
  if (n > 0 && (!x || !codes || !aligned(x, 16) || !aligned(codes, 16))) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!scale || !aligned(scale, 4) || !amax_history || !aligned(amax_history, 4)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (counts && !aligned(counts, 8)) return FP8Q_ERR_INVALID_ARGUMENT;
  const size_t need = fp8q_workspace_bytes(rows, cols, FP8Q_PER_TENSOR);
  if (!ws || ws_bytes < need || !aligned(ws, 4)) return FP8Q_ERR_WORKSPACE;
  return from_cuda(fp8q::launch_quant_delayed(static_cast<const uint16_t*>(x), nullptr, codes, nullptr, scale, nullptr,
                                              1, rows, 1, cols, f, amax_history, nullptr, history_len, step, counts,
                                              static_cast<float*>(ws), (cudaStream_t)stream));
}

fp8q_status fp8_dequantize(const uint8_t* codes, const float* scales, int64_t rows, int64_t cols, fp8q_format f,
                           fp8q_granularity g, void* y, fp8q_stream_t stream) {
  const int64_t n = checked_elems(rows, cols);
  if (rows < 0 || cols < 0 || !valid_fmt(f) || !valid_gran(g) || cols % 8 != 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n < 0) return FP8Q_ERR_UNSUPPORTED;
  if (n == 0) return FP8Q_OK;
  if (!codes || !scales || !y || !aligned(codes, 16) || !aligned(y, 16) || !aligned(scales, 4))
    return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_dequant(codes, scales, rows, cols, f, g, static_cast<uint16_t*>(y),
                                        (cudaStream_t)stream));
}

fp8q_status fp8_kv_quantize(const void* k, const void* v, int64_t tokens, int64_t heads, int64_t head_dim,
                            fp8q_format f, fp8q_kv_granularity g, uint8_t* k_codes, uint8_t* v_codes,
                            float* k_scales, float* v_scales, void* ws, size_t ws_bytes, fp8q_stream_t stream) {
  if (tokens < 0 || heads < 0 || head_dim < 0 || !valid_fmt(f) || !valid_kv_gran(g) || head_dim % 8 != 0)
    return FP8Q_ERR_INVALID_ARGUMENT;
  const int64_t row = checked_elems(heads, head_dim);
  const int64_t n = row < 0 ? -1 : checked_elems(tokens, row);
  if (n < 0) return FP8Q_ERR_UNSUPPORTED;
  if (g == FP8Q_KV_PER_HEAD_TOK128 && head_dim > 256) return FP8Q_ERR_UNSUPPORTED;
  if (g == FP8Q_KV_PER_HEAD && (heads > 128 || head_dim > 256)) return FP8Q_ERR_UNSUPPORTED;
  const size_t nsc = fp8q_kv_num_scales(tokens, heads, g);
  if (n > 0 && (!k || !v || !k_codes || !v_codes || !aligned(k, 16) || !aligned(v, 16) || !aligned(k_codes, 16) ||
                !aligned(v_codes, 16)))
    return FP8Q_ERR_INVALID_ARGUMENT;
  if (nsc > 0 && (!k_scales || !v_scales || !aligned(k_scales, 4) || !aligned(v_scales, 4)))
    return FP8Q_ERR_INVALID_ARGUMENT;
  const cudaStream_t st = (cudaStream_t)stream;
  const uint16_t* ks = static_cast<const uint16_t*>(k);
  const uint16_t* vs = static_cast<const uint16_t*>(v);
  if (g == FP8Q_KV_PER_HEAD_TOK128) {
    if (n == 0) return FP8Q_OK;
    return from_cuda(fp8q::launch_quant_tiles(ks, vs, k_codes, v_codes, k_scales, v_scales, 2, tokens, row, row,
                                              (int)head_dim, f, st));
  }
  if (nsc == 0) return FP8Q_OK;   // no heads: nothing to write
  const size_t need = fp8q_kv_workspace_bytes(tokens, heads, head_dim, g);
  if (!ws || ws_bytes < need || !aligned(ws, 4)) return FP8Q_ERR_WORKSPACE;
  const int64_t h = g == FP8Q_KV_PER_TENSOR ? 1 : heads;
  const int64_t d = g == FP8Q_KV_PER_TENSOR ? row : head_dim;
  return from_cuda(fp8q::launch_quant_two_pass(ks, vs, k_codes, v_codes, k_scales, v_scales, 2, tokens, h, d, f,
                                               static_cast<float*>(ws), st));
}

fp8q_status fp8_kv_quantize_delayed(const void* k, const void* v, int64_t tokens, int64_t heads, int64_t head_dim,
                                    fp8q_format f, fp8q_kv_granularity g, float* k_history, float* v_history,
                                    int64_t history_len, int64_t step, uint8_t* k_codes, uint8_t* v_codes,
                                    float* k_scales, float* v_scales, unsigned long long* counts, void* ws,
                                    size_t ws_bytes, fp8q_stream_t stream) {
  if (tokens < 0 || heads < 0 || head_dim < 0 || !valid_fmt(f) || !valid_kv_gran(g) || head_dim % 8 != 0 ||
      history_len < 1 || step < 0)
    return FP8Q_ERR_INVALID_ARGUMENT;
  if (g == FP8Q_KV_PER_HEAD_TOK128) return FP8Q_ERR_UNSUPPORTED;   // already one pass: no history to keep
  const int64_t row = checked_elems(heads, head_dim);
  const int64_t n = row < 0 ? -1 : checked_elems(tokens, row);
  if (n < 0 || history_len > kMaxHistory) return FP8Q_ERR_UNSUPPORTED;
  if (g == FP8Q_KV_PER_HEAD && (heads > 128 || head_dim > 256)) return FP8Q_ERR_UNSUPPORTED;
  const size_t nsc = fp8q_kv_num_scales(tokens, heads, g);
  if (n > 0 && (!k || !v || !k_codes || !v_codes || !aligned(k, 16) || !aligned(v, 16) || !aligned(k_codes, 16) ||
                !aligned(v_codes, 16)))
    return FP8Q_ERR_INVALID_ARGUMENT;
  if (nsc > 0 && (!k_scales || !v_scales || !aligned(k_scales, 4) || !aligned(v_scales, 4) || !k_history ||
                  !v_history || !aligned(k_history, 4) || !aligned(v_history, 4)))
    return FP8Q_ERR_INVALID_ARGUMENT;
  if (counts && !aligned(counts, 8)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (nsc == 0) return FP8Q_OK;   // no heads: nothing to write
  const size_t need = fp8q_kv_workspace_bytes(tokens, heads, head_dim, g);
  if (!ws || ws_bytes < need || !aligned(ws, 4)) return FP8Q_ERR_WORKSPACE;
  const int64_t h = g == FP8Q_KV_PER_TENSOR ? 1 : heads;
  const int64_t d = g == FP8Q_KV_PER_TENSOR ? row : head_dim;
  return from_cuda(fp8q::launch_quant_delayed(static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
                                              k_codes, v_codes, k_scales, v_scales, 2, tokens, h, d, f, k_history,
                                              v_history, history_len, step, counts, static_cast<float*>(ws),
                                              (cudaStream_t)stream));
}

fp8q_status fp8_gemm_blockscaled(const uint8_t* A, const float* sA, fp8q_granularity gA, const uint8_t* B,
                                 const float* sB, fp8q_granularity gB, int64_t M, int64_t N, int64_t K, void* C,
                                 void* ws, size_t ws_bytes, fp8q_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!(gA == FP8Q_GROUP_1x128 || gA == FP8Q_PER_TENSOR)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!(gB == FP8Q_BLOCK_128x128 || gB == FP8Q_PER_TENSOR)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return FP8Q_OK;
  if (N % 128 != 0 || K % 128 != 0 || K == 0) return FP8Q_ERR_UNSUPPORTED;
  if (checked_elems(M, K) < 0 || checked_elems(N, K) < 0 || checked_elems(M, N) < 0) return FP8Q_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1) return FP8Q_ERR_UNSUPPORTED;
  if (!A || !B || !C || !sA || !sB || !aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(sA, 4) ||
      !aligned(sB, 4))
    return FP8Q_ERR_INVALID_ARGUMENT;
  const size_t need = fp8q::gemm_workspace_bytes(M, N, K);
  if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return FP8Q_ERR_WORKSPACE;
  const cudaError_t e = fp8q::launch_gemm(A, sA, gA, B, false, sB, gB, M, N, K, static_cast<uint16_t*>(C), ws,
                                          ws_bytes, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return FP8Q_ERR_UNSUPPORTED;
  return from_cuda(e);
}

fp8q_status fp8_scale_histogram(const void* scales, int64_t n, fp8q_scale_kind kind, uint32_t* hist,
                                fp8q_stream_t stream) {
  if (n < 0 || !(kind == FP8Q_SCALES_F32 || kind == FP8Q_SCALES_MX)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n > kMaxElems) return FP8Q_ERR_UNSUPPORTED;
  if (n == 0) return FP8Q_OK;
  if (!scales || !hist || !aligned(hist, 4) || (kind == FP8Q_SCALES_F32 && !aligned(scales, 4)))
    return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_scale_histogram(scales, n, kind, hist, (cudaStream_t)stream));
}

fp8q_status fp8_count_underflow(const void* x, const uint8_t* codes, int64_t n, unsigned long long* count,
                                fp8q_stream_t stream) {
  if (n < 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (n > kMaxElems) return FP8Q_ERR_UNSUPPORTED;
  if (n == 0) return FP8Q_OK;
  if (!x || !codes || !count || !aligned(x, 16) || !aligned(codes, 16) || !aligned(count, 8))
    return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_count_underflow(static_cast<const uint16_t*>(x), codes, n, count,
                                                (cudaStream_t)stream));
}

fp8q_status fp8_gemm_blockscaled_to_fp8(const uint8_t* A, const float* sA, fp8q_granularity gA, const uint8_t* B,
                                        const float* sB, fp8q_granularity gB, int64_t M, int64_t N, int64_t K,
                                        uint8_t* codes, float* scales, fp8q_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!(gA == FP8Q_GROUP_1x128 || gA == FP8Q_PER_TENSOR)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!(gB == FP8Q_BLOCK_128x128 || gB == FP8Q_PER_TENSOR)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return FP8Q_OK;
  if (N % 128 != 0 || K % 128 != 0 || K == 0) return FP8Q_ERR_UNSUPPORTED;
  if (checked_elems(M, K) < 0 || checked_elems(N, K) < 0 || checked_elems(M, N) < 0) return FP8Q_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1) return FP8Q_ERR_UNSUPPORTED;
  if (M <= 64) return FP8Q_ERR_UNSUPPORTED;   // decode shapes: the decode kernel has no such epilogue
  if (!A || !B || !codes || !sA || !sB || !scales || !aligned(A, 16) || !aligned(B, 16) || !aligned(codes, 16) ||
      !aligned(sA, 4) || !aligned(sB, 4) || !aligned(scales, 4))
    return FP8Q_ERR_INVALID_ARGUMENT;
  const cudaError_t e = fp8q::launch_gemm_to_fp8(A, sA, gA, B, false, sB, gB, M, N, K, codes, scales,
                                                 (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return FP8Q_ERR_UNSUPPORTED;
  return from_cuda(e);
}

fp8q_status fp8_pack_b_tiles(const uint8_t* B, int64_t N, int64_t K, uint8_t* packed, fp8q_stream_t stream) {
  if (N < 0 || K < 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_UNSUPPORTED;
  if (checked_elems(N, K) < 0) return FP8Q_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return FP8Q_OK;
  if (!B || !packed || !aligned(B, 16) || !aligned(packed, 16) || B == packed) return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_pack_b_tiles(B, N, K, packed, (cudaStream_t)stream));
}

fp8q_status fp8_gemm_blockscaled_packed(const uint8_t* A, const float* sA, fp8q_granularity gA, const uint8_t* Bp,
                                        const float* sB, fp8q_granularity gB, int64_t M, int64_t N, int64_t K,
                                        void* C, void* ws, size_t ws_bytes, fp8q_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!(gA == FP8Q_GROUP_1x128 || gA == FP8Q_PER_TENSOR)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!(gB == FP8Q_BLOCK_128x128 || gB == FP8Q_PER_TENSOR)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return FP8Q_OK;
  if (N % 128 != 0 || K % 128 != 0 || K == 0) return FP8Q_ERR_UNSUPPORTED;
  if (checked_elems(M, K) < 0 || checked_elems(N, K) < 0 || checked_elems(M, N) < 0) return FP8Q_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1) return FP8Q_ERR_UNSUPPORTED;
  if (!A || !Bp || !C || !sA || !sB || !aligned(A, 16) || !aligned(Bp, 16) || !aligned(C, 16) || !aligned(sA, 4) ||
      !aligned(sB, 4))
    return FP8Q_ERR_INVALID_ARGUMENT;
  const size_t need = fp8q::gemm_workspace_bytes(M, N, K);
  if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return FP8Q_ERR_WORKSPACE;
  const cudaError_t e = fp8q::launch_gemm(A, sA, gA, Bp, true, sB, gB, M, N, K, static_cast<uint16_t*>(C), ws,
                                          ws_bytes, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return FP8Q_ERR_UNSUPPORTED;
  return from_cuda(e);
}

fp8q_status fp8_linear_dynamic(const void* X, int64_t M, int64_t N, int64_t K, const uint8_t* B, const float* sB,
                               fp8q_granularity gB, void* C, void* act_ws, size_t act_ws_bytes, void* gemm_ws,
                               size_t gemm_ws_bytes, fp8q_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!(gB == FP8Q_BLOCK_128x128 || gB == FP8Q_PER_TENSOR)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return FP8Q_OK;
  if (N % 128 != 0 || K % 128 != 0 || K == 0) return FP8Q_ERR_UNSUPPORTED;
  if (checked_elems(M, K) < 0 || checked_elems(N, K) < 0 || checked_elems(M, N) < 0) return FP8Q_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1) return FP8Q_ERR_UNSUPPORTED;
  if (!X || !B || !C || !sB || !aligned(X, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(sB, 4))
    return FP8Q_ERR_INVALID_ARGUMENT;
  if (!act_ws || act_ws_bytes < fp8q::linear_act_workspace_bytes(M, K) || !aligned(act_ws, 16))
    return FP8Q_ERR_WORKSPACE;
  const size_t need = fp8q::gemm_workspace_bytes(M, N, K);
  if (need > 0 && (!gemm_ws || gemm_ws_bytes < need || !aligned(gemm_ws, 16))) return FP8Q_ERR_WORKSPACE;
  const cudaError_t e = fp8q::launch_linear(static_cast<const uint16_t*>(X), B, sB, gB, M, N, K,
                                            static_cast<uint16_t*>(C), act_ws, gemm_ws, gemm_ws_bytes,
                                            (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return FP8Q_ERR_UNSUPPORTED;
  return from_cuda(e);
}

size_t fp8q_linear_fused_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 64 || K <= 0 || K % 128 != 0 || checked_elems(M, K) < 0) return 0;
  return fp8q::linear_fused_workspace_bytes(M, K);
}

fp8q_status fp8_linear_dynamic_fused(const void* X, int64_t M, int64_t N, int64_t K, const uint8_t* B, const float* sB,
                                     fp8q_granularity gB, void* C, void* act_ws, size_t act_ws_bytes,
                                     fp8q_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_INVALID_ARGUMENT;
  if (!(gB == FP8Q_BLOCK_128x128 || gB == FP8Q_PER_TENSOR)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return FP8Q_OK;
  if (M <= 64) return FP8Q_ERR_UNSUPPORTED;   // decode shapes: fp8_linear_dynamic
  if (N % 128 != 0 || K % 128 != 0 || K == 0) return FP8Q_ERR_UNSUPPORTED;
  if (checked_elems(M, K) < 0 || checked_elems(N, K) < 0 || checked_elems(M, N) < 0) return FP8Q_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1) return FP8Q_ERR_UNSUPPORTED;
  if (!X || !B || !C || !sB || !aligned(X, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(sB, 4))
    return FP8Q_ERR_INVALID_ARGUMENT;
  if (!act_ws || act_ws_bytes < fp8q::linear_fused_workspace_bytes(M, K) || !aligned(act_ws, 256))
    return FP8Q_ERR_WORKSPACE;
  const cudaError_t e = fp8q::launch_linear_fused(static_cast<const uint16_t*>(X), B, sB, gB, M, N, K,
                                                  static_cast<uint16_t*>(C), act_ws, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported || e == cudaErrorCooperativeLaunchTooLarge) return FP8Q_ERR_UNSUPPORTED;
  return from_cuda(e);
}

fp8q_status fp8_gemm_mx(const uint8_t* A, const uint8_t* sA, fp8q_format fa, const uint8_t* B, const uint8_t* sB,
                        fp8q_format fb, int64_t M, int64_t N, int64_t K, void* C, fp8q_stream_t stream) {
  if (M < 0 || N < 0 || K < 0 || !valid_fmt(fa) || !valid_fmt(fb)) return FP8Q_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return FP8Q_OK;
  if (N % 128 != 0 || K % 128 != 0 || K == 0) return FP8Q_ERR_UNSUPPORTED;
  if (checked_elems(M, K) < 0 || checked_elems(N, K) < 0 || checked_elems(M, N) < 0) return FP8Q_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1) return FP8Q_ERR_UNSUPPORTED;
  if (!A || !B || !C || !sA || !sB || !aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(sA, 16) ||
      !aligned(sB, 16))
    return FP8Q_ERR_INVALID_ARGUMENT;
  return from_cuda(fp8q::launch_gemm_mx(A, sA, fa, B, sB, fb, M, N, K, static_cast<uint16_t*>(C),
                                        (cudaStream_t)stream));
}

}  // extern "C"
