/*
 * fp8q — FP8 (E4M3 / E5M2) scaled quantization, dequantization, KV-cache
 * quantization and block-scaled FP8 GEMM on NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every pointer argument named as a tensor is a DEVICE pointer owned
 * by the caller; the library allocates no memory.  Every compute call is
 * asynchronous on the caller's stream (NULL = the legacy default stream) and
 * never synchronizes the host.  Argument errors are reported before anything
 * is launched; a launch failure returns FP8Q_ERR_CUDA; faults inside a kernel
 * surface at the caller's next synchronization.  No C++ exception crosses
 * this interface.
 *
 * Method (web pages the definitions come from, cited by title and section):
 *   [W] wangyu.me, "大语言模型量化技术（五）：FP8" — format table and step
 *       sizes ("FP8 是什么"); quantization steps s = amax/448, x/s, round to
 *       nearest, saturate ("什么是 FP8 量化"); 128x128 weight blocks and the
 *       weight_scale_inv layout ("权重量化：128x128 分块 FP8"); dynamic
 *       per-token / per-128-group activation scales and the GEMM identity
 *       ("激活动态量化"); fp32 accumulation with scales applied on
 *       accumulation ("FP8 矩阵乘").
 *   [C] charles2530.github.io, "量化：FP8 与混合精度推理" — x_fp8 =
 *       FP8Cast(x/s), x_hat = s * x_fp8.
 *   [P] pwwt.cn, "从权重到激活：FP8 量化到底动了哪些东西" — separate K and V
 *       scales, per-head keys (section 1); per-head x per-128-token KV blocks
 *       (section 3).
 *   [M] api.makesence.top, "LLM推理量化:FP8 versus INT8" — W8A8 E4M3 with
 *       an E5M2 KV cache (section 二).
 *
 * Arithmetic, per scale group G (bit-exact contract):
 *   amax = max over G of |x|        (x is bf16, widened exactly to fp32;
 *                                    a NaN anywhere in G makes amax NaN)
 *   s    = amax / FMAX              (one IEEE fp32 division; FMAX = 448 for
 *                                    E4M3, 57344 for E5M2; stored as the
 *                                    group's fp32 scale, a dequant multiplier)
 *   code = FP8_RNE_SAT(x / s)       (the quotient is the IEEE fp32
 *                                    round-to-nearest-even quotient; it is
 *                                    then rounded to nearest-even on the FP8
 *                                    grid, subnormals included, saturating to
 *                                    +-FMAX; Inf saturates too)
 *   amax == 0 gives s = 0 and signed-zero codes (no division).
 *   dequant: y = bf16_rne( fp32( decode(code) * s ) ).
 *
 * Layouts (row-major, contiguous):
 *   tensors, codes, outputs   [rows][cols]
 *   FP8Q_PER_TENSOR scales    [1]
 *   FP8Q_GROUP_1x128 scales   [ceil(cols/128)][rows]   (group-major: the 128
 *                             row scales of one K-block are contiguous)
 *   FP8Q_BLOCK_128x128 scales [ceil(rows/128)][ceil(cols/128)]
 *                             (the weight_scale_inv layout of [W])
 *   KV caches                 [tokens][heads][head_dim]
 *   KV scales                 per-tensor [1]; per-head [heads];
 *                             per-head x 128-token [ceil(tokens/128)][heads]
 *   GEMM                      C[M][N] = A[M][K] . B[N][K]^T, A and B K-major.
 *
 * Alignment: tensor, code and output pointers 16-byte aligned; scale
 * pointers 4-byte aligned; cols (and head_dim) a multiple of 8.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8Q_API __attribute__((visibility("default")))
#else
#define FP8Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so this header needs no CUDA headers. */
typedef struct CUstream_st *fp8q_stream_t;

typedef enum {
    FP8Q_OK = 0,
    FP8Q_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, misalignment, bad enum  */
    FP8Q_ERR_UNSUPPORTED = 2,      /* valid request outside what this build implements     */
    FP8Q_ERR_WORKSPACE = 3,        /* workspace missing or smaller than *_workspace_bytes() */
    FP8Q_ERR_CUDA = 4              /* a CUDA call or launch failed                          */
} fp8q_status;

typedef enum { FP8Q_E4M3 = 0, FP8Q_E5M2 = 1 } fp8q_format;

typedef enum {
    FP8Q_PER_TENSOR = 0,    /* one scale for the whole tensor                             */
    FP8Q_GROUP_1x128 = 1,   /* one scale per row and 128 consecutive columns ([W] 激活动态量化) */
    FP8Q_BLOCK_128x128 = 2  /* one scale per 128x128 block ([W] 权重量化)                  */
} fp8q_granularity;

typedef enum {
    FP8Q_KV_PER_TENSOR = 0,      /* one scale for K, one for V ([M] section 二)           */
    FP8Q_KV_PER_HEAD = 1,        /* one scale per head, separately for K and V ([P] 1)    */
    FP8Q_KV_PER_HEAD_TOK128 = 2  /* one per head and 128-token block ([P] section 3)       */
} fp8q_kv_granularity;

/* Human-readable name of a status code (static storage; never NULL). */
FP8Q_API const char *fp8q_status_string(fp8q_status status);

/* Library version as major*10000 + minor*100 + patch. */
FP8Q_API int fp8q_version(void);

/*
 * Synchronizes the current device, returns the library's device error bits and clears them.
 * 0: no error.  Bit 0: a bounded wait inside a kernel (a pipeline barrier that never completed)
 * gave up after its time limit, so that kernel's outputs are incomplete.  Bit 1: a GEMM
 * workspace was not zero-filled (see fp8_gemm_blockscaled), so some output tiles were not
 * written.  0xFFFFFFFF: the device could not be queried (e.g. an earlier fault).
 */
FP8Q_API uint32_t fp8q_device_status(void);

/*
 * Failure-detection self-test: launches one block whose thread waits, through the same bounded
 * wait every kernel of the library uses, on a pipeline barrier that nothing ever completes.
 * After the time limit (2 s) the wait gives up, sets bit 0 of the device error bits and the
 * kernel returns normally (no trap, no fault; the context stays usable).  A following
 * fp8q_device_status() therefore returns bit 0 set.  Asynchronous on `stream`.
 */
FP8Q_API fp8q_status fp8q_selftest_wait_timeout(fp8q_stream_t stream);

/*
 * Host-only self-check of the decode GEMM's work split (no device work, no GPU needed): for the
 * plan fp8_gemm_blockscaled uses for a decode shape (M <= 64) on a device with `sms` SMs, walks
 * every CTA's contiguous range of (weight tile, K block) units with the kernel's own range
 * functions and checks what its split-tile hand-off relies on: each CTA holds at most one
 * segment of a tile a lower CTA started (its first segment) and at most one of a tile it starts
 * but a higher CTA ends (its last); the promotion warps and the bookkeeping warp pick out the same
 * segments; every shared tile has exactly one starting CTA (its lowest, which finishes it or
 * publishes its own partial) and c_last - c_first later contributors; every partial slot, the
 * starting CTA's included, lies inside the workspace.  Returns 0 when all hold,
 * a positive code naming the first violation, or -1 for a shape that is not a decode shape.
 */
FP8Q_API int fp8q_check_decode_split(int64_t M, int64_t N, int64_t K, int sms);

/*
 * Host-only self-check of the prefill GEMMs' persistent tile walk (no device work): for an
 * M x N x K product with M > 64 (128 x 256 output tiles, in the block-scaled, per-tensor and
 * MXFP8 kernels alike) walks tile indices 0 .. tiles-1 through the kernels' own walk function
 * (bands of M tiles when A does not fit in L2) and checks that every output tile is visited
 * exactly once and that every coordinate lies inside the matrix.  Returns 0 when it
 * holds, a positive code for the first violation, or -1 for a shape that is not a prefill shape.
 */
FP8Q_API int fp8q_check_tile_walk(int64_t M, int64_t N, int64_t K);

/* ---------------------------------------------------------------- sizes */

/* Number of fp32 scales fp8_quantize writes for a [rows][cols] tensor; 0 on a bad argument. */
FP8Q_API size_t fp8q_num_scales(int64_t rows, int64_t cols, fp8q_granularity g);

/* Device workspace bytes fp8_quantize needs (per-tensor partial maxima; 0 for one-pass granularities). */
FP8Q_API size_t fp8q_workspace_bytes(int64_t rows, int64_t cols, fp8q_granularity g);

/* Number of fp32 scales fp8_kv_quantize writes into EACH of k_scales and v_scales. */
FP8Q_API size_t fp8q_kv_num_scales(int64_t tokens, int64_t heads, fp8q_kv_granularity g);

/* Device workspace bytes fp8_kv_quantize needs (0 for the one-pass per-head x 128-token case). */
FP8Q_API size_t fp8q_kv_workspace_bytes(int64_t tokens, int64_t heads, int64_t head_dim, fp8q_kv_granularity g);

/* Device workspace bytes fp8_gemm_blockscaled needs for this shape (0 when none is needed). */
FP8Q_API size_t fp8q_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* ---------------------------------------------------------------- codec */

/*
 * Element-wise FP8 encode: codes[i] = FP8_RNE_SAT(q[i]) ([W] "FP8 是什么": round to
 * the nearest representable value, ties to even, out-of-range values saturate to
 * +-max; NaN stays NaN).  q: fp32 [n]; codes: uint8 [n].  Both 16-byte aligned.
 * n == 0 is a no-op.
 */
FP8Q_API fp8q_status fp8_encode(const float *q, int64_t n, fp8q_format f, uint8_t *codes, fp8q_stream_t stream);

/*
 * Element-wise FP8 decode to the exact fp32 value ([W] format table).  codes: uint8 [n];
 * out: fp32 [n].  Both 16-byte aligned.  E4M3 has no Inf; S.1111.111 decodes to NaN.
 */
FP8Q_API fp8q_status fp8_decode(const uint8_t *codes, int64_t n, fp8q_format f, float *out, fp8q_stream_t stream);

/* ---------------------------------------------------------------- quantize */

/*
 * Scaled FP8 quantization of one bf16 tensor ([W] "什么是 FP8 量化", "权重量化",
 * "激活动态量化"; [C] x_fp8 = FP8Cast(x/s)).
 *   x       bf16 [rows][cols] (device)
 *   codes   uint8 [rows][cols] (device, written)
 *   scales  fp32, fp8q_num_scales(rows, cols, g) entries in the layout above (device, written)
 *   ws      device workspace of at least fp8q_workspace_bytes(rows, cols, g) bytes
 *           (may be NULL when that is 0); its contents need no initialisation
 * Per-tensor runs two kernels (the whole tensor's amax must be known before any
 * element is cast); the 1x128 and 128x128 granularities run one fused kernel.
 * rows == 0 or cols == 0 writes nothing, except that a per-tensor call writes s = 0.
 */
FP8Q_API fp8q_status fp8_quantize(const void *x, int64_t rows, int64_t cols, fp8q_format f, fp8q_granularity g,
                         uint8_t *codes, float *scales, void *ws, size_t ws_bytes, fp8q_stream_t stream);

/*
 * Dequantization x_hat = s * x_fp8 ([C]; [W] "什么是 FP8 量化", restore x ~ x_hat * s),
 * computed as y = bf16_rne(fp32(decode(code) * s)).
 *   codes   uint8 [rows][cols] (device);  scales as written by fp8_quantize (device)
 *   y       bf16 [rows][cols] (device, written)
 */
FP8Q_API fp8q_status fp8_dequantize(const uint8_t *codes, const float *scales, int64_t rows, int64_t cols,
                           fp8q_format f, fp8q_granularity g, void *y, fp8q_stream_t stream);

/*
 * KV-cache quantization with separate K and V scales ([P] sections 1 and 3; [M] 二).
 *   k, v                 bf16 [tokens][heads][head_dim] (device); head_dim % 8 == 0, head_dim <= 256
 *   k_codes, v_codes     uint8, same shape (device, written)
 *   k_scales, v_scales   fp32, fp8q_kv_num_scales(tokens, heads, g) entries each (device, written)
 *   ws                   at least fp8q_kv_workspace_bytes(...) bytes (device), may be NULL when 0
 * Per-tensor and per-head run two kernels; per-head x 128-token runs one.
 */
FP8Q_API fp8q_status fp8_kv_quantize(const void *k, const void *v, int64_t tokens, int64_t heads, int64_t head_dim,
                            fp8q_format f, fp8q_kv_granularity g, uint8_t *k_codes, uint8_t *v_codes,
                            float *k_scales, float *v_scales, void *ws, size_t ws_bytes,
                            fp8q_stream_t stream);

/*
 * fp8_kv_quantize without a workspace, for callers that cannot allocate device memory (an
 * engine that owns all device memory up front, a latency-critical path where an allocation may
 * stall or fail, a plug-in that receives tensors but has no way to request scratch).  The
 * source pages have no counterpart to this entry point: it is a deployment convenience.
 * Arguments, layouts and results are exactly those of fp8_kv_quantize without ws / ws_bytes.
 * The partial maxima of the two-pass granularities live in a fixed 256 KB array inside the
 * library, one per device that loads it, kept until the process exits; per-head quantization
 * therefore supports at most 32 heads (more returns FP8Q_ERR_WORKSPACE).  The first call on a
 * device looks up that array's device address (cudaGetSymbolAddress) with the device current,
 * so make that first call before any stream capture.  All calls share the array: calls whose
 * kernels can overlap on the GPU (e.g. on unordered streams) race on it and must not be made.
 */
FP8Q_API fp8q_status fp8_kv_quantize_noalloc(const void *k, const void *v, int64_t tokens, int64_t heads,
                                             int64_t head_dim, fp8q_format f, fp8q_kv_granularity g,
                                             uint8_t *k_codes, uint8_t *v_codes, float *k_scales,
                                             float *v_scales, fp8q_stream_t stream);

/*
 * Several tensors in one launch ([W] "权重量化：128x128 分块 FP8" and "激活动态量化": e.g. a
 * layer's weight blocks and its activations).  Each entry is quantized exactly as fp8_quantize
 * with its granularity would (same codes, same scales, same layouts); one persistent kernel
 * walks the 128 x 128 boxes of all entries, so the launch overhead, ramp and tail are paid once.
 *   tensors  host array of n entries (1 <= n <= 8); each: x bf16 [rows][cols] (device, 16-byte
 *            aligned, cols % 8 == 0), granularity FP8Q_GROUP_1x128 or FP8Q_BLOCK_128x128
 *            (FP8Q_PER_TENSOR needs two passes: FP8Q_ERR_UNSUPPORTED), codes uint8
 *            [rows][cols] (16-byte aligned), scales fp32, fp8q_num_scales(rows, cols, g)
 *            entries (4-byte aligned).  Entries must not overlap one another's outputs.
 *   f        one format for all entries
 * The array is read during the call only.
 */
typedef struct {
  const void *x;
  int64_t rows, cols;
  fp8q_granularity g;
  uint8_t *codes;
  float *scales;
} fp8q_quant_tensor;
FP8Q_API fp8q_status fp8_quantize_many(const fp8q_quant_tensor *tensors, int n, fp8q_format f,
                                       fp8q_stream_t stream);

/* ---------------------------------------------------------------- MXFP8 */

/*
 * MXFP8 quantization: block scaling with blocks of 32 ([M] section on Microscaling, block
 * size 32).  The scale of each 1x32 group of a row is a power of two 2^k, the smallest with
 * amax <= FMAX * 2^k (the pages' rule s = amax / FMAX restricted to powers of two: no element
 * saturates), stored as the byte k + 127 (k clamped at -127; 255 marks a NaN or infinite amax);
 * codes = FP8(RN(x / 2^k)).
 *   x       bf16 [rows][cols] (device, 16-byte aligned), cols % 32 == 0
 *   codes   uint8 [rows][cols] (device, written)
 *   scales  uint8 [rows][cols / 32] (device, written)
 */
FP8Q_API fp8q_status fp8_quantize_mx(const void *x, int64_t rows, int64_t cols, fp8q_format f, uint8_t *codes,
                                     uint8_t *scales, fp8q_stream_t stream);

/*
 * The same quantization with the scales written in the BLOCKED layout that fp8_gemm_mx reads
 * (the tensor cores' block-scaled MMA takes one 512-byte chunk per 128 rows x 128 columns):
 *   chunk (rb, cb) = rows [128 rb, 128 rb + 128) x columns [128 cb, 128 cb + 128) starts at byte
 *   512 * (rb * ceil(cols / 128) + cb); inside it the scale of row r and 32-column group j
 *   (j = 0..3 within the chunk) sits at byte 16 * (r % 32) + 4 * ((r % 128) / 32) + j.
 * Rows past `rows` and groups past cols / 32 in the last chunks are written as 0.
 *   scales  uint8, fp8q_mx_blocked_scale_bytes(rows, cols) bytes (device, written)
 * Other arguments and the codes as fp8_quantize_mx.
 */
FP8Q_API size_t fp8q_mx_blocked_scale_bytes(int64_t rows, int64_t cols);
FP8Q_API fp8q_status fp8_quantize_mx_blocked(const void *x, int64_t rows, int64_t cols, fp8q_format f,
                                             uint8_t *codes, uint8_t *scales, fp8q_stream_t stream);

/* y = bf16_rne(fp32(decode(code) * 2^(scale - 127))), layouts as fp8_quantize_mx. */
FP8Q_API fp8q_status fp8_dequantize_mx(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                                       fp8q_format f, void *y, fp8q_stream_t stream);

/* ---------------------------------------------------------------- delayed scaling */

/*
 * Per-tensor quantization with delayed scaling ([C] "scale 是控制面": the scale follows a
 * history of amax values instead of the tensor being cast; [M] 二: the forward pass takes its
 * scale factor from the previous micro-batch's max), with the overflow / underflow counts
 * that section asks to be observable.
 *   x             bf16 [rows][cols] (device); cols % 8 == 0
 *   amax_history  fp32 [history_len] (device, read and written): amax values of earlier calls,
 *                 zero-filled by the caller before step 0; entries must be >= 0 or NaN
 *   step          this call's index, 0, 1, 2, ...: step 0 scales from x's own amax (two
 *                 kernels, as fp8_quantize per-tensor); step t >= 1 uses
 *                 s = RN(max(amax_history) / FMAX) and reads x once.  An all-zero history gives
 *                 s = 0 and sign-only codes.  Afterwards amax_history[step % history_len] holds
 *                 x's own amax.
 *   codes         uint8 [rows][cols] (device, written);  scale: fp32 [1] (device, written)
 *   counts        NULL, or uint64 [2] (device, 8-byte aligned) to which the call adds the
 *                 number of elements that saturated (|x / s| rounds above FMAX: E4M3 > 464,
 *                 E5M2 >= 61440) and of nonzero elements whose code is +-0
 *   ws            at least fp8q_workspace_bytes(rows, cols, FP8Q_PER_TENSOR) bytes (device)
 * history_len in 1 .. 2^20.  Calls that share a history must be ordered (one stream).
 */
FP8Q_API fp8q_status fp8_quantize_delayed(const void *x, int64_t rows, int64_t cols, fp8q_format f,
                                          float *amax_history, int64_t history_len, int64_t step,
                                          uint8_t *codes, float *scale, unsigned long long *counts,
                                          void *ws, size_t ws_bytes, fp8q_stream_t stream);

/*
 * KV-cache quantization with delayed scaling, per tensor or per head (the two-pass
 * granularities; per-head x 128-token is one pass already and returns FP8Q_ERR_UNSUPPORTED).
 * Arguments as fp8_kv_quantize, plus histories as for fp8_quantize_delayed, one per tensor:
 *   k_history, v_history   fp32 [history_len][heads] (per head) or [history_len] (per tensor)
 *   counts                 NULL or uint64 [2], K and V together
 *   ws                     at least fp8q_kv_workspace_bytes(tokens, heads, head_dim, g) bytes
 * With step >= 1 the cache is read once (3 B per element instead of 5).
 */
FP8Q_API fp8q_status fp8_kv_quantize_delayed(const void *k, const void *v, int64_t tokens, int64_t heads,
                                             int64_t head_dim, fp8q_format f, fp8q_kv_granularity g,
                                             float *k_history, float *v_history, int64_t history_len,
                                             int64_t step, uint8_t *k_codes, uint8_t *v_codes,
                                             float *k_scales, float *v_scales, unsigned long long *counts,
                                             void *ws, size_t ws_bytes, fp8q_stream_t stream);

/* ---------------------------------------------------------------- GEMM */

/*
 * Block-scaled FP8 GEMM ([W] "激活动态量化", "FP8 矩阵乘"):
 *   C[m][n] = bf16_rne( sum_kb sA(m,kb) * sB(n,kb) * P_kb[m][n] ),
 *   P_kb[m][n] = sum over k in K-block kb (128 wide) of decode(A[m][k]) * decode(B[n][k]),
 * with P_kb from the FP8 tensor cores and all accumulation in fp32.
 *   A   E4M3 codes [M][K] (K-major);  sA: gA = FP8Q_GROUP_1x128 ([K/128][M]) or FP8Q_PER_TENSOR ([1])
 *   B   E4M3 codes [N][K] (K-major, W in R^{N x K});
 *       sB: gB = FP8Q_BLOCK_128x128 ([N/128][K/128]) or FP8Q_PER_TENSOR ([1])
 *   C   bf16 [M][N] (device, written)
 * When both are per-tensor and M > 64 the product is accumulated over all of K and
 * scaled once at the end: C = bf16(sA * sB * sum_k a*b).
 * Decode shapes (M <= 64) split the (128-row weight tile, K block) pairs evenly over the SMs;
 * per-tensor scales are then applied per K block.  A tile shared by several SMs has its fp32
 * partial sums added in a fixed order, so results are deterministic.  No block waits for
 * another (the last contributor to count in finishes a shared tile), so the call completes and
 * is correct however many of its blocks the device runs at once (other streams' kernels, MPS
 * or a partitioned device taking SMs make it slower, not wrong).  ws: caller-owned device
 * memory of at least fp8q_gemm_workspace_bytes(M, N, K) bytes, 16-byte aligned (else
 * FP8Q_ERR_WORKSPACE).  Its first 65536 bytes hold per-tile counters and must be ZERO-FILLED
 * before its first use; every call that runs to completion leaves them zero again, so the
 * workspace can be reused as is, by calls of any shape (the rest is scratch that each call
 * writes before reading).  After a device error (fp8q_device_status() != 0) zero the counters
 * again.  The size is 0 (ws may be NULL) when each block of the call holds whole weight tiles
 * (the 8B shapes on a full B200) and for M > 64; decode shapes with more than 16384 weight
 * tiles (N > 2,097,152) run on the prefill kernel and need none either.  Calls that may run concurrently (e.g. on
 * unordered streams) need separate workspaces.  Detection of a workspace that was not zero is
 * best effort: a tile counter at or above the tile's number of contributors raises device error
 * bit 1 and leaves that tile unwritten; a smaller stale count may go unseen and leave the tile
 * summed from incomplete partials.  The call completes either way.
 * Requirements: M >= 1; N % 128 == 0; K % 128 == 0 (else FP8Q_ERR_UNSUPPORTED);
 * A, B, C 16-byte aligned.  ws may be NULL when fp8q_gemm_workspace_bytes() is 0.
 */
FP8Q_API fp8q_status fp8_gemm_blockscaled(const uint8_t *A, const float *sA, fp8q_granularity gA,
                                 const uint8_t *B, const float *sB, fp8q_granularity gB,
                                 int64_t M, int64_t N, int64_t K, void *C,
                                 void *ws, size_t ws_bytes, fp8q_stream_t stream);

/* ---------------------------------------------------------------- scale health */

/*
 * Observability of the scales and of the values they lose ([C] "scale 是控制面": scales,
 * overflow and underflow should be observable; saturation counts come with the delayed-scaling
 * calls, the only path where a value can exceed the scale's range).
 *
 * fp8_scale_histogram adds to hist[256] (uint32, device) a histogram of n scales by power of
 * two: FP8Q_SCALES_F32 takes fp32 scales (4-byte aligned) and counts each in the bucket of its
 * biased exponent field (bucket e holds scales in [2^(e-127), 2^(e-126)); 0: zero or subnormal;
 * 255: Inf or NaN), so amax = s * FMAX lies in a known octave; FP8Q_SCALES_MX takes MX scale
 * bytes and counts each by value (the biased exponent itself).  Any layout works: scales are
 * counted, not located.
 *
 * fp8_count_underflow adds to *count (uint64, device, 8-byte aligned) the number of elements of
 * x (bf16 [n], 16-byte aligned) that are nonzero and not NaN while their code (uint8 [n],
 * 16-byte aligned, any format) is +-0: values the quantization flushed to zero.
 */
typedef enum { FP8Q_SCALES_F32 = 0, FP8Q_SCALES_MX = 1 } fp8q_scale_kind;
FP8Q_API fp8q_status fp8_scale_histogram(const void *scales, int64_t n, fp8q_scale_kind kind, uint32_t *hist,
                                         fp8q_stream_t stream);
FP8Q_API fp8q_status fp8_count_underflow(const void *x, const uint8_t *codes, int64_t n,
                                         unsigned long long *count, fp8q_stream_t stream);

/*
 * The block-scaled GEMM with its output quantized for the next layer ([W] "激活动态量化": the
 * next GEMM's activations in 1x128 groups): the epilogue rounds each output to bf16, as
 * fp8_gemm_blockscaled stores it, and quantizes every 1x128 group of C to E4M3 in place of the
 * bf16 store, so C never round-trips through memory.  codes and scales are bit-identical to
 * fp8_gemm_blockscaled followed by fp8_quantize(C, FP8Q_E4M3, FP8Q_GROUP_1x128).
 *   A, sA, gA, B, sB, gB, M, N, K  as fp8_gemm_blockscaled
 *   codes   uint8 [M][N] (device, 16-byte aligned, written)
 *   scales  fp32 [N/128][M] (device, written): the 1x128 layout of fp8_quantize
 * Prefill shapes only: M must exceed 64 (decode shapes, M <= 64, return FP8Q_ERR_UNSUPPORTED:
 * quantize their bf16 output with fp8_quantize).  No workspace.
 */
FP8Q_API fp8q_status fp8_gemm_blockscaled_to_fp8(const uint8_t *A, const float *sA, fp8q_granularity gA,
                                                 const uint8_t *B, const float *sB, fp8q_granularity gB,
                                                 int64_t M, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                                 fp8q_stream_t stream);

/*
 * Packed weight tiles for the GEMMs.  Repacks B codes [N][K] (row-major, K-major rows) so
 * that each 128 x 128 tile is one contiguous 16384-byte block: tile (nb, kb) = rows
 * [128 nb, +128) x columns [128 kb, +128) starts at byte 16384 * (nb * K/128 + kb); inside it
 * row r occupies bytes [128 r, 128 r + 128) with its eight 16-byte pieces in swizzled order
 * (piece j at position j XOR (r % 8)).  This is the shared-memory image the tensor cores read,
 * so the GEMMs fetch a tile with one bulk copy instead of 128 row requests (decode shapes
 * stream the weights at the DRAM rate).  A one-time step per weight, like the quantization.
 *   B       uint8 [N][K] codes (device, 16-byte aligned);  packed: N * K bytes (device, written,
 *           16-byte aligned, not overlapping B)
 * Requirements: N % 128 == 0, K % 128 == 0 (else FP8Q_ERR_UNSUPPORTED).
 */
FP8Q_API fp8q_status fp8_pack_b_tiles(const uint8_t *B, int64_t N, int64_t K, uint8_t *packed,
                                      fp8q_stream_t stream);

/*
 * fp8_gemm_blockscaled with B given as packed tiles (fp8_pack_b_tiles): the same product, the
 * same scales, workspace rules and requirements; the results are identical to
 * fp8_gemm_blockscaled on the unpacked codes.
 */
FP8Q_API fp8q_status fp8_gemm_blockscaled_packed(const uint8_t *A, const float *sA, fp8q_granularity gA,
                                                 const uint8_t *Bp, const float *sB, fp8q_granularity gB,
                                                 int64_t M, int64_t N, int64_t K, void *C,
                                                 void *ws, size_t ws_bytes, fp8q_stream_t stream);

/*
 * Linear layer with dynamic activation quantization ([W] "激活动态量化": per-token 1x128
 * groups computed at run time, then "FP8 矩阵乘"):
 *   C = fp8_gemm_blockscaled(codes, scales, FP8Q_GROUP_1x128, B, sB, gB)  with
 *   (codes, scales) = fp8_quantize(X, E4M3, FP8Q_GROUP_1x128),
 * bit-identical to those two calls, issued as two programmatic-dependent launches on `stream`
 * (for decode shapes the codes stay in L2 between them).
 *   X        bf16 [M][K] (device, K-major);  B, sB, gB, C as for fp8_gemm_blockscaled
 *   act_ws   device, 16-byte aligned, at least fp8q_linear_act_workspace_bytes(M, K) bytes:
 *            receives the activation codes and scales; needs no initialisation
 *   gemm_ws  the GEMM's workspace, fp8q_gemm_workspace_bytes(M, N, K) bytes (may be NULL
 *            when that is 0), under the zero-fill rule stated for fp8_gemm_blockscaled
 * Requirements as for fp8_gemm_blockscaled: N % 128 == 0, K % 128 == 0.
 */
FP8Q_API size_t fp8q_linear_act_workspace_bytes(int64_t M, int64_t K);

/*
 * The same linear layer at prefill shapes (M > 64; decode shapes return FP8Q_ERR_UNSUPPORTED) as
 * ONE cooperative launch: the block-scaled GEMM kernel first quantizes X into act_ws (every
 * warp of the grid takes a share of the 1x128 groups, with the stand-alone quantizer's
 * arithmetic), all blocks meet at a grid barrier, and the GEMM then reads the codes back, from
 * L2 where they fit.  Output bit-identical to fp8_linear_dynamic.  The pages describe the quantizer and the
 * GEMM as two steps ([W] "激活动态量化", "FP8 矩阵乘"); this is the fused form of the two.
 *   act_ws   device, 256-byte aligned, at least fp8q_linear_fused_workspace_bytes(M, K) bytes:
 *            two grid-barrier words (an arrival count and a generation) in its first 256 bytes,
 *            then the codes [M][K] (rows of K bytes, the block padded to a multiple of 256
 *            bytes), then the fp32 scales [K/128][M].  The first 256 bytes must be ZERO-FILLED
 *            before the first use; every call that completes leaves the arrival count at zero,
 *            so the buffer is reused as is, by calls of any shape it is large enough for.  After
 *            a device error zero them again.  Calls sharing one act_ws must not overlap.
 * Needs every SM free for the grid (a cooperative launch): FP8Q_ERR_UNSUPPORTED when the device
 * cannot hold the grid at once.  On the measured prefill shapes this form is slower than
 * fp8_linear_dynamic (its quantize phase runs at the GEMM kernel's occupancy, one block of twelve
 * warps per SM), which remains the faster call.
 */
FP8Q_API size_t fp8q_linear_fused_workspace_bytes(int64_t M, int64_t K);
FP8Q_API fp8q_status fp8_linear_dynamic_fused(const void *X, int64_t M, int64_t N, int64_t K, const uint8_t *B,
                                              const float *sB, fp8q_granularity gB, void *C, void *act_ws,
                                              size_t act_ws_bytes, fp8q_stream_t stream);
FP8Q_API fp8q_status fp8_linear_dynamic(const void *X, int64_t M, int64_t N, int64_t K, const uint8_t *B,
                                        const float *sB, fp8q_granularity gB, void *C, void *act_ws,
                                        size_t act_ws_bytes, void *gemm_ws, size_t gemm_ws_bytes,
                                        fp8q_stream_t stream);

/*
 * MXFP8 GEMM on the tensor cores' native block-scaled MMA ([M] section on Microscaling: blocks
 * of 32 with power-of-two scales, native on Blackwell; [W] "FP8 矩阵乘": FP8 products, fp32
 * accumulation):
 *   C[m][n] = bf16_rne( sum_k decode(A[m][k]) 2^(sA(m,k/32) - 127) * decode(B[n][k]) 2^(sB(n,k/32) - 127) )
 * The tensor core applies the scales inside each MMA, so all of K accumulates in fp32 without
 * a promotion step.
 *   A    uint8 codes [M][K] in format fa (device, K-major), e.g. fp8_quantize_mx_blocked(X)
 *   sA   blocked scales of A: fp8q_mx_blocked_scale_bytes(M, K) bytes (device)
 *   B    uint8 codes [N][K] in format fb (W in R^{N x K}); sB: fp8q_mx_blocked_scale_bytes(N, K)
 *   C    bf16 [M][N] (device, written)
 * E4M3 and E5M2 mix freely (fa, fb).  A scale byte of 255 (NaN) gives NaN in the outputs it
 * touches.  Requirements: M >= 1; N % 128 == 0; K % 128 == 0 (else FP8Q_ERR_UNSUPPORTED);
 * A, B, C, sA, sB 16-byte aligned.  No workspace.
 */
FP8Q_API fp8q_status fp8_gemm_mx(const uint8_t *A, const uint8_t *sA, fp8q_format fa, const uint8_t *B,
                                 const uint8_t *sB, fp8q_format fb, int64_t M, int64_t N, int64_t K, void *C,
                                 fp8q_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
