/*
 * CPU oracle for FP8 (E4M3 / E5M2) scaled quantization, dequantization,
 * KV-cache quantization and the block-scaled FP8 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the GPU library computes.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header, table or constant generator with the CUDA path.
 *
 * Sources (web pages; cited by title and section):
 *   [W]  wangyu.me, "大语言模型量化技术（五）：FP8" (LLM quantization V: FP8)
 *        - "FP8 是什么": format table (sign/exponent/mantissa, max, min normal,
 *          min subnormal), relative step sizes, E4M3 saturates to +-448.
 *        - "什么是 FP8 量化": steps: s = max|x|/448, divide by s, round to the
 *          nearest E4M3 value, saturate, keep codes and s, restore x ~ x_hat*s.
 *        - "FP8 与 INT8 量化精度对比": worked example s = 10/448.
 *        - "权重量化：128x128 分块 FP8": per-block amax, s_i = a_i/448, cast of
 *          W/s_i with round-to-nearest ties-to-even and saturation, fp32 scale,
 *          scale tensor of shape ceil(N/128) x ceil(K/128) (weight_scale_inv).
 *        - "激活动态量化": per-token amax/448, optionally per 128-group along K;
 *          the GEMM identity y ~ s_x sum_j s_w,j (x_hat^(j) W_hat^(j)).
 *        - "FP8 矩阵乘": fp32 accumulation of FP8 block products, scales
 *          multiplied back on accumulation.
 *   [C]  charles2530.github.io, "量化：FP8 与混合精度推理", section
 *        "E4M3 和 E5M2 是范围与格点的取舍": x_fp8 = FP8Cast(x/s), x_hat = s*x_fp8.
 *   [P]  pwwt.cn, "从权重到激活：FP8 量化到底动了哪些东西", section 1 (separate
 *        K and V scales, per-head keys) and section 3 (per-head / per-128-token
 *        KV blocks).
 *   [M]  api.makesence.top, "LLM推理量化:FP8 versus INT8", section 二 (W8A8
 *        E4M3 with the KV cache in E5M2).
 *
 * Readings where the pages are silent or garbled (each also listed in the
 * design notes):
 *   - Bias, subnormals, NaN/Inf: derived from the table's constants.  E4M3:
 *     bias 7 (min normal 2^-6), subnormal m*2^-9, no Inf, S.1111.111 is NaN
 *     (max 448 = 1.75*2^8 leaves m=7 at e=15 unused).  E5M2: bias 15, subnormal
 *     m*2^-16, e=31 holds Inf (m=0) and NaN (m!=0).
 *   - Overflow saturates to +-max for both formats, Inf included.
 *   - The quotient x/s is one IEEE fp32 division (round to nearest even), then
 *     one rounding to the FP8 grid.  The scale is s = RN_fp32(amax / FMAX).
 *   - amax = 0 (all-zero group): s = 0 is stored, every code is the zero with
 *     the element's sign, no division happens.
 *   - NaN in a group makes amax NaN; NaN codes carry the fp32 payload's top
 *     mantissa bits so that encode(decode(c)) = c for all 256 codes.
 *   - Dequantize: y = RN_bf16(RN_fp32(decode(code) * s)).
 *
 * Parity pins for every function live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#if defined(__x86_64__)
#include <xmmintrin.h>
#endif

/* ------------------------------------------------------------------------ */
/* floating-point environment: IEEE round-to-nearest, no flush-to-zero       */

#if defined(__x86_64__)
#define FPENV_ENTER unsigned int saved_csr_ = _mm_getcsr(); _mm_setcsr(saved_csr_ & ~(0x8000u | 0x0040u | 0x6000u))
#define FPENV_LEAVE _mm_setcsr(saved_csr_)
#else
#define FPENV_ENTER do {} while (0)
#define FPENV_LEAVE do {} while (0)
#endif

/* ------------------------------------------------------------------------ */
/* formats, from the table in [W] "FP8 是什么"                               */

enum { ORC_E4M3 = 0, ORC_E5M2 = 1 };

typedef struct {
    int ebits;        /* exponent field width                 */
    int mbits;        /* mantissa field width                 */
    int bias;         /* 1 - log2(min normal)                 */
    float fmax;       /* largest finite magnitude             */
    int max_code;     /* positive code of fmax                */
} orc_fmt;

static orc_fmt fmt_of(int fmt) {
    orc_fmt f;
    if (fmt == ORC_E4M3) {        /* 1/4/3, max 448, min normal 2^-6, min subnormal 2^-9 */
        f.ebits = 4; f.mbits = 3; f.bias = 7; f.fmax = 448.0f; f.max_code = 0x7E;
    } else {                      /* 1/5/2, max 57344, min normal 2^-14, min subnormal 2^-16 */
        f.ebits = 5; f.mbits = 2; f.bias = 15; f.fmax = 57344.0f; f.max_code = 0x7B;
    }
    return f;
}

float orc_fmax(int fmt) { return fmt_of(fmt).fmax; }

static int is_nan_code(orc_fmt f, uint8_t c) {
    int e = (c >> f.mbits) & ((1 << f.ebits) - 1);
    int m = c & ((1 << f.mbits) - 1);
    if (f.ebits == 4) return e == 15 && m == 7;
    return e == 31 && m != 0;
}

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* code -> exact fp32 value */
float orc_decode(int fmt, uint8_t c) {
    orc_fmt f = fmt_of(fmt);
    int s = c >> 7;
    int e = (c >> f.mbits) & ((1 << f.ebits) - 1);
    int m = c & ((1 << f.mbits) - 1);
    if (is_nan_code(f, c))   /* keep the code's mantissa in the top mantissa bits of the NaN */
        return bits_to_f32(((uint32_t)s << 31) | 0x7F800000u | ((uint32_t)m << (23 - f.mbits)));
    if (f.ebits == 5 && e == 31)
        return s ? -INFINITY : INFINITY;
    double v;
    if (e == 0)
        v = ldexp((double)m, 1 - f.bias - f.mbits);                    /* subnormal: m * 2^(emin-M) */
    else
        v = ldexp(1.0 + (double)m / (double)(1 << f.mbits), e - f.bias); /* (1 + m/2^M) * 2^(e-bias) */
    return (float)(s ? -v : v);
}

/*
 * fp32 -> code: round to nearest, ties to even, saturating to +-max.
 * Works on the fp32 bit pattern with integer arithmetic.
 */
uint8_t orc_encode(int fmt, float q) {
    orc_fmt f = fmt_of(fmt);
    uint32_t b = f32_to_bits(q);
    uint8_t sign = (uint8_t)((b >> 24) & 0x80u);
    uint32_t a = b & 0x7FFFFFFFu;
    if (a > 0x7F800000u) {                                  /* NaN: keep payload's top bits */
        int m = (int)((a >> (23 - f.mbits)) & ((1u << f.mbits) - 1));
        if (f.ebits == 4) return sign | 0x7F;
        if (m == 0) m = 3;
        return (uint8_t)(sign | 0x7C | m);
    }
    if (fabsf(q) >= f.fmax)                                  /* Inf and overflow saturate */
        return (uint8_t)(sign | f.max_code);
    int exp32 = (int)(a >> 23);
    if (exp32 == 0)                                          /* below 2^-126: rounds to zero */
        return sign;
    int E = exp32 - 127;                                     /* |q| = sig * 2^(E-23) */
    uint64_t sig = (uint64_t)((a & 0x7FFFFFu) | 0x800000u);
    int emin = 1 - f.bias;
    int shift;                                               /* bits of sig below the FP8 ulp */
    int e8;
    if (E >= emin) { shift = 23 - f.mbits; e8 = E + f.bias; }
    else           { shift = 23 - f.mbits + (emin - E); e8 = 0; }
    if (shift > 40) return sign;                             /* far below half the min subnormal */
    uint64_t r = sig >> shift;
    uint64_t rem = sig & ((1ull << shift) - 1);
    uint64_t half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (r & 1))) r += 1;     /* ties to even */
    int code;
    if (e8 == 0)
        code = (int)r;                                       /* subnormal; r == 2^M is the min normal */
    else
        code = (e8 << f.mbits) + (int)r - (1 << f.mbits);    /* a carry moves into the exponent */
    if (code > f.max_code) code = f.max_code;
    return (uint8_t)(sign | code);
}

/*
 * fp32 -> code by brute force: the nearest of the format's finite values,
 * ties to the even code.  Independent of orc_encode; used to cross-check it.
 */
static uint8_t nearest_in_table(orc_fmt f, const double *tab, float q) {
    uint8_t sign = (uint8_t)((f32_to_bits(q) >> 24) & 0x80u);
    double aq = fabs((double)q);
    int best = 0;
    for (int c = 1; c <= f.max_code; ++c) {                  /* positive finite codes in increasing order */
        if (tab[c] <= aq) { best = c; continue; }
        double mid = 0.5 * (tab[best] + tab[c]);             /* aq lies in [tab[best], tab[c]) */
        if (aq > mid || (aq == mid && (c & 1) == 0)) best = c;
        break;
    }
    return (uint8_t)(sign | best);
}

static void decode_table(int fmt, double *tab) {
    for (int c = 0; c < 256; ++c) tab[c] = (double)orc_decode(fmt, (uint8_t)c);
}

/*
 * fp32 -> code by brute force: the nearest of the format's finite values,
 * ties to the even code (linear scan of the decoded table).  Independent of
 * orc_encode; used to cross-check it.  NaN is not a nearest-value question
 * and is passed to orc_encode.
 */
uint8_t orc_encode_nearest(int fmt, float q) {
    double tab[256];
    if (isnan(q)) return orc_encode(fmt, q);
    decode_table(fmt, tab);
    return nearest_in_table(fmt_of(fmt), tab, q);
}

void orc_decode_array(int fmt, const uint8_t *c, int64_t n, float *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_decode(fmt, c[i]);
}

void orc_encode_array(int fmt, const float *q, int64_t n, uint8_t *out) {
    FPENV_ENTER;
    for (int64_t i = 0; i < n; ++i) out[i] = orc_encode(fmt, q[i]);
    FPENV_LEAVE;
}

void orc_encode_nearest_array(int fmt, const float *q, int64_t n, uint8_t *out) {
    double tab[256];
    orc_fmt f = fmt_of(fmt);
    FPENV_ENTER;
    decode_table(fmt, tab);
    for (int64_t i = 0; i < n; ++i)
        out[i] = isnan(q[i]) ? orc_encode(fmt, q[i]) : nearest_in_table(f, tab, q[i]);
    FPENV_LEAVE;
}

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                             */

static float bf16_value(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

static uint16_t bf16_round(float v) {
    uint32_t u = f32_to_bits(v);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t hi = u >> 16, lo = u & 0xFFFFu;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1;
    return (uint16_t)hi;
}

/* ------------------------------------------------------------------------ */
/* scale and cast, [W] "什么是 FP8 量化" and "权重量化：128x128 分块 FP8"     */

/* s = amax / FMAX, one fp32 division */
float orc_scale(int fmt, float amax) {
    volatile float fm = fmt_of(fmt).fmax;
    return amax / fm;
}

/* one element: FP8(x / s); an all-zero group (s == 0) keeps only the sign */
static uint8_t cast_one(int fmt, float x, float s) {
    if (s == 0.0f) return (uint8_t)((f32_to_bits(x) >> 24) & 0x80u);
    float q = x / s;
    return orc_encode(fmt, q);
}

/* amax over a strided region; NaN is sticky */
static float region_amax(const uint16_t *x, int64_t nr, int64_t nc, int64_t ld) {
    float amax = 0.0f;
    for (int64_t r = 0; r < nr; ++r)
        for (int64_t c = 0; c < nc; ++c) {
            float v = fabsf(bf16_value(x[r * ld + c]));
            if (isnan(v) || isnan(amax)) amax = NAN;
            else if (v > amax) amax = v;
        }
    return amax;
}

/* quantize one scale group (a strided nr x nc region) and return its scale */
static float quantize_region(int fmt, const uint16_t *x, int64_t nr, int64_t nc, int64_t ld, uint8_t *codes) {
    float s = orc_scale(fmt, region_amax(x, nr, nc, ld));
    for (int64_t r = 0; r < nr; ++r)
        for (int64_t c = 0; c < nc; ++c)
            codes[r * ld + c] = cast_one(fmt, bf16_value(x[r * ld + c]), s);
    return s;
}

enum { ORC_PER_TENSOR = 0, ORC_GROUP_1x128 = 1, ORC_BLOCK_128x128 = 2 };

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

/*
 * x: bf16 [rows][cols] row-major.  codes: [rows][cols].  scales:
 *   per-tensor: [1]
 *   1x128 groups along a row ([W] "激活动态量化"): [ceil(cols/128)][rows],
 *        group-major so that one column of 128-groups is contiguous
 *   128x128 blocks ([W] "权重量化"): [ceil(rows/128)][ceil(cols/128)]
 * Returns 0, or -1 for a bad granularity.
 */
int orc_quantize(const uint16_t *x, int64_t rows, int64_t cols, int fmt, int gran, uint8_t *codes, float *scales) {
    FPENV_ENTER;
    int rc = 0;
    if (gran == ORC_PER_TENSOR) {
        scales[0] = quantize_region(fmt, x, rows, cols, cols, codes);
    } else if (gran == ORC_GROUP_1x128) {
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t g = 0; g < cdiv(cols, 128); ++g) {
                int64_t c0 = g * 128, nc = cols - c0 < 128 ? cols - c0 : 128;
                scales[g * rows + r] = quantize_region(fmt, x + r * cols + c0, 1, nc, cols, codes + r * cols + c0);
            }
    } else if (gran == ORC_BLOCK_128x128) {
        int64_t nbc = cdiv(cols, 128);
        for (int64_t bi = 0; bi < cdiv(rows, 128); ++bi)
            for (int64_t bj = 0; bj < nbc; ++bj) {
                int64_t r0 = bi * 128, c0 = bj * 128;
                int64_t nr = rows - r0 < 128 ? rows - r0 : 128;
                int64_t nc = cols - c0 < 128 ? cols - c0 : 128;
                scales[bi * nbc + bj] = quantize_region(fmt, x + r0 * cols + c0, nr, nc, cols, codes + r0 * cols + c0);
            }
    } else {
        rc = -1;
    }
    FPENV_LEAVE;
    return rc;
}

/* scale that applies to element (r, c) under a granularity, layouts as above */
static float scale_at(const float *scales, int64_t rows, int64_t cols, int gran, int64_t r, int64_t c) {
    if (gran == ORC_PER_TENSOR) return scales[0];
    if (gran == ORC_GROUP_1x128) return scales[(c / 128) * rows + r];
    return scales[(r / 128) * cdiv(cols, 128) + c / 128];
}

/* [C] x_hat = s * x_fp8, then rounded to bf16 */
int orc_dequantize(const uint8_t *codes, const float *scales, int64_t rows, int64_t cols, int fmt, int gran, uint16_t *y) {
    if (gran < 0 || gran > 2) return -1;
    FPENV_ENTER;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float v = orc_decode(fmt, codes[r * cols + c]) * scale_at(scales, rows, cols, gran, r, c);
            y[r * cols + c] = bf16_round(v);
        }
    FPENV_LEAVE;
    return 0;
}

/*
 * KV cache [tokens][heads][head_dim] bf16, K and V quantized separately ([P] section 1).
 *   0 per-tensor: one scale each for K and V ([M] section 二 uses E5M2 here)
 *   1 per-head:   k_scales[h], v_scales[h]
 *   2 per-head x per-128-token block ([P] section 3): scales[tb * heads + h]
 */
enum { ORC_KV_PER_TENSOR = 0, ORC_KV_PER_HEAD = 1, ORC_KV_PER_HEAD_TOK128 = 2 };

static void kv_one(const uint16_t *x, int64_t T, int64_t H, int64_t D, int fmt, int g, uint8_t *codes, float *scales) {
    int64_t ld = H * D;
    if (g == ORC_KV_PER_TENSOR) {
        scales[0] = quantize_region(fmt, x, T, ld, ld, codes);
    } else if (g == ORC_KV_PER_HEAD) {
        for (int64_t h = 0; h < H; ++h)
            scales[h] = quantize_region(fmt, x + h * D, T, D, ld, codes + h * D);
    } else {
        for (int64_t tb = 0; tb < cdiv(T, 128); ++tb)
            for (int64_t h = 0; h < H; ++h) {
                int64_t t0 = tb * 128, nt = T - t0 < 128 ? T - t0 : 128;
                scales[tb * H + h] = quantize_region(fmt, x + t0 * ld + h * D, nt, D, ld, codes + t0 * ld + h * D);
            }
    }
}

int orc_kv_quantize(const uint16_t *k, const uint16_t *v, int64_t T, int64_t H, int64_t D, int fmt, int g,
                    uint8_t *k_codes, uint8_t *v_codes, float *k_scales, float *v_scales) {
    if (g < 0 || g > 2) return -1;
    FPENV_ENTER;
    kv_one(k, T, H, D, fmt, g, k_codes, k_scales);
    kv_one(v, T, H, D, fmt, g, v_codes, v_scales);
    FPENV_LEAVE;
    return 0;
}

/*
 * Reference GEMM, [W] "激活动态量化" and "FP8 矩阵乘":
 *   C[m][n] = sum_k (decode(A[m][k]) * sA(m,k)) * (decode(B[n][k]) * sB(n,k))   in fp64
 * A [M][K] codes with scales per-tensor (gA = 0) or 1x128 groups (gA = 1, layout
 * [K/128][M]); B [N][K] codes (W in R^{N x K}) with scales per-tensor (gB = 0) or
 * 128x128 blocks (gB = 2, layout [ceil(N/128)][ceil(K/128)]).  Only the listed rows of
 * C are computed: out[i][n] = C[rows[i]][n].
 */
int orc_gemm_rows(const uint8_t *A, const float *sA, int gA, const uint8_t *B, const float *sB, int gB,
                  int fmtA, int fmtB, int64_t M, int64_t N, int64_t K,
                  const int64_t *rows, int64_t nrows, double *out) {
    if (!(gA == ORC_PER_TENSOR || gA == ORC_GROUP_1x128)) return -1;
    if (!(gB == ORC_PER_TENSOR || gB == ORC_BLOCK_128x128)) return -1;
    FPENV_ENTER;
    double *a = (double *)malloc(sizeof(double) * (size_t)(K * nrows));
    double *b = (double *)malloc(sizeof(double) * (size_t)K);
    for (int64_t i = 0; i < nrows; ++i)
        for (int64_t k = 0; k < K; ++k)
            a[i * K + k] = (double)orc_decode(fmtA, A[rows[i] * K + k]) * (double)scale_at(sA, M, K, gA, rows[i], k);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k)
            b[k] = (double)orc_decode(fmtB, B[n * K + k]) * (double)scale_at(sB, N, K, gB, n, k);
        for (int64_t i = 0; i < nrows; ++i) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += a[i * K + k] * b[k];
            out[i * N + n] = acc;
        }
    }
    free(a);
    free(b);
    FPENV_LEAVE;
    return 0;
}

/*
 * Symmetric INT8 on a uniform grid, step amax/127 ([W] "FP8 与 INT8 量化精度对比"):
 * the comparison the worked example draws.  Returns the integer level.
 */
int orc_int8_level(double x, double amax) {
    double step = amax / 127.0;
    double l = nearbyint(x / step);
    if (l > 127) l = 127;
    if (l < -127) l = -127;
    return (int)l;
}

/* ------------------------------------------------------------------------ */
/* delayed scaling and per-call counts                                       */
/*
 * Delayed scaling ([C] "scale 是控制面": the scale follows a history of amax
 * values recorded by earlier steps instead of the tensor being cast; [M]
 * section 二: the forward pass takes its scale factor from the previous
 * micro-batch's max).  Counts of saturated and underflowed elements are the
 * overflow / underflow signals [C] "scale 是控制面" asks to be observable.
 *
 * Readings (also in the design notes):
 *   - One scale group is a column block over all rows: columns
 *     [g*gw, (g+1)*gw) of x [rows][ngroups*gw] (per-tensor: ngroups = 1,
 *     gw = cols; a KV cache per head: rows = tokens, ngroups = heads,
 *     gw = head_dim).
 *   - history [H][ngroups] holds amax values of earlier calls, zero where no
 *     call has written; entries are >= 0 or NaN.
 *   - step 0 has no history yet: its scale comes from its own amax (the
 *     dynamic rule).  Step t >= 1: s = RN(max over the H entries / FMAX), NaN
 *     sticky.  Either way the cast is the usual FP8(RN(x / s)), saturating; an
 *     all-zero history gives s = 0 and sign-only codes (as for an all-zero
 *     group).
 *   - Afterwards history[t mod H][g] = this call's own amax of group g.
 *   - counts[0] += elements that saturate: round-to-nearest-even of |x / s| on
 *     the format's grid continued past FMAX lands above FMAX.
 *     counts[1] += elements with x != 0 (NaN excluded) whose code is +-0.
 */

/* does |q| round (ties to even) above FMAX on the grid continued past FMAX? */
static int saturates(int fmt, float q) {
    orc_fmt f = fmt_of(fmt);
    double a = fabs((double)q);
    if (isnan(q)) return 0;
    /* FMAX = (2 - 2^(1-M)) * 2^E: the next point of the continued grid is FMAX + 2^(E-M) */
    int e;
    frexp((double)f.fmax, &e);                 /* FMAX = m * 2^e with m in [0.5, 1): E = e - 1 */
    double next = (double)f.fmax + ldexp(1.0, (e - 1) - f.mbits);
    double mid = 0.5 * ((double)f.fmax + next);
    if (a > mid) return 1;
    if (a < mid) return 0;
    return (f.max_code & 1) != 0;              /* a tie goes to the even mantissa: next if FMAX's is odd */
}

int orc_quantize_delayed(const uint16_t *x, int64_t rows, int64_t ngroups, int64_t gw, int fmt,
                         float *history, int64_t H, int64_t step, uint8_t *codes, float *scales,
                         uint64_t *counts) {
    if (H < 1 || step < 0 || ngroups < 1 || gw < 1) return -1;
    FPENV_ENTER;
    int64_t ld = ngroups * gw;
    float *cur = (float *)malloc(sizeof(float) * (size_t)ngroups);
    for (int64_t g = 0; g < ngroups; ++g) {
        cur[g] = region_amax(x + g * gw, rows, gw, ld);
        float a = cur[g];
        if (step > 0) {
            a = 0.0f;
            for (int64_t t = 0; t < H; ++t) {
                float h = history[t * ngroups + g];
                if (isnan(h) || isnan(a)) a = NAN;
                else if (h > a) a = h;
            }
        }
        float s = orc_scale(fmt, a);
        scales[g] = s;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < gw; ++c) {
                float xv = bf16_value(x[r * ld + g * gw + c]);
                uint8_t code = cast_one(fmt, xv, s);
                codes[r * ld + g * gw + c] = code;
                if (counts) {
                    if (s != 0.0f && saturates(fmt, xv / s)) counts[0] += 1;
                    if (!isnan(xv) && xv != 0.0f && (code & 0x7F) == 0) counts[1] += 1;
                }
            }
    }
    for (int64_t g = 0; g < ngroups; ++g) history[(step % H) * ngroups + g] = cur[g];
    free(cur);
    FPENV_LEAVE;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MXFP8: 1x32 groups with power-of-two scales                               */
/*
 * [M] section on Microscaling (block size 32, native on Blackwell): per-block
 * scaling with blocks of 32 elements.  The pages give no scale rule for it;
 * the reading taken (design notes) is the pages' own rule restricted to powers
 * of two: the scale of a group is the smallest 2^k with amax <= FMAX * 2^k (so
 * the amax element never saturates), stored as the 8-bit exponent k + 127, k
 * clamped at -127 (byte 0); an all-zero group takes byte 0; NaN or infinite
 * amax takes byte 255 (a NaN scale).  Codes are FP8(RN(x / 2^k)).
 */

/* smallest k with amax <= fmax * 2^k, by exact comparison (both sides binary) */
int orc_mx_exponent(int fmt, float amax) {
    double fm = (double)fmt_of(fmt).fmax;
    if (isnan(amax) || isinf(amax)) return 128;              /* NaN scale */
    if (amax == 0.0f) return -127;
    int k = 0;
    while ((double)amax > ldexp(fm, k)) ++k;
    while (k > -127 && (double)amax <= ldexp(fm, k - 1)) --k;
    return k;
}

/* x bf16 [rows][cols], cols % 32 == 0; codes [rows][cols]; scales uint8 [rows][cols / 32] */
int orc_quantize_mx(const uint16_t *x, int64_t rows, int64_t cols, int fmt, uint8_t *codes, uint8_t *scales) {
    if (cols % 32 != 0) return -1;
    FPENV_ENTER;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < cols / 32; ++g) {
            const uint16_t *xg = x + r * cols + g * 32;
            float amax = region_amax(xg, 1, 32, 32);
            int k = orc_mx_exponent(fmt, amax);
            scales[r * (cols / 32) + g] = (uint8_t)(k + 127);
            for (int c = 0; c < 32; ++c) {
                float xv = bf16_value(xg[c]);
                float q = (k == 128) ? xv / NAN : xv / (float)ldexp(1.0, k);
                codes[r * cols + g * 32 + c] = orc_encode(fmt, q);
            }
        }
    FPENV_LEAVE;
    return 0;
}

/* y = RN_bf16(RN_fp32(decode(code) * 2^(byte - 127))); byte 255 is a NaN scale */
int orc_dequantize_mx(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols, int fmt,
                      uint16_t *y) {
    if (cols % 32 != 0) return -1;
    FPENV_ENTER;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            int b = scales[r * (cols / 32) + c / 32];
            float s = b == 255 ? NAN : (float)ldexp(1.0, b - 127);
            y[r * cols + c] = bf16_round(orc_decode(fmt, codes[r * cols + c]) * s);
        }
    FPENV_LEAVE;
    return 0;
}

/*
 * MXFP8 GEMM ([M] section on Microscaling: every 32 consecutive elements along K
 * carry one power-of-two scale; [W] "FP8 矩阵乘": FP8 products, accumulation in
 * high precision, the scales multiplied back):
 *   C[m][n] = sum_k (decode(A[m][k]) * 2^(sA[m][k/32] - 127))
 *                 * (decode(B[n][k]) * 2^(sB[n][k/32] - 127))            in fp64
 * A [M][K] and B [N][K] codes (K % 32 == 0), scale bytes row-major [rows][K/32];
 * byte 255 is a NaN scale.  Only the listed rows of C are computed:
 * out[i][n] = C[rows[i]][n].
 */
static double mx_scale_value(uint8_t b) { return b == 255 ? NAN : ldexp(1.0, (int)b - 127); }

int orc_gemm_mx_rows(const uint8_t *A, const uint8_t *sA, const uint8_t *B, const uint8_t *sB, int fmtA, int fmtB,
                     int64_t M, int64_t N, int64_t K, const int64_t *rows, int64_t nrows, double *out) {
    if (K % 32 != 0) return -1;
    FPENV_ENTER;
    const int64_t G = K / 32;
    double *a = (double *)malloc(sizeof(double) * (size_t)(K * nrows));
    double *b = (double *)malloc(sizeof(double) * (size_t)K);
    for (int64_t i = 0; i < nrows; ++i)
        for (int64_t k = 0; k < K; ++k)
            a[i * K + k] = (double)orc_decode(fmtA, A[rows[i] * K + k]) * mx_scale_value(sA[rows[i] * G + k / 32]);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k)
            b[k] = (double)orc_decode(fmtB, B[n * K + k]) * mx_scale_value(sB[n * G + k / 32]);
        for (int64_t i = 0; i < nrows; ++i) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += a[i * K + k] * b[k];
            out[i * N + n] = acc;
        }
    }
    free(a);
    free(b);
    (void)M;
    FPENV_LEAVE;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* scale health                                                              */
/*
 * [C] "scale 是控制面": the scales and the overflow / underflow they cause
 * should be observable.  Two plain counts:
 *   - a histogram of scales by power of two: kind 0 takes fp32 scales and
 *     counts each in the bucket of its biased exponent field (bucket 0: zero
 *     or subnormal, 255: Inf or NaN; so amax = s * FMAX falls in a known
 *     octave); kind 1 takes MX scale bytes (the biased exponent itself);
 *     hist[256] is added to;
 *   - underflow to zero: nonzero, non-NaN inputs whose code is +-0 (added to
 *     *count).
 */
int orc_scale_histogram(const void *scales, int64_t n, int kind, uint32_t *hist) {
    if (kind != 0 && kind != 1) return -1;
    for (int64_t i = 0; i < n; ++i) {
        int b;
        if (kind == 0) {
            float s = ((const float *)scales)[i];
            uint32_t bits;
            memcpy(&bits, &s, 4);
            b = (int)((bits >> 23) & 0xFF);
        } else {
            b = ((const uint8_t *)scales)[i];
        }
        hist[b] += 1;
    }
    return 0;
}

int orc_count_underflow(const uint16_t *x, const uint8_t *codes, int64_t n, uint64_t *count) {
    for (int64_t i = 0; i < n; ++i) {
        float xv = bf16_value(x[i]);
        if (!isnan(xv) && xv != 0.0f && (codes[i] & 0x7F) == 0) *count += 1;
    }
    return 0;
}
