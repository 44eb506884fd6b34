/*
 * Seeded, counter-based generators for the synthetic input tensors.
 *
 * This file is shared by the CPU oracle's tests and by the GPU path's tests
 * and benchmark.  It holds no FP8 arithmetic: it only draws random numbers and
 * formats them as bfloat16 input tensors.
 *
 * Random source: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  The i-th output of a
 * generator seeded with `key` is mix(key + (i + 1) * GAMMA), so any element of
 * a stream can be produced on its own, in any order, by any thread.
 *
 * Normals come from the Box-Muller transform: element 2j takes the cosine
 * branch and element 2j+1 the sine branch of the pair built from uniforms
 * 2j and 2j+1 of the same stream.  Samples are drawn in double precision,
 * rounded to float (round-to-nearest) and then to bfloat16 (round to nearest,
 * ties to even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SM_GAMMA 0x9E3779B97F4A7C15ull

static uint64_t sm_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* i-th output of a SplitMix64 generator seeded with key */
static uint64_t sm_at(uint64_t key, uint64_t i) { return sm_mix(key + (i + 1) * SM_GAMMA); }

/* stream key for (seed, stream id): output `stream` of a generator seeded with seed */
uint64_t synth_key(uint64_t seed, uint64_t stream) { return sm_at(seed * 0xD1B54A32D192ED03ull, stream); }

/* uniform double in [0, 1) with 53 random bits */
static double u01(uint64_t key, uint64_t i) { return (double)(sm_at(key, i) >> 11) * 0x1.0p-53; }

static double normal_at(uint64_t key, uint64_t i) {
    uint64_t j = i >> 1;
    double u1 = 1.0 - u01(key, 2 * j);     /* (0, 1] so the log is finite */
    double u2 = u01(key, 2 * j + 1);
    double r = sqrt(-2.0 * log(u1));
    double t = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(t) : r * cos(t);
}

/* double -> float (round to nearest) -> bfloat16 bits (nearest, ties to even) */
static uint16_t to_bf16_bits(double v) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* raw 64-bit outputs [start, start + n) of stream `key` */
void synth_u64(uint64_t key, int64_t start, int64_t n, uint64_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = sm_at(key, (uint64_t)(start + i));
}

/* uniform doubles in [lo, hi) for elements [start, start + n) */
void synth_uniform_f64(uint64_t key, int64_t start, int64_t n, double lo, double hi, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = lo + (hi - lo) * u01(key, (uint64_t)(start + i));
}

/* normal doubles N(mean, std^2) for elements [start, start + n) */
void synth_normal_f64(uint64_t key, int64_t start, int64_t n, double mean, double std, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = mean + std * normal_at(key, (uint64_t)(start + i));
}

/* bf16 tensor elements [start, start + n) drawn from U(lo, hi) */
void synth_uniform_bf16(uint64_t key, int64_t start, int64_t n, double lo, double hi, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16_bits(lo + (hi - lo) * u01(key, (uint64_t)(start + i)));
}

/* bf16 tensor elements [start, start + n) drawn from N(mean, std^2) */
void synth_normal_bf16(uint64_t key, int64_t start, int64_t n, double mean, double std, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16_bits(mean + std * normal_at(key, (uint64_t)(start + i)));
}

/*
 * bf16 tensor elements [start, start + n) of a row-major [rows][cols] tensor
 * drawn from N(0, std^2) * row_gain[row] * col_gain[col]; either gain array
 * may be NULL (gain 1).  Used for outlier channels (col_gain) and for the
 * per-position / per-head magnitude profile of the key cache, flattened as
 * rows = tokens, cols = heads * head_dim, with col_gain repeating the head
 * multiplier over head_dim.
 */
void synth_normal_gain_bf16(uint64_t key, int64_t start, int64_t n, int64_t cols, double std,
                            const double *row_gain, const double *col_gain, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) {
        int64_t e = start + i;
        double v = std * normal_at(key, (uint64_t)e);
        if (row_gain) v *= row_gain[e / cols];
        if (col_gain) v *= col_gain[e % cols];
        out[i] = to_bf16_bits(v);
    }
}

/* re-draw listed elements with a multiplier: out[idx[j] - start] = bf16(base(idx[j]) * gain) */
void synth_scale_points_normal_bf16(uint64_t key, double std, const int64_t *idx, int64_t n_idx,
                                    int64_t start, int64_t n, double gain, uint16_t *out) {
    for (int64_t j = 0; j < n_idx; ++j) {
        int64_t e = idx[j];
        if (e < start || e >= start + n) continue;
        out[e - start] = to_bf16_bits(std * normal_at(key, (uint64_t)e) * gain);
    }
}
