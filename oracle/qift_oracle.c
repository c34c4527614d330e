/*
 * qift_oracle.c -- plain, slow, obviously-correct CPU oracle for the Qift W2A4 linear path.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the CPU-baseline leg of the
 * benchmark are the only code that loads this library.  The product (the CUDA library in
 * w2a4_gemm_b200/) never calls it, and this file shares no code, header, table or constant
 * with it: each side derives its constants from the definitions on its own.
 *
 * What it follows: "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated
 * W2A4/KV4 LLM Inference" (Huang, Tsai, arXiv 2606.02823v1), Abstract:
 *   - weights and activations pass through a Hadamard-rotated pipeline;
 *   - the main 2-bit level set is {+-0.5, +-1.5} (times the per-channel scale s), the same
 *     set as {+-1, +-3} under the half-scale t = s/2;
 *   - a power-of-two variant uses {+-1, +-4} so a weight is applied by sign and shift;
 *   - the standard W2 set {-2, -1, 0, +1} is the baseline;
 *   - one scale per output channel, no zero point, no groups;
 *   - W2A4: 2-bit weights against 4-bit activations.
 * Where the abstract is silent the functions below state the reading they take (R1..R16).
 *
 * Arithmetic: IEEE binary32 / binary64 with round-to-nearest-even.  Build with
 * -O2 -ffp-contract=off and without -ffast-math so no operation is fused or reordered.
 * OpenMP only splits independent rows / tokens across threads; it changes no result.
 *
 * Every function returns 0 on success and a negative number on a bad argument.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define QO_SET_QIFT 0 /* levels {-3,-1,+1,+3} * t, t = s/2  ({-1.5,-0.5,+0.5,+1.5} * s) */
#define QO_SET_POT 1  /* levels {-4,-1,+1,+4} * t                                       */
#define QO_SET_STD 2  /* levels {-2,-1, 0,+1} * t                                       */

static int is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

/* ---------------------------------------------------------------------------------------
 * Hadamard rotation (Abstract: "Hadamard-rotated quantization pipeline").
 *
 * R1: H_b is the Sylvester Hadamard matrix, H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]],
 *     normalised by 1/sqrt(b), applied block-diagonally: every length-b segment of a row
 *     is rotated on its own.  H_b is symmetric, so W H_b^T = W H_b row by row.
 * R2: the fast transform runs stages h = 1, 2, 4, ..., b/2; in a stage every pair (i, i+h)
 *     with (i & h) == 0 becomes (u + v, u - v); after the last stage every element is
 *     multiplied once by the normalisation constant.
 * ------------------------------------------------------------------------------------- */

/* fp64 form: the exact definition, used by the mathematical pins. */
int qo_fwht_f64(double* x, int64_t rows, int64_t n, int32_t b) {
    if (!x || rows < 0 || n < 0 || !is_pow2(b) || (n % b) != 0) return -1;
    const double c = 1.0 / sqrt((double)b);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t seg = 0; seg < n; seg += b) {
            double* v = x + r * n + seg;
            for (int64_t h = 1; h < b; h <<= 1) {
                for (int64_t i = 0; i < b; ++i) {
                    if (i & h) continue;
                    double u = v[i], w = v[i + h];
                    v[i] = u + w;
                    v[i + h] = u - w;
                }
            }
            for (int64_t i = 0; i < b; ++i) v[i] = v[i] * c;
        }
    }
    return 0;
}

/* fp32 form: the same stages in binary32, then one multiply by (float)(1/sqrt(b)).
 * This is the precision the CUDA path computes in, so it decides the codes downstream. */
int qo_rotate_f32(float* x, int64_t rows, int64_t n, int32_t b) {
    if (!x || rows < 0 || n < 0 || !is_pow2(b) || (n % b) != 0) return -1;
    const float c = (float)(1.0 / sqrt((double)b));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t seg = 0; seg < n; seg += b) {
            float* v = x + r * n + seg;
            for (int64_t h = 1; h < b; h <<= 1) {
                for (int64_t i = 0; i < b; ++i) {
                    if (i & h) continue;
                    float u = v[i], w = v[i + h];
                    v[i] = u + w;
                    v[i + h] = u - w;
                }
            }
            for (int64_t i = 0; i < b; ++i) v[i] = v[i] * c;
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * Level sets (Abstract: "{+/-0.5, +/-1.5}, equivalently {+/-1, +/-3} under a half-scale
 * reparameterization"; "a power-of-two variant uses {+/-1, +/-4}"; "the standard W2 level
 * set {-2,-1,0,+1}").
 * R6: the 2-bit code is monotone in the level: code 0 is the most negative level and code 3
 *     the most positive one.
 * ------------------------------------------------------------------------------------- */
static const int32_t LEVELS[3][4] = {
    {-3, -1, +1, +3}, /* Qift, half-scale integers */
    {-4, -1, +1, +4}, /* power-of-two variant      */
    {-2, -1, 0, +1},  /* standard W2               */
};

int32_t qo_level(int32_t set, int32_t code) {
    if (set < 0 || set > 2 || code < 0 || code > 3) return -1000;
    return LEVELS[set][code];
}

/* Largest level magnitude of each set in the units the scale grid is written in
 * (Qift: the s-form {+-0.5, +-1.5} s, so 1.5; PoT: 4; standard: 2). */
static double outer_level(int32_t set) { return set == QO_SET_QIFT ? 1.5 : (set == QO_SET_POT ? 4.0 : 2.0); }

/* R3: candidate k of G (k = 0..G-1) for a row whose largest magnitude is m:
 *     f_k = lo + ((hi - lo) * k) / (G - 1);  s_k = (float)((f_k * m) / lambda)
 * every operation in binary64, in that order, one rounding to binary32 at the end.  For
 * G = 100, lo = 0.2, hi = 1.0 this is the 100-point grid over [0.2, 1.0] * max|w| / 1.5. */
int qo_candidate_scales(float m, int32_t set, int32_t grid_points, double lo, double hi, float* s) {
    if (!s || set < 0 || set > 2 || grid_points < 2) return -1;
    const double lambda = outer_level(set);
    for (int32_t k = 0; k < grid_points; ++k) {
        double f = lo + ((hi - lo) * (double)k) / (double)(grid_points - 1);
        s[k] = (float)((f * (double)m) / lambda);
    }
    return 0;
}

/* Nearest-level code of one weight for a candidate s (in the grid's units).
 * Thresholds are the midpoints of neighbouring levels, compared in binary64, where every
 * threshold below is exact (a binary32 times 0.5, 1, 1.5 or 2.5).
 * R7: w >= 0 (so -0.0 too) takes the positive side.
 * R8: a weight exactly on a threshold takes the level of smaller magnitude. */
static int32_t encode_one(float w, float s, int32_t set) {
    const double a = fabs((double)w), sd = (double)s, wd = (double)w;
    switch (set) {
        case QO_SET_QIFT: { /* levels +-0.5 s, +-1.5 s: the midpoint is s */
            int outer = a > sd;
            if (w >= 0.0f) return outer ? 3 : 2;
            return outer ? 0 : 1;
        }
        case QO_SET_POT: { /* levels +-s, +-4 s: the midpoint is 2.5 s */
            int outer = a > 2.5 * sd;
            if (w >= 0.0f) return outer ? 3 : 2;
            return outer ? 0 : 1;
        }
        default: { /* levels -2s, -s, 0, +s: midpoints -1.5 s, -0.5 s, +0.5 s */
            if (wd < -1.5 * sd) return 0;
            if (wd < -0.5 * sd) return 1;
            if (wd <= 0.5 * sd) return 2;
            return 3;
        }
    }
}

/* Reconstruction error of one weight for its code, in binary32 (R9):
 *   Qift: e = |w| - l, l = 0.5f * s (inner) or 1.5f * s (outer), each product in binary32;
 *   PoT:  e = |w| - l, l = s or 4.0f * s;
 *   std:  e = w - l,   l = level * s  (level in {-2,-1,0,1}).
 * The squared error e * e is rounded to binary32 as well. */
static float sq_err(float w, float s, int32_t set, int32_t code) {
    float e;
    if (set == QO_SET_STD) {
        float l = (float)LEVELS[QO_SET_STD][code] * s;
        e = w - l;
    } else {
        int outer = (code == 0 || code == 3);
        float l;
        if (set == QO_SET_QIFT) l = outer ? 1.5f * s : 0.5f * s;
        else l = outer ? 4.0f * s : s;
        e = fabsf(w) - l;
    }
    return e * e;
}

/* ---------------------------------------------------------------------------------------
 * Per-channel scale search, nearest-level encoding and 2-bit packing (Abstract: "retaining
 * the standard per-channel scale"; "fixed two-bit code-to-level mapping"; zero-point-free,
 * group-grid-free).
 *
 * For each output row n of the rotated weights w[n][0..K):
 *   m = max_k |w[n][k]| (binary32);
 *   for every candidate s_k: MSE_k = sum over k of sq_err, accumulated in binary64 in
 *   index order 0..K-1 (R9);
 *   s_best = the candidate with the smallest MSE_k; on equal MSE the smaller k wins (R4);
 *   the codes are the nearest-level codes for s_best; the stored scale is the half scale
 *   t = s_best / 2 for Qift (so levels {+-1, +-3} * t) and s_best itself for PoT and std.
 * R5: an all-zero row has m = 0, every candidate is 0, every MSE is 0, so s_best = 0 and every
 *     code is 2 (the +inner level; level 0 for std) -- the general rule, no special case.
 * R10: the code of input index k goes to word codes[n*(K/16) + k/16], bits 2*(k%16) and
 *      2*(k%16)+1 (least significant first).
 * row_mse[n] = (MSE of the best candidate) / K in binary64; best_k[n] = its index.  Either may be NULL.
 * ------------------------------------------------------------------------------------- */
int qo_quantize_weights(const float* w, int64_t n_out, int64_t n_in, int32_t set, int32_t grid_points,
                        double lo, double hi, uint32_t* codes, float* scales, double* row_mse,
                        int32_t* best_k) {
    if (!w || !codes || !scales || n_out < 0 || n_in <= 0 || (n_in % 16) != 0) return -1;
    if (set < 0 || set > 2 || grid_points < 2 || grid_points > 4096) return -1;
    const int64_t words = n_in / 16;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < n_out; ++n) {
        const float* row = w + n * n_in;
        float m = 0.0f;
        for (int64_t k = 0; k < n_in; ++k) {
            float a = fabsf(row[k]);
            if (a > m) m = a;
        }
        float* cand = (float*)malloc(sizeof(float) * (size_t)grid_points);
        if (!cand) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        qo_candidate_scales(m, set, grid_points, lo, hi, cand);
        int32_t kbest = 0;
        double best = 0.0;
        for (int32_t g = 0; g < grid_points; ++g) {
            const float s = cand[g];
            double acc = 0.0;
            for (int64_t k = 0; k < n_in; ++k) {
                int32_t c = encode_one(row[k], s, set);
                acc += (double)sq_err(row[k], s, set, c);
            }
            if (g == 0 || acc < best) {
                best = acc;
                kbest = g;
            }
        }
        const float s = cand[kbest];
        free(cand);
        uint32_t* out = codes + n * words;
        for (int64_t j = 0; j < words; ++j) out[j] = 0u;
        for (int64_t k = 0; k < n_in; ++k) {
            uint32_t c = (uint32_t)encode_one(row[k], s, set);
            out[k / 16] |= c << (2 * (k % 16));
        }
        scales[n] = (set == QO_SET_QIFT) ? s * 0.5f : s;
        if (row_mse) row_mse[n] = best / (double)n_in;
        if (best_k) best_k[n] = kbest;
    }
    return bad ? -2 : 0;
}

/* Unpack: codes[n*(K/16) + k/16] bits 2*(k%16).. -> one code per byte (R10). */
int qo_unpack_codes(const uint32_t* codes, int64_t n_out, int64_t n_in, uint8_t* out) {
    if (!codes || !out || n_out < 0 || n_in <= 0 || (n_in % 16) != 0) return -1;
    const int64_t words = n_in / 16;
    for (int64_t n = 0; n < n_out; ++n)
        for (int64_t k = 0; k < n_in; ++k)
            out[n * n_in + k] = (uint8_t)((codes[n * words + k / 16] >> (2 * (k % 16))) & 3u);
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * W4 weights (the Abstract's "L-layer mixed W2/W4": 4-bit layers beside the 2-bit ones).  The
 * page gives no W4 scheme; the reading (R20) keeps this method's rule -- one scale per output
 * channel, no zero point, the same MSE-searched candidate grid (R3, outer level 7) -- with the
 * symmetric 4-bit integer levels {-7, ..., +7} * s.
 *   encode: |w| against the midpoints (j + 0.5) s, j = 0..6, in binary64 (exact: a binary32
 *           times j + 0.5 needs at most 28 bits); level magnitude = the number of midpoints
 *           strictly below |w|, so a tie takes the smaller magnitude (R8); w >= 0 (and -0.0)
 *           takes the positive side (R7);
 *   error:  e = |w| - l, l = j * s in binary32, e * e in binary32, summed in binary64 in index
 *           order (R9);
 *   code:   the level as a 4-bit two's-complement nibble, eight per u32 (R21): word k/8 holds
 *           inputs 8w .. 8w+7, byte j of it input 8w+j in the low nibble and input 8w+j+4 in
 *           the high nibble, i.e. input k at bits 8*(k%4) + 4*((k%8)/4) .. +3.  The stored
 *           scale is s itself.
 * ------------------------------------------------------------------------------------- */
/* Bit position of input k's nibble inside its word (R21). */
static int w4_shift(int64_t k) { return (int)(8 * (k % 4) + 4 * ((k % 8) / 4)); }

/* The level a nibble stores: its two's-complement value, -8..7. */
static int32_t w4_level(uint32_t nibble) { return nibble >= 8u ? (int32_t)nibble - 16 : (int32_t)nibble; }

static int32_t encode_w4(float w, float s) {
    const double a = fabs((double)w), sd = (double)s;
    int32_t j = 0;
    while (j < 7 && a > ((double)j + 0.5) * sd) ++j;
    return w >= 0.0f ? j : -j;
}

static float sq_err_w4(float w, float s, int32_t level) {
    const float l = (float)(level < 0 ? -level : level) * s;
    const float e = fabsf(w) - l;
    return e * e;
}

int qo_quantize_weights_w4(const float* w, int64_t n_out, int64_t n_in, int32_t grid_points, double lo, double hi,
                           uint32_t* codes, float* scales, double* row_mse, int32_t* best_k) {
    if (!w || !codes || !scales || n_out < 0 || n_in <= 0 || (n_in % 8) != 0) return -1;
    if (grid_points < 2 || grid_points > 4096) return -1;
    const int64_t words = n_in / 8;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < n_out; ++n) {
        const float* row = w + n * n_in;
        float m = 0.0f;
        for (int64_t k = 0; k < n_in; ++k) {
            const float a = fabsf(row[k]);
            if (a > m) m = a;
        }
        float* cand = (float*)malloc(sizeof(float) * (size_t)grid_points);
        if (!cand) {
#pragma omp atomic write
            bad = 1;
            continue;
        }
        for (int32_t g = 0; g < grid_points; ++g) {  /* R3 with the outer level 7 */
            const double f = lo + ((hi - lo) * (double)g) / (double)(grid_points - 1);
            cand[g] = (float)((f * (double)m) / 7.0);
        }
        int32_t kbest = 0;
        double best = 0.0;
        for (int32_t g = 0; g < grid_points; ++g) {
            const float s = cand[g];
            double acc = 0.0;
            for (int64_t k = 0; k < n_in; ++k) acc += (double)sq_err_w4(row[k], s, encode_w4(row[k], s));
            if (g == 0 || acc < best) {
                best = acc;
                kbest = g;
            }
        }
        const float s = cand[kbest];
        free(cand);
        uint32_t* out = codes + n * words;
        for (int64_t j = 0; j < words; ++j) out[j] = 0u;
        for (int64_t k = 0; k < n_in; ++k)
            out[k / 8] |= ((uint32_t)encode_w4(row[k], s) & 0xFu) << w4_shift(k);
        scales[n] = s;
        if (row_mse) row_mse[n] = best / (double)n_in;
        if (best_k) best_k[n] = kbest;
    }
    return bad ? -2 : 0;
}

/* W4A4 linear: acc[t][n] = sum_k q[t][k] * level(code) exactly (int64, must fit int32), then
 * y = ((float)acc * s_w[n]) * s_a[t] (R13).  acc and y may be NULL. */
int qo_linear_w4(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int64_t tokens,
                 int64_t n_out, int64_t n_in, int32_t* acc_out, float* y) {
    if (!q || !s_a || !codes || !s_w || tokens < 0 || n_out < 0 || n_in <= 0 || (n_in % 8) != 0) return -1;
    const int64_t words = n_in / 8;
    int overflow = 0;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t t = 0; t < tokens; ++t) {
        for (int64_t n = 0; n < n_out; ++n) {
            int64_t sum = 0;
            for (int64_t k = 0; k < n_in; ++k) {
                const uint32_t nib = (codes[n * words + k / 8] >> w4_shift(k)) & 0xFu;
                sum += (int64_t)q[t * n_in + k] * (int64_t)w4_level(nib);
            }
            if (sum > INT32_MAX || sum < INT32_MIN) {
#pragma omp atomic write
                overflow = 1;
            }
            if (acc_out) acc_out[t * n_out + n] = (int32_t)sum;
            if (y) y[t * n_out + n] = ((float)sum * s_w[n]) * s_a[t];
        }
    }
    return overflow ? -3 : 0;
}

/* ---------------------------------------------------------------------------------------
 * Conventional asymmetric W2 (the Abstract's comparison baseline, "Conventional asymmetric
 * W2"): four uniform levels with a per-channel zero point.  The page gives no formula; the
 * reading (R22) is the usual min-max affine quantizer with an integer zero point, searched
 * over the same candidate grid as the other sets (R3) by shrinking the range:
 *   lo_w = min(min_k w, 0), hi_w = max(max_k w, 0) (binary32; the range always holds 0);
 *   candidate g: f_g as in R3; s_g = (float)((f_g * (hi_w - lo_w)) / 3) in binary64, one
 *                rounding; z_g = nearest integer (ties to even) of -(f_g * lo_w) / s_g in
 *                binary64, clamped to [0, 3] (0 when s_g = 0);
 *   encode:      c = clamp(rint(w / s) + z, 0, 3), w / s one binary32 division, rint to
 *                nearest even (c = z when s = 0);
 *   error:       e = w - (float)(c - z) * s in binary32, e * e in binary32, summed in binary64
 *                in index order (R9); smallest sum wins, the smaller g on ties (R4).
 * The weight is (c - z) * s: code z is exactly 0.  Codes are packed as R10; the row keeps s and
 * z.  The linear then reads the levels c - z: acc = sum q * (c - z) = sum q * c - z * sum q.
 * ------------------------------------------------------------------------------------- */
static int32_t asym_zero(double f, float lo_w, float s) {
    if (!(s > 0.0f)) return 0;
    double z = nearbyint(-(f * (double)lo_w) / (double)s);
    return z < 0.0 ? 0 : (z > 3.0 ? 3 : (int32_t)z);
}

static int32_t encode_asym(float w, float s, int32_t z) {
    if (!(s > 0.0f)) return z;
    const float r = rintf(w / s);
    const int32_t c = (int32_t)r + z;
    return c < 0 ? 0 : (c > 3 ? 3 : c);
}

static float sq_err_asym(float w, float s, int32_t z, int32_t c) {
    const float l = (float)(c - z) * s;
    const float e = w - l;
    return e * e;
}

int qo_quantize_weights_asym(const float* w, int64_t n_out, int64_t n_in, int32_t grid_points, double lo,
                             double hi, uint32_t* codes, float* scales, int32_t* zeros, double* row_mse,
                             int32_t* best_k) {
    if (!w || !codes || !scales || !zeros || n_out < 0 || n_in <= 0 || (n_in % 16) != 0) return -1;
    if (grid_points < 2 || grid_points > 4096) return -1;
    const int64_t words = n_in / 16;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < n_out; ++n) {
        const float* row = w + n * n_in;
        float lo_w = 0.0f, hi_w = 0.0f;
        for (int64_t k = 0; k < n_in; ++k) {
            if (row[k] < lo_w) lo_w = row[k];
            if (row[k] > hi_w) hi_w = row[k];
        }
        int32_t kbest = 0;
        double best = 0.0;
        for (int32_t g = 0; g < grid_points; ++g) {
            const double f = lo + ((hi - lo) * (double)g) / (double)(grid_points - 1);
            const float s = (float)((f * ((double)hi_w - (double)lo_w)) / 3.0);
            const int32_t z = asym_zero(f, lo_w, s);
            double acc = 0.0;
            for (int64_t k = 0; k < n_in; ++k) acc += (double)sq_err_asym(row[k], s, z, encode_asym(row[k], s, z));
            if (g == 0 || acc < best) {
                best = acc;
                kbest = g;
            }
        }
        const double f = lo + ((hi - lo) * (double)kbest) / (double)(grid_points - 1);
        const float s = (float)((f * ((double)hi_w - (double)lo_w)) / 3.0);
        const int32_t z = asym_zero(f, lo_w, s);
        uint32_t* out = codes + n * words;
        for (int64_t j = 0; j < words; ++j) out[j] = 0u;
        for (int64_t k = 0; k < n_in; ++k) out[k / 16] |= (uint32_t)encode_asym(row[k], s, z) << (2 * (k % 16));
        scales[n] = s;
        zeros[n] = z;
        if (row_mse) row_mse[n] = best / (double)n_in;
        if (best_k) best_k[n] = kbest;
    }
    return 0;
}

/* Asymmetric W2A4 linear: acc[t][n] = sum_k q[t][k] * (c[n][k] - z[n]) exactly (int64, must fit
 * int32), then y = ((float)acc * s_w[n]) * s_a[t] (R13).  acc and y may be NULL. */
int qo_linear_asym(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, const int32_t* zeros,
                   int64_t tokens, int64_t n_out, int64_t n_in, int32_t* acc_out, float* y) {
    if (!q || !s_a || !codes || !s_w || !zeros || tokens < 0 || n_out < 0 || n_in <= 0 || (n_in % 16) != 0)
        return -1;
    const int64_t words = n_in / 16;
    int overflow = 0;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t t = 0; t < tokens; ++t) {
        for (int64_t n = 0; n < n_out; ++n) {
            int64_t sum = 0;
            for (int64_t k = 0; k < n_in; ++k) {
                const int32_t c = (int32_t)((codes[n * words + k / 16] >> (2 * (k % 16))) & 3u);
                sum += (int64_t)q[t * n_in + k] * (int64_t)(c - zeros[n]);
            }
            if (sum > INT32_MAX || sum < INT32_MIN) {
#pragma omp atomic write
                overflow = 1;
            }
            if (acc_out) acc_out[t * n_out + n] = (int32_t)sum;
            if (y) y[t * n_out + n] = ((float)sum * s_w[n]) * s_a[t];
        }
    }
    return overflow ? -3 : 0;
}

/* ---------------------------------------------------------------------------------------
 * Symmetric per-token INT4 activation quantization (the "A4" of W2A4 in the Abstract).
 * Input: the rotated activations after their single rounding to binary16, given here as
 * the binary32 values of those binary16 numbers.
 *   m = max_k |x[t][k]| (binary32);  inv = 7.0f / m (one binary32 division);
 *   q = clamp(round_half_even(x * inv), -7, 7);  s_a[t] = m / 7.0f.
 * R11: round half to even, the symmetric range [-7, 7] (no -8), multiply by the inverse.
 * R12: m = 0 gives s_a = 0 and q = 0 everywhere.
 * ------------------------------------------------------------------------------------- */
int qo_quantize_acts(const float* x, int64_t tokens, int64_t n_in, int8_t* q, float* scales) {
    if (!x || !q || !scales || tokens < 0 || n_in <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < tokens; ++t) {
        const float* row = x + t * n_in;
        float m = 0.0f;
        for (int64_t k = 0; k < n_in; ++k) {
            float a = fabsf(row[k]);
            if (a > m) m = a;
        }
        int8_t* qr = q + t * n_in;
        if (m == 0.0f) {
            for (int64_t k = 0; k < n_in; ++k) qr[k] = 0;
            scales[t] = 0.0f;
            continue;
        }
        const float inv = 7.0f / m;
        for (int64_t k = 0; k < n_in; ++k) {
            float v = rintf(row[k] * inv); /* default rounding mode: nearest, ties to even */
            if (v > 7.0f) v = 7.0f;
            if (v < -7.0f) v = -7.0f;
            qr[k] = (int8_t)v;
        }
        scales[t] = m / 7.0f;
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * KV4 (the title's "Rotated W2A4/KV4 LLM Inference"): keys and values kept in 4 bits.  The page
 * gives no scheme; the reading used here is the activation path's -- the K or V row of a token
 * is Hadamard-rotated by blocks of the head dimension and quantized to symmetric per-token INT4
 * (qo_quantize_acts) -- with the codes stored two per byte.
 *   pack:   byte j of a row = (q[2j] & 0xF) | ((q[2j+1] & 0xF) << 4)  (two's-complement nibbles,
 *           the lower index in the low nibble);
 *   unpack: the inverse, sign-extending each nibble;
 *   dequantize: x = (float)q * s (one binary32 multiply), then the inverse rotation, which for
 *           the normalised Sylvester matrix is the rotation itself (H/sqrt(b) is symmetric and
 *           orthogonal): qo_rotate_f32's stages and final multiply.  The caller rounds to fp16.
 * ------------------------------------------------------------------------------------- */
int qo_pack_int4(const int8_t* q, int64_t n, uint8_t* out) {
    if (!q || !out || n < 0 || (n & 1)) return -1;
    for (int64_t j = 0; j < n / 2; ++j)
        out[j] = (uint8_t)(((uint8_t)q[2 * j] & 0xFu) | (((uint8_t)q[2 * j + 1] & 0xFu) << 4));
    return 0;
}

int qo_unpack_int4(const uint8_t* p, int64_t n, int8_t* q) {
    if (!p || !q || n < 0 || (n & 1)) return -1;
    for (int64_t j = 0; j < n / 2; ++j) {
        const int lo = p[j] & 0xF, hi = p[j] >> 4;
        q[2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
        q[2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
    }
    return 0;
}

int qo_dequantize_kv(const uint8_t* packed, const float* scales, int64_t tokens, int64_t n, int32_t b,
                     float* out) {
    if (!packed || !scales || !out || tokens < 0 || n <= 0 || (n & 1)) return -1;
    if (b != 0 && (!is_pow2(b) || (n % b) != 0)) return -1;
    for (int64_t t = 0; t < tokens; ++t) {
        int8_t* q = (int8_t*)malloc((size_t)n);
        if (!q) return -2;
        qo_unpack_int4(packed + t * (n / 2), n, q);
        for (int64_t k = 0; k < n; ++k) out[t * n + k] = (float)q[k] * scales[t];
        free(q);
    }
    if (b != 0) return qo_rotate_f32(out, tokens, n, b);
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * W2A4 linear (Abstract: "sign-and-shift decoded weight application").
 *   acc[t][n] = sum_k q[t][k] * L(code[n][k])   (exact integer arithmetic, int64 here;
 *                                                 the result must fit int32)
 *   y[t][n]   = ((float)acc * s_w[n]) * s_a[t]   (R13: binary32, left to right)
 * L is the integer level table of the set.  acc (int32) and y (binary32) may be NULL.
 * Returns -3 when an accumulator does not fit in int32.
 * ------------------------------------------------------------------------------------- */
int qo_linear(const int8_t* q, const float* s_a, const uint32_t* codes, const float* s_w, int32_t set,
              int64_t tokens, int64_t n_out, int64_t n_in, int32_t* acc, float* y) {
    if (!q || !codes || set < 0 || set > 2 || tokens < 0 || n_out < 0 || n_in <= 0 || (n_in % 16) != 0)
        return -1;
    if (y && (!s_a || !s_w)) return -1;
    const int64_t words = n_in / 16;
    int overflow = 0;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_out; ++n) {
        const uint32_t* crow = codes + n * words;
        for (int64_t t = 0; t < tokens; ++t) {
            const int8_t* qr = q + t * n_in;
            int64_t sum = 0;
            for (int64_t k = 0; k < n_in; ++k) {
                int32_t c = (int32_t)((crow[k / 16] >> (2 * (k % 16))) & 3u);
                sum += (int64_t)qr[k] * (int64_t)LEVELS[set][c];
            }
            if (sum > INT32_MAX || sum < INT32_MIN) {
#pragma omp atomic write
                overflow = 1;
            }
            if (acc) acc[t * n_out + n] = (int32_t)sum;
            if (y) {
                float v = (float)(int32_t)sum;
                v = v * s_w[n];
                v = v * s_a[t];
                y[t * n_out + n] = v;
            }
        }
    }
    return overflow ? -3 : 0;
}

/* Host threads for the OpenMP loops above: n > 0 sets the count for later calls; returns the
 * count now in force.  (Timing control only; no arithmetic depends on it.) */
int qo_set_threads(int n) {
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
}
