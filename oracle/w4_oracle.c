/*
 * w4_oracle.c -- CPU oracle for blockwise 4-bit weight quantization and the matmuls that
 * consume it.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark load this file's library. It shares no code, header, table or constant with
 * the CUDA library; the only inputs both sides see come from the seeded generators.
 *
 * Plain scalar C, built with -O2 -ffp-contract=off and no fast-math, so every fp32
 * operation below is one IEEE-754 single-precision operation in the written order.
 * OpenMP is used only across independent rows.
 *
 * Sources (page title, section):
 *   [P2] "Quantizing LLMs Without Guesswork: What 4 Bits Really Cost" -- "Scale and zero
 *        point" (symmetric and asymmetric formulas, error <= scale/2), "Granularity"
 *        (group-wise scales along a row, FP16 scale per group), "Quantize, then dequantize"
 *        (fake_quant: zero-range guard scale=1, np.round = half-to-even; rel_error;
 *        bits_per_weight).
 *   [P3] "Four-bit inference ... Tahoma" -- "The naive symmetric baseline" (a/7, code -8
 *        unused), "Achievement 1: asymmetric W4" (unsigned codes 0..15, integer zero point,
 *        groups of 128 along K, 16-bit scale and 16-bit zero term), "MSE clipping"
 *        (per-block search over ranges contracted about the midpoint, strict improvement,
 *        error over the whole block including clipped values), "Achievement 2: 8-bit
 *        activations" (per-row E4M3 scale from the row max-abs over 448, 1e-8 floor,
 *        all-zero rows stay zero), the W4A8 dataflow list (FP32 accumulation, per-token
 *        scale in the epilogue, BF16 result).
 *   [P5] "The outlier problem that reshaped how we quantize LLMs" -- symmetric INT8 formula,
 *        error bound scale/2, quantize_blocked.
 *   FP8 E4M3 ("FP8 Formats for Deep Learning", as summarised by [P2] "Number formats"):
 *        4 exponent bits (bias 7), 3 mantissa bits, no infinities, max finite 448.
 *
 * Readings where the pages are silent or garbled (each also listed in the design notes):
 *   R2/R3  the block scale is rounded to its 16-bit storage type (IEEE binary16, RNE) first,
 *          and codes, zero point and reconstruction error all use the stored value.
 *   R3     asymmetric contraction about the midpoint: h = 0.5*(hi-lo), c = (1-r)*h,
 *          lo_r = lo + c, hi_r = hi - c (r = 1 leaves lo, hi untouched); zero point is
 *          rint(-lo_r/s) saturated to int16 and not clamped to [0,15].
 *   R4     rint = round half to even everywhere.
 *   R5     the block error is a sum of squares (same argmin as the mean) reduced in a fixed
 *          tree: 32 contiguous chunks of g/32 elements summed left to right, then the 32
 *          partials combined pairwise at distances 16, 8, 4, 2, 1; ties keep the earlier ratio.
 *   R7     per-row activation scale s = max(amax, 1e-8) / 448, codes = e4m3(x / s) with RNE
 *          and saturation to +-448.
 *   Symmetric codes are stored offset-binary: nibble = c + 8, c in [-7, 7].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------ number formats */

/* bf16 bit pattern -> fp32 (exact: bf16 is the upper half of an fp32). */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

EXPORT float o_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }

/* IEEE binary16, round to nearest even, written out from the format definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; subnormal quantum 2^-24;
 * largest finite 65504; values at or above the midpoint 65520 round to infinity. */
EXPORT uint16_t o_f32_to_f16_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if (isnan(f)) return (uint16_t)(sign | 0x7E00u);
    double a = fabs((double)f);
    if (a >= 65520.0) return (uint16_t)(sign | 0x7C00u);
    if (a < ldexp(1.0, -14)) {                 /* subnormal range: multiples of 2^-24 */
        double m = rint(a / ldexp(1.0, -24));  /* a / 2^-24 is exact in double */
        return (uint16_t)(sign | (uint16_t)m); /* m == 1024 encodes the smallest normal */
    }
    int ex;
    frexp(a, &ex);                 /* a = fr * 2^ex, fr in [0.5, 1) */
    int E = ex - 1;                /* a in [2^E, 2^(E+1)), E in [-14, 15] */
    double m = rint(a / ldexp(1.0, E - 10)); /* in [1024, 2048] */
    uint32_t bits = ((uint32_t)(E + 15) << 10) + (uint32_t)(m - 1024.0); /* carry is fine */
    return (uint16_t)(sign | bits);
}

EXPORT float o_f16_bits_to_f32(uint16_t h) {
    int sign = (h >> 15) & 1;
    int E = (h >> 10) & 0x1F;
    int M = h & 0x3FF;
    double v;
    if (E == 0) v = ldexp((double)M, -24);
    else if (E == 31) v = M ? NAN : INFINITY;
    else v = ldexp(1024.0 + M, E - 25);
    return (float)(sign ? -v : v);
}

static float f16_round(float x) { return o_f16_bits_to_f32(o_f32_to_f16_bits(x)); }

/* FP8 E4M3 (the "fn" variant: no infinities): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits. Subnormals (exponent field 0) are m * 2^-9; normals are (8 + m) * 2^(E-10).
 * Exponent 15 with mantissa 7 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.
 * Encoding: round to nearest even, then saturate to +-448 ("satfinite"). */
EXPORT uint8_t o_e4m3_encode(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x)) return (uint8_t)(sign | 0x7F);
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {                     /* subnormal: multiples of 2^-9 */
        double m = rint(a / ldexp(1.0, -9));      /* m == 8 encodes the smallest normal */
        return (uint8_t)(sign | (uint8_t)m);
    }
    int ex;
    frexp(a, &ex);
    int E = ex - 1;                               /* a in [2^E, 2^(E+1)), E in [-6, 8] */
    double m = rint(a / ldexp(1.0, E - 3));       /* in [8, 16] */
    uint32_t bits = ((uint32_t)(E + 7) << 3) + (uint32_t)(m - 8.0);
    return (uint8_t)(sign | bits);                /* a < 448 keeps bits <= 0x7E */
}

EXPORT float o_e4m3_decode(uint8_t b) {
    int sign = (b >> 7) & 1;
    int E = (b >> 3) & 0xF;
    int M = b & 7;
    double v;
    if (E == 15 && M == 7) v = NAN;
    else if (E == 0) v = ldexp((double)M, -9);
    else v = ldexp(8.0 + M, E - 10);
    return (float)(sign ? -v : v);
}

/* ------------------------------------------------------------------ the block quantizer */

/* Block error: sum of squared errors in the fixed reduction tree (reading R5). */
static float sse_tree(const float *e2, int g) {
    float p[32], t[32];
    int chunk = g / 32;
    for (int c = 0; c < 32; ++c) {
        float acc = e2[c * chunk];
        for (int i = 1; i < chunk; ++i) acc = acc + e2[c * chunk + i];
        p[c] = acc;
    }
    for (int off = 16; off >= 1; off >>= 1) {
        for (int j = 0; j < 32; ++j) t[j] = p[j] + p[j ^ off];
        for (int j = 0; j < 32; ++j) p[j] = t[j];
    }
    return p[0];
}

static int16_t sat_i16(float v) {
    if (v > 32767.0f) return 32767;
    if (v < -32768.0f) return -32768;
    return (int16_t)v;
}

/* One candidate of the clip search for one block of g weights.
 * Symmetric ([P2] "Scale and zero point", [P3] "The naive symmetric baseline"):
 *   a = max|w|, a_r = r*a, s = fp16(a_r / 7), s == 0 -> 1,
 *   c = clamp(rint(w / s), -7, 7), stored nibble c + 8, reconstruction c * s.
 * Asymmetric ([P2] "Scale and zero point", [P3] "Achievement 1", "MSE clipping"):
 *   range [lo, hi] contracted about its midpoint by r, s = fp16((hi_r - lo_r) / 15),
 *   s == 0 -> 1, z = rint(-lo_r / s), q = clamp(rint(w / s) + z, 0, 15),
 *   reconstruction (q - z) * s.
 * Returns the block's sum of squared errors; writes nibbles, scale bits and zero. */
static float candidate(const float *w, int g, int asym, float r, float lo, float hi, float amax,
                       uint8_t *nib, uint16_t *s_bits, int16_t *z_out, float *e2) {
    float s;
    int16_t z = 0;
    if (!asym) {
        float a_r = r * amax;
        s = f16_round(a_r / 7.0f);
        if (s == 0.0f) s = 1.0f;
        for (int k = 0; k < g; ++k) {
            float c = rintf(w[k] / s);
            if (c > 7.0f) c = 7.0f;
            if (c < -7.0f) c = -7.0f;
            nib[k] = (uint8_t)((int)c + 8);
            float rec = c * s;
            float e = w[k] - rec;
            e2[k] = e * e;
        }
        z = 8;
    } else {
        float h = 0.5f * (hi - lo);
        float cc = (1.0f - r) * h;
        float lo_r = lo + cc;
        float hi_r = hi - cc;
        s = f16_round((hi_r - lo_r) / 15.0f);
        if (s == 0.0f) s = 1.0f;
        z = sat_i16(rintf(-lo_r / s));
        for (int k = 0; k < g; ++k) {
            float q = rintf(w[k] / s) + (float)z;
            if (q > 15.0f) q = 15.0f;
            if (q < 0.0f) q = 0.0f;
            nib[k] = (uint8_t)q;
            float rec = (float)((int)q - (int)z) * s;
            float e = w[k] - rec;
            e2[k] = e * e;
        }
    }
    *s_bits = o_f32_to_f16_bits(s);
    *z_out = z;
    return sse_tree(e2, g);
}

/* Quantize one block with the clip search ([P3] "MSE clipping"): the first grid ratio is the
 * incumbent, a later ratio replaces it only with a strictly smaller error. */
static void quantize_block(const float *w, int g, int asym, const float *grid, int ngrid,
                           uint8_t *nib_out, uint16_t *s_out, int16_t *z_out, uint8_t *idx_out) {
    float lo = w[0], hi = w[0], amax = fabsf(w[0]);
    for (int k = 1; k < g; ++k) {
        if (w[k] < lo) lo = w[k];
        if (w[k] > hi) hi = w[k];
        if (fabsf(w[k]) > amax) amax = fabsf(w[k]);
    }
    uint8_t nib[256];
    float e2[256];
    float best = 0.0f;
    for (int i = 0; i < ngrid; ++i) {
        uint16_t sb;
        int16_t z;
        float sse = candidate(w, g, asym, grid[i], lo, hi, amax, nib, &sb, &z, e2);
        if (i == 0 || sse < best) {
            best = sse;
            memcpy(nib_out, nib, (size_t)g);
            *s_out = sb;
            *z_out = z;
            *idx_out = (uint8_t)i;
        }
    }
}

/* Row-major W[N,K] (bf16 bits) -> packed codes [N, K/2] (byte j = q[2j] | q[2j+1] << 4),
 * fp16 scales [N, K/g], int16 zeros [N, K/g] (asym; may be NULL for sym), chosen ratio
 * index [N, K/g] (may be NULL). Groups are g consecutive weights along K inside a row. */
EXPORT int o_quantize(const uint16_t *W, int64_t N, int64_t K, int g, int asym,
                      const float *grid, int ngrid, uint8_t *codes, uint16_t *scales,
                      int16_t *zeros, uint8_t *chosen) {
    if (g != 32 && g != 64 && g != 128 && g != 256) return 1;
    if (K % g != 0 || K % 2 != 0 || ngrid < 1) return 1;
    int64_t J = K / g;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        float w[256];
        uint8_t nib[256];
        for (int64_t j = 0; j < J; ++j) {
            for (int k = 0; k < g; ++k) w[k] = bf16_to_f32(W[n * K + j * g + k]);
            uint16_t s;
            int16_t z;
            uint8_t idx;
            quantize_block(w, g, asym, grid, ngrid, nib, &s, &z, &idx);
            scales[n * J + j] = s;
            if (zeros) zeros[n * J + j] = asym ? z : 8;
            if (chosen) chosen[n * J + j] = idx;
            for (int k = 0; k < g; k += 2)
                codes[n * (K / 2) + (j * g + k) / 2] = (uint8_t)(nib[k] | (nib[k + 1] << 4));
        }
    }
    return 0;
}

/* Candidate error of one block for one ratio, exposed for the brute-force tests. */
EXPORT float o_block_sse(const uint16_t *wb, int g, int asym, float r) {
    float w[256], e2[256];
    uint8_t nib[256];
    float lo, hi, amax;
    for (int k = 0; k < g; ++k) w[k] = bf16_to_f32(wb[k]);
    lo = hi = w[0];
    amax = fabsf(w[0]);
    for (int k = 1; k < g; ++k) {
        if (w[k] < lo) lo = w[k];
        if (w[k] > hi) hi = w[k];
        if (fabsf(w[k]) > amax) amax = fabsf(w[k]);
    }
    uint16_t sb;
    int16_t z;
    return candidate(w, g, asym, r, lo, hi, amax, nib, &sb, &z, e2);
}

/* Dequantize: W'[n,k] = (q - z) * s in double (exact: |q - z| < 2^16, s has 11 bits). */
EXPORT void o_dequantize(const uint8_t *codes, const uint16_t *scales, const int16_t *zeros,
                         int64_t N, int64_t K, int g, int asym, double *out) {
    int64_t J = K / g;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[n * (K / 2) + k / 2];
            int q = (k & 1) ? (byte >> 4) : (byte & 0xF);
            int z = asym ? zeros[n * J + k / g] : 8;
            double s = (double)o_f16_bits_to_f32(scales[n * J + k / g]);
            out[n * K + k] = (double)(q - z) * s;
        }
    }
}

/* ------------------------------------------------------------------ activation row quant */

/* Per-row FP8 E4M3 ([P3] "Achievement 2"): amax = max|x| of the row,
 * s = max(amax, 1e-8) / 448, codes = e4m3(x / s). Also the per-group sums of the E4M3
 * values G[m, j] = sum_{k in group j} e4m3val(code[m,k]), summed exactly (every E4M3 value
 * is an integer multiple of 2^-9 and a group of <= 128 of them is below 2^25 * 2^-9) and
 * rounded once to fp32. */
/* Row quant of one row of K fp32 values: amax, s = max(amax, 1e-8) / 448, codes e4m3(x / s),
 * and the exact per-group sums of the E4M3 values when g > 0. */
static void row_quant_one(const float *x, int64_t K, int g, uint8_t *X8, float *row_scale, float *gsum) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(x[k]);
        if (a > amax) amax = a;
    }
    float floor_amax = amax > 1e-8f ? amax : 1e-8f;
    float s = floor_amax / 448.0f;
    *row_scale = s;
    for (int64_t k = 0; k < K; ++k) X8[k] = o_e4m3_encode(x[k] / s);
    if (gsum && g > 0) {
        for (int64_t j = 0; j < K / g; ++j) {
            int64_t acc = 0; /* exact sum in units of 2^-9 */
            for (int k = 0; k < g; ++k) {
                double v = (double)o_e4m3_decode(X8[j * g + k]);
                acc += (int64_t)llrint(v * 512.0);
            }
            gsum[j] = (float)ldexp((double)acc, -9);
        }
    }
}

/* Per-row FP8 E4M3 ([P3] "Achievement 2"): amax = max|x| of the row,
 * s = max(amax, 1e-8) / 448, codes = e4m3(x / s). Also the per-group sums of the E4M3 values
 * G[m, j] = sum_{k in group j} e4m3val(code[m,k]), summed exactly (every E4M3 value is an
 * integer multiple of 2^-9 and a group of <= 128 of them is below 2^25 * 2^-9) and rounded
 * once to fp32. */
EXPORT void o_row_quant(const uint16_t *X, int64_t M, int64_t K, int g, uint8_t *X8,
                        float *row_scale, float *gsum) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float *x = (float *)malloc((size_t)K * sizeof(float));
        for (int64_t k = 0; k < K; ++k) x[k] = bf16_to_f32(X[m * K + k]);
        row_quant_one(x, K, g, X8 + m * K, row_scale + m, gsum ? gsum + m * (K / (g > 0 ? g : 1)) : NULL);
        free(x);
    }
}

/* ------------------------------------------------------------------ mixture-of-experts layer */

/* Router ("4-bit by default", the MoE expert weights of gpt-oss; the pages leave the router
 * open): the k largest logits of each token in descending order, equal logits taken in
 * ascending expert order; gate weights are the softmax of the k selected logits (fp64). */
EXPORT void o_moe_route(const float *logits, int64_t T, int E, int k, int32_t *experts, double *gates) {
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        unsigned char taken[1024];
        memset(taken, 0, sizeof(taken));
        for (int i = 0; i < k; ++i) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
            taken[best] = 1;
            experts[t * k + i] = best;
        }
        double mx = l[experts[t * k]], den = 0.0;
        for (int i = 0; i < k; ++i) den += exp((double)l[experts[t * k + i]] - mx);
        for (int i = 0; i < k; ++i) gates[t * k + i] = exp((double)l[experts[t * k + i]] - mx) / den;
    }
}

/* SwiGLU between the two expert projections, then the per-row E4M3 quantization of the
 * down projection's input. A row of the gate_up output holds [gate (H) | up (H)] (bf16);
 * h = silu(gate) * up = gate * up / (1 + exp(-gate)), evaluated in fp64 and rounded to fp32
 * (the precision in which the GPU quantizes it), then the row quant above. h_out (may be
 * NULL) receives the fp32 h. */
EXPORT void o_swiglu_row_quant(const uint16_t *Y, int64_t R, int64_t H, uint8_t *X8, float *row_scale,
                               float *h_out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        float *h = (float *)malloc((size_t)H * sizeof(float));
        for (int64_t j = 0; j < H; ++j) {
            double gv = (double)bf16_to_f32(Y[r * 2 * H + j]);
            double uv = (double)bf16_to_f32(Y[r * 2 * H + H + j]);
            h[j] = (float)(gv * uv / (1.0 + exp(-gv)));
        }
        row_quant_one(h, H, 0, X8 + r * H, row_scale + r, NULL);
        if (h_out) memcpy(h_out + r * H, h, (size_t)H * sizeof(float));
        free(h);
    }
}

/* Weighted combine of the experts' outputs: y[t, n] = sum_i gates[t, i] * rows[row_of[t, i], n]
 * (fp64), rows being the down projection's outputs in expert-grouped order. */
EXPORT void o_moe_combine(const double *rows, int64_t N, const int32_t *row_of, const double *gates, int64_t T,
                          int k, double *y) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int i = 0; i < k; ++i) acc += gates[t * k + i] * rows[(int64_t)row_of[t * k + i] * N + n];
            y[t * N + n] = acc;
        }
}

/* ------------------------------------------------------------------ reference products */

/* W4A16 GEMV reference: y[m,n] = sum_k x[m,k] * (q[n,k] - z[n,j]) * s[n,j] in double. */
EXPORT void o_gemv_ref(const uint16_t *x, int64_t M, const uint8_t *codes, const uint16_t *scales,
                       const int16_t *zeros, int64_t N, int64_t K, int g, int asym, double *y) {
    int64_t J = K / g;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                uint8_t byte = codes[n * (K / 2) + k / 2];
                int q = (k & 1) ? (byte >> 4) : (byte & 0xF);
                int z = asym ? zeros[n * J + k / g] : 8;
                double w = (double)(q - z) * (double)o_f16_bits_to_f32(scales[n * J + k / g]);
                acc += (double)bf16_to_f32(x[m * K + k]) * w;
            }
            y[m * N + n] = acc;
        }
    }
}

/* W4A8 reference on chosen outputs: Y[m,n] = sum_k (e4m3val(X8[m,k]) * s_a[m]) *
 * ((q[n,k] - z[n,j]) * s_w[n,j]) in double -- the product of the two dequantized operands.
 * rows/cols list the (m, n) pairs to evaluate (count entries). Packed weights of expert e
 * start at codes + e*N*K/2 etc. when expert_of_row is given (NULL: one weight). */
EXPORT void o_w4a8_ref_pairs(const uint8_t *X8, const float *s_a, int64_t K, const uint8_t *codes,
                             const uint16_t *scales, const int16_t *zeros, int64_t N, int g,
                             int asym, const int32_t *expert_of_row, const int64_t *rows,
                             const int64_t *cols, int64_t count, double *out) {
    int64_t J = K / g;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = rows[i], n = cols[i];
        int64_t e = expert_of_row ? expert_of_row[m] : 0;
        const uint8_t *cw = codes + e * N * (K / 2);
        const uint16_t *sw = scales + e * N * J;
        const int16_t *zw = zeros ? zeros + e * N * J : NULL;
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = cw[n * (K / 2) + k / 2];
            int q = (k & 1) ? (byte >> 4) : (byte & 0xF);
            int z = asym ? zw[n * J + k / g] : 8;
            double w = (double)(q - z) * (double)o_f16_bits_to_f32(sw[n * J + k / g]);
            double a = (double)o_e4m3_decode(X8[m * K + k]) * (double)s_a[m];
            acc += a * w;
        }
        out[i] = acc;
    }
}

/* ------------------------------------------------------------------ generic fake quant */

/* A b-bit uniform quantizer of one block is a lattice: integer codes c in [c_lo, c_hi], a
 * step (the scale) and an integer offset (the zero point, 0 for symmetric codes). A value v
 * goes to c = clamp(rint(v / step) + offset, c_lo, c_hi) and comes back as (c - offset) * step.
 * [P2] "Scale and zero point" fixes the lattice of a block from its extremes:
 *   symmetric   step = max|v| / (2^(b-1) - 1), codes -(2^(b-1) - 1) .. 2^(b-1) - 1
 *   asymmetric  step = (max - min) / (2^b - 1), offset = rint(-min / step), codes 0 .. 2^b - 1
 * and [P2] "Quantize, then dequantize" replaces a zero step (a constant block) by 1 before the
 * offset is formed; [P5] states the same symmetric lattice and its scale/2 error bound. */
typedef struct {
    double step, offset, c_lo, c_hi;
} lattice;

static lattice block_lattice(const double *v, int64_t len, int bits, int symmetric) {
    double lo = v[0], hi = v[0];
    for (int64_t i = 1; i < len; ++i) {
        lo = v[i] < lo ? v[i] : lo;
        hi = v[i] > hi ? v[i] : hi;
    }
    lattice L;
    if (symmetric) {
        L.c_hi = ldexp(1.0, bits - 1) - 1.0;
        L.c_lo = -L.c_hi;
        L.step = fmax(fabs(lo), fabs(hi)) / L.c_hi;
    } else {
        L.c_lo = 0.0;
        L.c_hi = ldexp(1.0, bits) - 1.0;
        L.step = (hi - lo) / L.c_hi;
    }
    if (L.step == 0.0) L.step = 1.0;
    L.offset = symmetric ? 0.0 : rint(-lo / L.step);
    return L;
}

static double lattice_round_trip(const lattice *L, double v) {
    double c = rint(v / L->step) + L->offset;
    c = c < L->c_lo ? L->c_lo : (c > L->c_hi ? L->c_hi : c);
    return (c - L->offset) * L->step;
}

/* Fake quantization of n doubles in blocks of `block` consecutive values (block = n for one
 * per-tensor scale; the last block may be shorter): every value goes through its block's
 * lattice. out receives the reconstructed values, scale_out (may be NULL) each block's step. */
EXPORT void o_fake_quant(const double *x, int64_t n, int64_t block, int bits, int symmetric,
                         double *out, double *scale_out) {
    for (int64_t b = 0; b * block < n; ++b) {
        const double *v = x + b * block;
        int64_t len = n - b * block < block ? n - b * block : block;
        lattice L = block_lattice(v, len, bits, symmetric);
        for (int64_t i = 0; i < len; ++i) out[b * block + i] = lattice_round_trip(&L, v[i]);
        if (scale_out) scale_out[b] = L.step;
    }
}

/* ------------------------------------------------------------------ NF4 comparator */

/* Inverse of the standard normal CDF, Phi(x) = erfc(-x / sqrt(2)) / 2: bisection to a
 * bracketing interval, then Newton steps on Phi(x) - p (Phi' is the normal density). */
static double inv_phi(double p) {
    double lo = -40.0, hi = 40.0;
    for (int i = 0; i < 200; ++i) {
        double mid = 0.5 * (lo + hi);
        if (0.5 * erfc(-mid / sqrt(2.0)) < p) lo = mid; else hi = mid;
    }
    double x = 0.5 * (lo + hi);
    for (int i = 0; i < 3; ++i) {
        double f = 0.5 * erfc(-x / sqrt(2.0)) - p;
        double d = exp(-0.5 * x * x) / sqrt(2.0 * 3.14159265358979323846);
        if (d > 0.0) x -= f / d;
    }
    return x;
}

/* NF4 levels ([P2] "Quantizing LLMs Without Guesswork", NF4 paragraph: 16 levels that are
 * quantiles of a normal distribution, blocks of 64). The pages leave the construction open;
 * this is the QLoRA one: with delta = (1/32 + 1/30) / 2, eight positive levels
 * Phi^-1(p) at p = 1 - delta + i (delta - 1/2) / 8, i = 0..7, seven negative levels
 * -Phi^-1(p) at p = 1 - delta + i (delta - 1/2) / 7, i = 0..6, and an exact zero, all divided
 * by Phi^-1(1 - delta) so that the extremes are -1 and 1; sorted ascending, rounded to fp32. */
EXPORT void o_nf4_levels(float *out) {
    const double delta = 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
    const double top = inv_phi(1.0 - delta);
    double v[16];
    int n = 0;
    for (int i = 0; i < 7; ++i) v[n++] = -inv_phi(1.0 - delta + i * (delta - 0.5) / 7.0) / top;
    v[n++] = 0.0;
    for (int i = 7; i >= 0; --i) v[n++] = inv_phi(1.0 - delta + i * (delta - 0.5) / 8.0) / top;
    /* ascending: the negatives were built from -1 upwards, the positives from the smallest */
    for (int i = 0; i < 16; ++i) out[i] = (float)v[i];
}

/* NF4 quantization of W[N, K] (bf16) in blocks of 64 along K: a = max|w| (fp32), stored as
 * the block's fp32 scale; each weight's code is the level nearest to w / a (fp32 IEEE
 * division, distances |w/a - level| in fp32, ties to the lower level); an all-zero block
 * has a = 0 and every code at the zero level. Codes packed as the INT4 ones: byte j of a
 * row = q[2j] | q[2j+1] << 4. */
EXPORT int o_nf4_quantize(const uint16_t *W, int64_t N, int64_t K, uint8_t *codes, float *absmax) {
    if (K % 64 != 0) return 1;
    float lv[16];
    o_nf4_levels(lv);
    int zero_code = 7;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < K / 64; ++b) {
            float w[64], a = 0.0f;
            for (int i = 0; i < 64; ++i) {
                w[i] = bf16_to_f32(W[n * K + b * 64 + i]);
                if (fabsf(w[i]) > a) a = fabsf(w[i]);
            }
            absmax[n * (K / 64) + b] = a;
            uint8_t q[64];
            for (int i = 0; i < 64; ++i) {
                if (a == 0.0f) { q[i] = (uint8_t)zero_code; continue; }
                float t = w[i] / a;
                int best = 0;
                float bd = fabsf(t - lv[0]);
                for (int c = 1; c < 16; ++c) {
                    float d = fabsf(t - lv[c]);
                    if (d < bd) { bd = d; best = c; }
                }
                q[i] = (uint8_t)best;
            }
            for (int i = 0; i < 64; i += 2)
                codes[n * (K / 2) + (b * 64 + i) / 2] = (uint8_t)(q[i] | (q[i + 1] << 4));
        }
    }
    return 0;
}

/* NF4 W4A16 GEMV reference: y[m, n] = sum_k x[m,k] * level[q[n,k]] * a[n, k/64] in fp64. */
EXPORT void o_nf4_gemv_ref(const uint16_t *x, int64_t M, const uint8_t *codes, const float *absmax, int64_t N,
                           int64_t K, double *y) {
    float lv[16];
    o_nf4_levels(lv);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                uint8_t byte = codes[n * (K / 2) + k / 2];
                int q = (k & 1) ? (byte >> 4) : (byte & 0xF);
                acc += (double)bf16_to_f32(x[m * K + k]) * (double)lv[q] * (double)absmax[n * (K / 64) + k / 64];
            }
            y[m * N + n] = acc;
        }
}
