// w4_quantize: group-wise INT4 quantizer with the data-free MSE clip search.
//
// "Quantizing LLMs Without Guesswork", Scale and zero point / Granularity / Quantize, then
// dequantize; "Four-bit inference ... Tahoma", The naive symmetric baseline, Achievement 1,
// MSE clipping.
//
// Eight lanes own one group of G weights (G = 32, 64, 128, 256), four groups per warp. The group
// is cut into 32 chunks of G/32 consecutive weights; lane j (0..7) of the group holds chunks
// j, j+8, j+16 and j+24. The group's min / max / max|w| come from shuffles (exact). Every
// clip ratio is evaluated in registers: scale rounded to fp16, zero point, codes,
// reconstruction and squared error. The block error follows the fixed tree of the search:
// each chunk summed in order, then pairs at distances 16 and 8 (inside the lane) and 4, 2, 1
// (across the group's lanes); every partial is a commutative fp32 sum of the same two
// values at both positions, so all eight lanes end with the same bits and the
// strict-improvement test is uniform over the group.
//
// The code of a weight needs rint(w / s) with the IEEE quotient. It is formed from the
// scale's reciprocal r = RN(1/s) by one exact correction step (Markstein 1990):
// q0 = w*r, e = fma(q0, s, -w), q = fma(-e, r, q0). An exhaustive host check
// (tests/quantizer_division_check.c) visits every finite bf16 w and every finite positive
// fp16 s with |w|*r < 2^126 and finds rint(q) equal to rint(w / s) everywhere; a block
// outside that range (max|w| * r >= 2^126, or an infinite scale) takes the IEEE division.
// The clamp is applied before the rounding (both bounds are integers, so the order does not
// matter) and rint is the round-to-nearest-even of adding and removing 1.5 * 2^23, exact for
// the clamped range. This translation unit is compiled with -fmad=false and spells every
// operation with an _rn intrinsic, so no multiply-add is ever contracted and the codes,
// scales and zeros are bit-identical to a plain IEEE evaluation of the formulas.
#include "w4_common.cuh"

namespace w4 {

struct ClipGrid {
    float r[64];
    int n;
};

__device__ __forceinline__ float f16_round(float x) { return __half2float(__float2half_rn(x)); }

__device__ __forceinline__ float sat_i16f(float v) { return fminf(fmaxf(v, -32768.0f), 32767.0f); }

// round to nearest even of a value in [-2^22, 2^22]
__device__ __forceinline__ float rint_small(float v) {
    return __fsub_rn(__fadd_rn(v, 12582912.0f), 12582912.0f);
}

// Quotient of w by the block scale as the clip search needs it: the IEEE quotient, or (fast
// path) the reciprocal-corrected one, which has the same rint.
template <bool FAST>
__device__ __forceinline__ float quot(float w, float s, float r) {
    if (FAST) {
        const float q0 = __fmul_rn(w, r);
        const float e = __fmaf_rn(q0, s, -w);
        return __fmaf_rn(-e, r, q0);
    }
    return __fdiv_rn(w, s);
}

// This lane's part of the block error for scale s, reciprocal r and code window
// [c_lo, c_hi] (the codes minus the zero point): its four chunks of C = E/4 weights, each
// summed in order, then the tree's pairs at distances 16 (chunks j, j+16 and j+8, j+24) and
// 8. The caller adds the group's lanes at distances 4, 2, 1.
template <int E, bool FAST>
__device__ __forceinline__ float lane_sse(const float (&w)[E], float s, float r, float c_lo, float c_hi) {
    constexpr int C = E / 4;
    float p[4];
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
        for (int i = 0; i < C; ++i) {
            const float v = fminf(fmaxf(quot<FAST>(w[ch * C + i], s, r), c_lo), c_hi);
            const float c = rint_small(v);
            const float err = __fsub_rn(w[ch * C + i], __fmul_rn(c, s));
            const float e2 = __fmul_rn(err, err);
            p[ch] = (i == 0) ? e2 : __fadd_rn(p[ch], e2);
        }
    }
    return __fadd_rn(__fadd_rn(p[0], p[2]), __fadd_rn(p[1], p[3]));
}

// q - z of one weight under the winning scale (integer-valued float)
template <bool FAST>
__device__ __forceinline__ float code_of(float w, float s, float r, float c_lo, float c_hi) {
    return rint_small(fminf(fmaxf(quot<FAST>(w, s, r), c_lo), c_hi));
}

template <int G, bool ASYM>
__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t *__restrict__ W, int64_t K,
                                                       int64_t total_groups, ClipGrid grid,
                                                       uint8_t *__restrict__ codes,
                                                       uint16_t *__restrict__ scales,
                                                       int16_t *__restrict__ zeros,
                                                       uint8_t *__restrict__ chosen) {
    constexpr int C = G / 32;  // weights per chunk
    constexpr int E = 4 * C;   // weights per lane
    const int lane = threadIdx.x & 31, j = lane & 7;
    const int64_t J = K / G;
    const int64_t slots = (int64_t)gridDim.x * (blockDim.x >> 5) * 4;
    for (int64_t gid = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4 + (lane >> 3);
         gid - (lane >> 3) < total_groups; gid += slots) {
        const bool live = gid < total_groups;
        const int64_t n = gid / J, jj = gid - n * J;
        const uint16_t *src = W + n * K + jj * G;
        float w[E];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            const uint16_t *cs = src + (j + 8 * ch) * C;
            if constexpr (C == 8) {
                const uint4 v = live ? *reinterpret_cast<const uint4 *>(cs) : make_uint4(0u, 0u, 0u, 0u);
                w[ch * 8 + 0] = bf16_lo(v.x); w[ch * 8 + 1] = bf16_hi(v.x);
                w[ch * 8 + 2] = bf16_lo(v.y); w[ch * 8 + 3] = bf16_hi(v.y);
                w[ch * 8 + 4] = bf16_lo(v.z); w[ch * 8 + 5] = bf16_hi(v.z);
                w[ch * 8 + 6] = bf16_lo(v.w); w[ch * 8 + 7] = bf16_hi(v.w);
            } else if constexpr (C == 4) {
                const uint2 v = live ? *reinterpret_cast<const uint2 *>(cs) : make_uint2(0u, 0u);
                w[ch * 4 + 0] = bf16_lo(v.x); w[ch * 4 + 1] = bf16_hi(v.x);
                w[ch * 4 + 2] = bf16_lo(v.y); w[ch * 4 + 3] = bf16_hi(v.y);
            } else if constexpr (C == 2) {
                const uint32_t v = live ? *reinterpret_cast<const uint32_t *>(cs) : 0u;
                w[ch * 2 + 0] = bf16_lo(v); w[ch * 2 + 1] = bf16_hi(v);
            } else {
                w[ch] = __uint_as_float(((uint32_t)(live ? cs[0] : 0)) << 16);
            }
        }
        float lo = w[0], hi = w[0], amax = fabsf(w[0]);
#pragma unroll
        for (int e = 1; e < E; ++e) {
            lo = fminf(lo, w[e]);
            hi = fmaxf(hi, w[e]);
            amax = fmaxf(amax, fabsf(w[e]));
        }
#pragma unroll
        for (int off = 4; off >= 1; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(FULL, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(FULL, hi, off));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, off));
        }

        float best_sse = 0.0f, best_s = 1.0f, best_z = 8.0f;
        int best_i = 0;
        for (int i = 0; i < grid.n; ++i) {
            const float rr = grid.r[i];
            float s, zf;
            if constexpr (!ASYM) {
                const float a_r = __fmul_rn(rr, amax);
                s = f16_round(__fdiv_rn(a_r, 7.0f));
                if (s == 0.0f) s = 1.0f;
                zf = 8.0f;
            } else {
                const float h = __fmul_rn(0.5f, __fsub_rn(hi, lo));
                const float cc = __fmul_rn(__fsub_rn(1.0f, rr), h);
                const float lo_r = __fadd_rn(lo, cc);
                const float hi_r = __fsub_rn(hi, cc);
                s = f16_round(__fdiv_rn(__fsub_rn(hi_r, lo_r), 15.0f));
                if (s == 0.0f) s = 1.0f;
                zf = sat_i16f(rintf(__fdiv_rn(-lo_r, s)));
            }
            // code window of c = q - z: [-7, 7] symmetric, [-z, 15 - z] asymmetric
            const float c_lo = ASYM ? -zf : -7.0f, c_hi = ASYM ? __fsub_rn(15.0f, zf) : 7.0f;
            const float r = __frcp_rn(s);
            const bool fast = s <= 65504.0f && __fmul_rn(amax, r) < 0x1p126f;
            float sse = fast ? lane_sse<E, true>(w, s, r, c_lo, c_hi) : lane_sse<E, false>(w, s, r, c_lo, c_hi);
#pragma unroll
            for (int off = 4; off >= 1; off >>= 1) sse = __fadd_rn(sse, __shfl_xor_sync(FULL, sse, off));
            if (i == 0 || sse < best_sse) {
                best_sse = sse;
                best_s = s;
                best_z = zf;
                best_i = i;
            }
        }

        // codes of the winning ratio, q = c + z (symmetric: c + 8)
        const float r = __frcp_rn(best_s);
        const bool fast = best_s <= 65504.0f && __fmul_rn(amax, r) < 0x1p126f;
        const float c_lo = ASYM ? -best_z : -7.0f, c_hi = ASYM ? __fsub_rn(15.0f, best_z) : 7.0f;
        const int zi = (int)best_z;
        uint32_t qv[4] = {0u, 0u, 0u, 0u};  // per chunk, nibble i at bits [4i, 4i+4)
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
            for (int i = 0; i < C; ++i) {
                const float wv = w[ch * C + i];
                const float c = fast ? code_of<true>(wv, best_s, r, c_lo, c_hi) : code_of<false>(wv, best_s, r, c_lo, c_hi);
                qv[ch] |= ((uint32_t)((int)c + zi) & 0xFu) << (4 * i);
            }
        }
        if constexpr (C == 1) {
            // chunk j+8ch is the single weight j+8ch; weights 2m, 2m+1 sit in lanes j, j+1 of
            // the group (j even): the even lane takes its neighbour's nibble
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) qv[ch] |= (__shfl_down_sync(FULL, qv[ch], 1) & 0xFu) << 4;
        }
        if (live) {
            uint8_t *dst = codes + n * (K / 2) + (jj * G) / 2;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int c0 = (j + 8 * ch) * C;  // first weight of the chunk
                if constexpr (C == 8) reinterpret_cast<uint32_t *>(dst)[c0 / 8] = qv[ch];
                else if constexpr (C == 4) reinterpret_cast<uint16_t *>(dst)[c0 / 4] = (uint16_t)qv[ch];
                else if constexpr (C == 2) dst[c0 / 2] = (uint8_t)qv[ch];
                else if ((j & 1) == 0) dst[c0 / 2] = (uint8_t)qv[ch];
            }
            if (j == 0) {
                scales[gid] = __half_as_ushort(__float2half_rn(best_s));
                if (ASYM) zeros[gid] = (int16_t)best_z;
                if (chosen) chosen[gid] = (uint8_t)best_i;
            }
        }
    }
}

}  // namespace w4

using namespace w4;

W4_API w4_status w4_quantize(const void *W_bf16, int64_t N, int64_t K, int group, int mode,
                             const float *clip_grid_host, int n_clip, uint8_t *codes,
                             uint16_t *scales_fp16, int16_t *zeros, uint8_t *chosen_idx,
                             cudaStream_t stream) {
    if (!W_bf16 || !clip_grid_host || !codes || !scales_fp16) return W4_ERR_NULL;
    if (!valid_mode(mode)) return W4_ERR_ARG;
    if (mode == W4_ASYM && !zeros) return W4_ERR_NULL;
    if (mode == W4_SYM && zeros) return W4_ERR_ARG;
    if (N < 1 || K < 32 || K % 32 != 0) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (n_clip < 1 || n_clip > 64) return W4_ERR_ARG;
    if (!aligned16(W_bf16) || !aligned16(codes) || !aligned16(scales_fp16) || (zeros && !aligned16(zeros)) ||
        (chosen_idx && !aligned16(chosen_idx)))
        return W4_ERR_ALIGN;
    ClipGrid grid;
    grid.n = n_clip;
    for (int i = 0; i < 64; ++i) grid.r[i] = 0.0f;
    for (int i = 0; i < n_clip; ++i) {
        const float r = clip_grid_host[i];
        if (!(r > 0.0f && r <= 1.0f)) return W4_ERR_ARG;  // also rejects NaN
        grid.r[i] = r;
    }
    if (grid.r[0] != 1.0f) return W4_ERR_ARG;

    const int64_t total = N * (K / group);
    const int64_t want = (total + 31) / 32;  // 8 warps of 4 groups per block
    const int blocks = (int)(want < (int64_t)num_sms() * 64 ? want : (int64_t)num_sms() * 64);
#define W4_Q(G_, A_)                                                                              \
    quantize_kernel<G_, A_><<<blocks, 256, 0, stream>>>(static_cast<const uint16_t *>(W_bf16), K, total, grid, \
                                                        codes, scales_fp16, zeros, chosen_idx)
    const bool asym = mode == W4_ASYM;
    if (group == 32) { if (asym) W4_Q(32, true); else W4_Q(32, false); }
    else if (group == 64) { if (asym) W4_Q(64, true); else W4_Q(64, false); }
    else if (group == 128) { if (asym) W4_Q(128, true); else W4_Q(128, false); }
    else { if (asym) W4_Q(256, true); else W4_Q(256, false); }
#undef W4_Q
    return launch_status();
}
