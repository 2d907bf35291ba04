// w4_quantize: group-wise INT4 quantizer with the data-free MSE clip search.
//
// "Quantizing LLMs Without Guesswork", Scale and zero point / Granularity / Quantize, then
// dequantize; "Four-bit inference ... Tahoma", The naive symmetric baseline, Achievement 1,
// MSE clipping.
//
// One warp owns one group of g weights (g = 32, 64, 128): lane l holds the contiguous chunk
// [l*g/32, (l+1)*g/32). The group's min / max / max|w| come from warp shuffles (exact), and
// every clip ratio is evaluated in registers: scale rounded to fp16, zero point, codes,
// reconstruction and squared error, then the block error is reduced in a fixed tree (each
// lane sums its chunk in order, then butterfly at distances 16, 8, 4, 2, 1), so every lane
// holds the same bit pattern and the strict-improvement test is warp-uniform. This
// translation unit is compiled with -fmad=false and spells every operation with an _rn
// intrinsic, so no multiply-add is ever contracted and results are reproducible bit for bit.
#include "w4_common.cuh"

namespace w4 {

struct ClipGrid {
    float r[64];
    int n;
};

__device__ __forceinline__ float f16_round(float x) { return __half2float(__float2half_rn(x)); }

__device__ __forceinline__ float sat_i16f(float v) { return fminf(fmaxf(v, -32768.0f), 32767.0f); }

template <int G, bool ASYM>
__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t *__restrict__ W, int64_t K,
                                                       int64_t total_groups, ClipGrid grid,
                                                       uint8_t *__restrict__ codes,
                                                       uint16_t *__restrict__ scales,
                                                       int16_t *__restrict__ zeros,
                                                       uint8_t *__restrict__ chosen) {
    constexpr int E = G / 32;  // weights per lane
    const int lane = threadIdx.x & 31;
    const int64_t J = K / G;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t gid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); gid < total_groups;
         gid += warps) {
        const int64_t n = gid / J, j = gid - n * J;
        const uint16_t *src = W + n * K + j * G + lane * E;
        float w[E];
        if constexpr (E == 4) {
            uint2 v = *reinterpret_cast<const uint2 *>(src);
            w[0] = bf16_lo(v.x); w[1] = bf16_hi(v.x); w[2] = bf16_lo(v.y); w[3] = bf16_hi(v.y);
        } else if constexpr (E == 2) {
            uint32_t v = *reinterpret_cast<const uint32_t *>(src);
            w[0] = bf16_lo(v); w[1] = bf16_hi(v);
        } else {
            w[0] = __uint_as_float(((uint32_t)src[0]) << 16);
        }
        float lo = w[0], hi = w[0], amax = fabsf(w[0]);
#pragma unroll
        for (int e = 1; e < E; ++e) {
            lo = fminf(lo, w[e]);
            hi = fmaxf(hi, w[e]);
            amax = fmaxf(amax, fabsf(w[e]));
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(FULL, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(FULL, hi, off));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, off));
        }

        float best_sse = 0.0f, best_s = 1.0f, best_z = 8.0f;
        uint32_t best_q = 0;  // E nibbles, nibble e at bits [4e, 4e+4)
        int best_i = 0;
        for (int i = 0; i < grid.n; ++i) {
            const float r = grid.r[i];
            float s, zf;
            if constexpr (!ASYM) {
                const float a_r = __fmul_rn(r, amax);
                s = f16_round(__fdiv_rn(a_r, 7.0f));
                if (s == 0.0f) s = 1.0f;
                zf = 8.0f;
            } else {
                const float h = __fmul_rn(0.5f, __fsub_rn(hi, lo));
                const float cc = __fmul_rn(__fsub_rn(1.0f, r), h);
                const float lo_r = __fadd_rn(lo, cc);
                const float hi_r = __fsub_rn(hi, cc);
                s = f16_round(__fdiv_rn(__fsub_rn(hi_r, lo_r), 15.0f));
                if (s == 0.0f) s = 1.0f;
                zf = sat_i16f(rintf(__fdiv_rn(-lo_r, s)));
            }
            uint32_t qv = 0;
            float part = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                float rec, nib;
                if constexpr (!ASYM) {
                    const float c = fminf(fmaxf(rintf(__fdiv_rn(w[e], s)), -7.0f), 7.0f);
                    rec = __fmul_rn(c, s);
                    nib = __fadd_rn(c, 8.0f);
                } else {
                    const float q = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w[e], s)), zf), 0.0f), 15.0f);
                    rec = __fmul_rn(__fsub_rn(q, zf), s);
                    nib = q;
                }
                const float err = __fsub_rn(w[e], rec);
                const float e2 = __fmul_rn(err, err);
                part = (e == 0) ? e2 : __fadd_rn(part, e2);
                qv |= ((uint32_t)nib) << (4 * e);
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) part = __fadd_rn(part, __shfl_xor_sync(FULL, part, off));
            if (i == 0 || part < best_sse) {
                best_sse = part;
                best_s = s;
                best_z = zf;
                best_q = qv;
                best_i = i;
            }
        }

        uint8_t *dst = codes + n * (K / 2) + (j * G) / 2;
        if constexpr (E == 4) {
            const uint16_t b = (uint16_t)((best_q & 0xFu) | (((best_q >> 4) & 0xFu) << 4) |
                                          (((best_q >> 8) & 0xFu) << 8) | (((best_q >> 12) & 0xFu) << 12));
            reinterpret_cast<uint16_t *>(dst)[lane] = b;
        } else if constexpr (E == 2) {
            dst[lane] = (uint8_t)((best_q & 0xFu) | (((best_q >> 4) & 0xFu) << 4));
        } else {
            const uint32_t other = __shfl_down_sync(FULL, best_q, 1);
            if ((lane & 1) == 0) dst[lane >> 1] = (uint8_t)((best_q & 0xFu) | ((other & 0xFu) << 4));
        }
        if (lane == 0) {
            scales[gid] = __half_as_ushort(__float2half_rn(best_s));
            if (ASYM) zeros[gid] = (int16_t)best_z;
            if (chosen) chosen[gid] = (uint8_t)best_i;
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
    const int64_t want = (total + 7) / 8;
    const int blocks = (int)(want < (int64_t)num_sms() * 64 ? want : (int64_t)num_sms() * 64);
#define W4_Q(G_, A_)                                                                              \
    quantize_kernel<G_, A_><<<blocks, 256, 0, stream>>>(static_cast<const uint16_t *>(W_bf16), K, total, grid, \
                                                        codes, scales_fp16, zeros, chosen_idx)
    const bool asym = mode == W4_ASYM;
    if (group == 32) { if (asym) W4_Q(32, true); else W4_Q(32, false); }
    else if (group == 64) { if (asym) W4_Q(64, true); else W4_Q(64, false); }
    else { if (asym) W4_Q(128, true); else W4_Q(128, false); }
#undef W4_Q
    return launch_status();
}
