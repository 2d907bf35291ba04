// Per-row FP8 E4M3 quantization steps shared by the row-quant kernels and the W4A8 GEMM
// that quantizes its own activation rows ("Four-bit inference ... Tahoma", Achievement 2:
// a per-token scale max|x| / 448 with a 1e-8 floor, recomputed on every forward pass).
// Every step rounds explicitly (_rn intrinsics, inline PTX conversions), so the codes do not
// depend on the including file's -fmad setting. Internal header: not part of the ABI.
#pragma once

#include "w4_common.cuh"

namespace w4 {

// Sum of the 8 E4M3 values in (o0, o1), times 2^9, as an integer. Each pair goes back to
// f16x2 (exact: E4M3 is a subset of binary16) and each half is added into an fp32 sum by a
// mixed-precision FMA with 1.0; the sum is exact in fp32 because every partial sum is a
// multiple of 2^-9 below 8 * 448 < 2^12, which needs at most 21 significant bits. The scaled
// total is an integer below 2^21, converted exactly.
__device__ __forceinline__ int e4m3x8_sum_times512(uint32_t o0, uint32_t o1) {
    float acc0 = 0.0f, acc1 = 0.0f;  // two chains (low and high halves of each pair)
    const uint16_t one = 0x3C00;     // binary16 1.0
    const uint32_t w[2] = {o0, o1};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint16_t pair = (uint16_t)(w[i] >> (16 * h));
            asm("{\n .reg .b32 f;\n .reg .b16 lo, hi;\n cvt.rn.f16x2.e4m3x2 f, %2;\n mov.b32 {lo, hi}, f;\n"
                " fma.rn.f32.f16 %0, lo, %3, %0;\n fma.rn.f32.f16 %1, hi, %3, %1;\n}\n"
                : "+f"(acc0), "+f"(acc1)
                : "h"(pair), "h"(one));
        }
    }
    return __float2int_rn(__fmul_rn(__fadd_rn(acc0, acc1), 512.0f));
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
// x / s rounded to nearest, from r = 1/s rounded to nearest, by Markstein's correction
// step (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Develop. 34(1), 1990): q0 = x*r, e = q0*s - x (exact with one
// FMA; minus the remainder, so that a zero x keeps its sign), q = q0 - e*r. For this
// kernel's operands -- s = max(amax, 1e-8)/448 with amax a finite bf16 magnitude, and
// |x| <= amax -- the result is the IEEE quotient wherever that can decide an E4M3 code: an
// exhaustive check of all such (amax, x) pairs finds no difference for |x/s| > 2^-11, for
// zero quotients, or in sign (smaller quotients may differ in the last bit; both round to a
// zero code). Rows holding an infinity or a NaN take the IEEE division instead.
__device__ __forceinline__ float div_by_scale(float x, float s, float r) {
    const float q0 = __fmul_rn(x, r);
    const float e = __fmaf_rn(q0, s, -x);
    return __fmaf_rn(-e, r, q0);
}

// two floats -> two e4m3 bytes (lo = a, hi = b), RNE, saturating
__device__ __forceinline__ uint32_t cvt_e4m3x2(float a, float b) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}

// 8 bf16 values -> 8 e4m3 bytes (o0: values 0-3, o1: values 4-7)
template <bool EXACT_DIV>
__device__ __forceinline__ uint2 quantize8(const uint4 &v, float s, float r) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    uint32_t p[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float lo = bf16_lo(u[t]), hi = bf16_hi(u[t]);
        p[t] = EXACT_DIV ? cvt_e4m3x2(__fdiv_rn(lo, s), __fdiv_rn(hi, s))
                         : cvt_e4m3x2(div_by_scale(lo, s, r), div_by_scale(hi, s, r));
    }
    return make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
}

// Row maximum of |x| as bf16 bits: a max over the 15 magnitude bits (16-bit SIMD max), which
// orders finite values, infinity (0x7F80) and NaN (above) the same way as their magnitudes.
__device__ __forceinline__ uint32_t absmax_bits(uint32_t acc, const uint4 &v) {
    acc = __vmaxu2(acc, v.x & 0x7FFF7FFFu);
    acc = __vmaxu2(acc, v.y & 0x7FFF7FFFu);
    acc = __vmaxu2(acc, v.z & 0x7FFF7FFFu);
    return __vmaxu2(acc, v.w & 0x7FFF7FFFu);
}

// max |x| ignoring NaNs (fmaxf semantics), for the rare rows that hold a NaN
__device__ __forceinline__ float absmax_float(float acc, const uint4 &v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) acc = fmaxf(acc, fmaxf(fabsf(bf16_lo(u[t])), fabsf(bf16_hi(u[t]))));
    return acc;
}
// row scale: max(amax, 1e-8) / 448, IEEE division
__device__ __forceinline__ float scale_of(float amax) { return __fdiv_rn(fmaxf(amax, 1e-8f), 448.0f); }

}  // namespace w4
