// fp8_row_quant: dynamic per-row FP8 E4M3 activation quantization.
//
// "Four-bit inference ... Tahoma", Achievement 2: 8-bit activations without a calibration
// set -- every row (token) gets its own scale from its max |x| over the E4M3 maximum 448,
// with a 1e-8 floor, recomputed on every call; an all-zero row stays zero.
//
// One 256-thread CTA per row. The row is held in registers (16-byte chunks, chunk c of the
// row goes to thread c mod 256), reduced to max|x| by warp shuffles and shared memory,
// then every element is divided by the scale (IEEE fp32) and converted with
// cvt.rn.satfinite.e4m3x2.f32. Optional per-group sums of the E4M3 values are formed as
// exact integer sums in units of 2^-9 (every E4M3 value is an integer multiple of 2^-9)
// and rounded once to fp32; from them the optional group-sum operand of the W4A8 GEMM is
// written: per row [hi(G) | lo(G) | hi(G) | 0 ...] in bf16, hi = bf16(G), lo = bf16(G - hi),
// padded to a multiple of 32 columns. HBM-bound: 2 bytes read and 1 written per element.
// Compiled with -fmad=false.
#include "w4_common.cuh"
#include "w4_layout.cuh"

namespace w4 {

// e4m3 byte -> its value times 2^9, as an integer (exact; |v| <= 448 * 512).
__device__ __forceinline__ int e4m3_times512(uint32_t b) {
    const int E = (b >> 3) & 15, M = b & 7;
    const int mag = (E == 0) ? M : ((8 + M) << (E - 1));
    return (b & 0x80) ? -mag : mag;
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// one group sum -> its three entries in the group-sum operand row (hi, lo, hi at j, Jr + j, 2 Jr + j)
__device__ __forceinline__ void write_gop(uint16_t *row, int64_t Jr, int64_t j, float G) {
    const uint16_t hi = bf16_rn_bits(G);
    row[j] = hi;
    row[Jr + j] = bf16_rn_bits(__fsub_rn(G, __uint_as_float((uint32_t)hi << 16)));
    row[2 * Jr + j] = hi;
}

// two floats -> two e4m3 bytes (lo = a, hi = b), RNE, saturating
__device__ __forceinline__ uint32_t cvt_e4m3x2(float a, float b) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}

template <int NC>  // 16-byte chunks per thread held in registers
__global__ void __launch_bounds__(256) row_quant_kernel(const uint16_t *__restrict__ X, int64_t K, int group,
                                                        uint8_t *__restrict__ X8, float *__restrict__ row_scale,
                                                        float *__restrict__ gsum, uint16_t *__restrict__ gop,
                                                        int64_t KZ) {
    __shared__ float red[8];
    const int64_t m = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t nchunk = K / 8;
    const uint4 *src = reinterpret_cast<const uint4 *>(X + m * K);
    uint4 v[NC];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int64_t c = tid + 256 * i;
        if (c < nchunk) {
            v[i] = src[c];
            const uint32_t *u = reinterpret_cast<const uint32_t *>(&v[i]);
#pragma unroll
            for (int t = 0; t < 4; ++t) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[t])), fabsf(bf16_hi(u[t]))));
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, off));
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float s = __fdiv_rn(fmaxf(amax, 1e-8f), 448.0f);
    if (tid == 0) row_scale[m] = s;

    uint2 *dst = reinterpret_cast<uint2 *>(X8 + m * K);
    const int lanes_per_group = group / 8;  // 4, 8 or 16 threads share a group
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int64_t c = tid + 256 * i;
        const bool live = c < nchunk;
        uint32_t o0 = 0, o1 = 0;
        int isum = 0;
        if (live) {
            const uint32_t *u = reinterpret_cast<const uint32_t *>(&v[i]);
            const uint32_t p0 = cvt_e4m3x2(__fdiv_rn(bf16_lo(u[0]), s), __fdiv_rn(bf16_hi(u[0]), s));
            const uint32_t p1 = cvt_e4m3x2(__fdiv_rn(bf16_lo(u[1]), s), __fdiv_rn(bf16_hi(u[1]), s));
            const uint32_t p2 = cvt_e4m3x2(__fdiv_rn(bf16_lo(u[2]), s), __fdiv_rn(bf16_hi(u[2]), s));
            const uint32_t p3 = cvt_e4m3x2(__fdiv_rn(bf16_lo(u[3]), s), __fdiv_rn(bf16_hi(u[3]), s));
            o0 = p0 | (p1 << 16);
            o1 = p2 | (p3 << 16);
            dst[c] = make_uint2(o0, o1);
            if (gsum || gop) {
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    isum += e4m3_times512((o0 >> (8 * t)) & 0xFF);
                    isum += e4m3_times512((o1 >> (8 * t)) & 0xFF);
                }
            }
        }
        if (gsum || gop) {
            // groups never straddle a 256-chunk stride (256 * 8 is a multiple of the group)
            for (int off = 1; off < lanes_per_group; off <<= 1) isum += __shfl_xor_sync(FULL, isum, off);
            if (live && (tid % lanes_per_group) == 0) {
                const int64_t j = (c * 8) / group;
                const float G = __fmul_rn(__int2float_rn(isum), 0.001953125f);
                if (gsum) gsum[m * (K / group) + j] = G;
                if (gop) write_gop(gop + m * KZ, K / group, j, G);
            }
        }
    }
    if (gop && tid < KZ - 3 * (K / group)) gop[m * KZ + 3 * (K / group) + tid] = 0;
}

// Rows longer than the register budget: three passes over global memory.
__global__ void __launch_bounds__(256) row_quant_long_kernel(const uint16_t *__restrict__ X, int64_t K, int group,
                                                             uint8_t *__restrict__ X8, float *__restrict__ row_scale,
                                                             float *__restrict__ gsum, uint16_t *__restrict__ gop,
                                                             int64_t KZ) {
    __shared__ float red[8];
    const int64_t m = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t nchunk = K / 8;
    const uint4 *src = reinterpret_cast<const uint4 *>(X + m * K);
    float amax = 0.0f;
    for (int64_t c = tid; c < nchunk; c += 256) {
        const uint4 v = src[c];
        const uint32_t *u = reinterpret_cast<const uint32_t *>(&v);
        for (int t = 0; t < 4; ++t) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[t])), fabsf(bf16_hi(u[t]))));
    }
    for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, off));
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float s = __fdiv_rn(fmaxf(amax, 1e-8f), 448.0f);
    if (tid == 0) row_scale[m] = s;
    uint2 *dst = reinterpret_cast<uint2 *>(X8 + m * K);
    const int lanes_per_group = group / 8;
    const int64_t iters = (nchunk + 255) / 256;
    for (int64_t i = 0; i < iters; ++i) {
        const int64_t c = tid + 256 * i;
        const bool live = c < nchunk;
        int isum = 0;
        if (live) {
            const uint4 v = src[c];
            const uint32_t *u = reinterpret_cast<const uint32_t *>(&v);
            uint32_t p[4];
            for (int t = 0; t < 4; ++t) p[t] = cvt_e4m3x2(__fdiv_rn(bf16_lo(u[t]), s), __fdiv_rn(bf16_hi(u[t]), s));
            const uint32_t o0 = p[0] | (p[1] << 16), o1 = p[2] | (p[3] << 16);
            dst[c] = make_uint2(o0, o1);
            if (gsum || gop)
                for (int t = 0; t < 4; ++t)
                    isum += e4m3_times512((o0 >> (8 * t)) & 0xFF) + e4m3_times512((o1 >> (8 * t)) & 0xFF);
        }
        if (gsum || gop) {
            for (int off = 1; off < lanes_per_group; off <<= 1) isum += __shfl_xor_sync(FULL, isum, off);
            if (live && (tid % lanes_per_group) == 0) {
                const int64_t j = (c * 8) / group;
                const float G = __fmul_rn(__int2float_rn(isum), 0.001953125f);
                if (gsum) gsum[m * (K / group) + j] = G;
                if (gop) write_gop(gop + m * KZ, K / group, j, G);
            }
        }
    }
    if (gop && tid < KZ - 3 * (K / group)) gop[m * KZ + 3 * (K / group) + tid] = 0;
}

}  // namespace w4

using namespace w4;

W4_API int64_t w4a8_gsum_op_cols(int64_t K, int group) {
    if (K < 1 || !valid_group(group) || K % group != 0) return 0;
    return zop_cols(K / group);
}

W4_API w4_status fp8_row_quant(const void *X_bf16, int64_t M, int64_t K, int group, uint8_t *X_e4m3,
                               float *row_scale, float *group_sums, uint16_t *gsum_op, cudaStream_t stream) {
    if (!X_bf16 || !X_e4m3 || !row_scale) return W4_ERR_NULL;
    if (M < 1 || M > 0x7fffffff || K < 16 || K % 16 != 0) return W4_ERR_SHAPE;
    const bool sums = group_sums || gsum_op;
    if (sums && (!valid_group(group) || K % group != 0)) return W4_ERR_GROUP;
    if (!aligned16(X_bf16) || !aligned16(X_e4m3) || !aligned16(row_scale) || (group_sums && !aligned16(group_sums)) ||
        (gsum_op && !aligned16(gsum_op)))
        return W4_ERR_ALIGN;
    const int g = sums ? group : 32;
    const int64_t KZ = gsum_op ? zop_cols(K / g) : 0;
    const int64_t nchunk = K / 8;
    const uint16_t *X = static_cast<const uint16_t *>(X_bf16);
    const dim3 grid((unsigned)M);
    if (nchunk <= 256) row_quant_kernel<1><<<grid, 256, 0, stream>>>(X, K, g, X_e4m3, row_scale, group_sums, gsum_op, KZ);
    else if (nchunk <= 512) row_quant_kernel<2><<<grid, 256, 0, stream>>>(X, K, g, X_e4m3, row_scale, group_sums, gsum_op, KZ);
    else if (nchunk <= 1024) row_quant_kernel<4><<<grid, 256, 0, stream>>>(X, K, g, X_e4m3, row_scale, group_sums, gsum_op, KZ);
    else if (nchunk <= 2048) row_quant_kernel<8><<<grid, 256, 0, stream>>>(X, K, g, X_e4m3, row_scale, group_sums, gsum_op, KZ);
    else row_quant_long_kernel<<<grid, 256, 0, stream>>>(X, K, g, X_e4m3, row_scale, group_sums, gsum_op, KZ);
    return launch_status();
}
