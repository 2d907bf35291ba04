// fp8_row_quant: dynamic per-row FP8 E4M3 activation quantization.
//
// "Four-bit inference ... Tahoma", Achievement 2: 8-bit activations without a calibration
// set -- every row (token) gets its own scale from its max |x| over the E4M3 maximum 448,
// with a 1e-8 floor, recomputed on every call; an all-zero row stays zero.
//
// One 256-thread CTA per row. The row is held in registers (16-byte chunks, chunk c of the
// row goes to thread c mod 256) and reduced to max|x| (a 16-bit SIMD max over the magnitude
// bits, then a warp reduction and shared memory); every element is then divided by the
// scale (the IEEE fp32 quotient, formed from the row's reciprocal by one exact correction
// step, see div_by_scale) and converted with cvt.rn.satfinite.e4m3x2.f32. Optional per-group
// sums of the E4M3 values are exact integer sums in units of 2^-9 (every E4M3 value is an
// integer multiple of 2^-9: a 16-byte chunk's values are added exactly in fp32, the chunks'
// sums as integers), rounded once to fp32; from them the optional group-sum operand of the
// W4A8 GEMM is written: per row [hi(G) | lo(G) | hi(G) | 0 ...] in bf16, hi = bf16(G),
// lo = bf16(G - hi), padded to a multiple of 32 columns. Optionally the E4M3 values are also
// (or only) written as binary16 -- the exact same values, in the operand type of the W4A8
// GEMM's split-weight path (groups of 32 and 256). HBM-bound: 2 bytes read and 1 written
// per element (+2 for the binary16 copy). Compiled with -fmad=false.
#include "w4_common.cuh"
#include "w4_layout.cuh"
#include "w4_rowquant.cuh"

namespace w4 {


// The 8 E4M3 values of (o.x: values 0-3, o.y: values 4-7) as binary16 (exact: E4M3 is a
// subset of binary16), in order.
__device__ __forceinline__ uint4 e4m3x8_to_f16x8(uint2 o) {
    const uint32_t w[2] = {o.x, o.y};
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint16_t pair = (uint16_t)(w[i >> 1] >> (16 * (i & 1)));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r[i]) : "h"(pair));
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// Store chunk c (8 values) of a row's outputs: the E4M3 codes and/or their binary16 values.
__device__ __forceinline__ void store_chunk(uint8_t *X8, uint16_t *x16, int64_t m, int64_t K, int64_t c, uint2 o) {
    if (X8) reinterpret_cast<uint2 *>(X8 + m * K)[c] = o;
    if (x16) reinterpret_cast<uint4 *>(x16 + m * K)[c] = e4m3x8_to_f16x8(o);
}

// Group outputs of groups [j0, j0 + nj) of row m, whose sums are in sh[0 .. nj), written by
// the whole block with consecutive threads on consecutive entries: the fp32 sums, and the
// group-sum operand entries hi(G) at column j, lo(G) at J + j and hi(G) at 2J + j
// (J = K / group; hi = bf16(G), lo = bf16(G - hi)).
// t0 / stride: this thread's first entry and the number of threads sharing the work.
__device__ __forceinline__ void write_group_outputs(const float *sh, int64_t j0, int nj, int64_t J, int64_t m,
                                                    float *gsum, uint16_t *gop, int64_t KZ, int t0, int stride) {
    if (gsum)
        for (int t = t0; t < nj; t += stride) gsum[m * J + j0 + t] = sh[t];
    if (gop) {
        uint16_t *row = gop + m * KZ;
        for (int t = t0; t < 3 * nj; t += stride) {
            const int region = t / nj, jj = t - region * nj;
            const float G = sh[jj];
            const uint16_t hi = bf16_rn_bits(G);
            row[region * J + j0 + jj] = region == 1 ? bf16_rn_bits(__fsub_rn(G, __uint_as_float((uint32_t)hi << 16))) : hi;
        }
    }
}


// Block-wide max of a per-thread value (256 threads); every thread gets the result.
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t *red) {
    v = __reduce_max_sync(FULL, v);
    __syncthreads();  // red may still be read from an earlier reduction
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    v = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) v = v > red[w] ? v : red[w];
    return v;
}

__device__ __forceinline__ float block_max_f32(float v, uint32_t *red) {
    // non-negative floats order like their bit patterns
    return __uint_as_float(block_max_u32(__float_as_uint(v), red));
}

// The group sum of the group holding 16-byte chunk c of E4M3 codes (8 values at columns
// 8c..8c+7), reduced over the lanes that share the group and stored by the first of them at
// sh[j - j0] (j the group's index).
__device__ __forceinline__ void group_sum(uint2 o, bool live, int64_t c, int group, int64_t j0, float *sh) {
    const int lanes_per_group = group / 8;  // 4, 8 or 16 threads share a group
    int isum = live ? e4m3x8_sum_times512(o.x, o.y) : 0;
    // groups never straddle a 256-chunk stride (256 * 8 is a multiple of the group)
    for (int off = 1; off < lanes_per_group; off <<= 1) isum += __shfl_xor_sync(FULL, isum, off);
    if (live && (threadIdx.x % lanes_per_group) == 0)
        sh[(c * 8) / group - j0] = __fmul_rn(__int2float_rn(isum), 0.001953125f);
}

// The source row of output row m (rows == nullptr: m itself); an index outside [0, msrc)
// is recorded as W4_ERR_DEVICE_CHECK and gives -1 (the row is then quantized as zeros).
__device__ __forceinline__ int64_t source_row(const int32_t *rows, int64_t m, int64_t msrc, int *status) {
    if (!rows) return m;
    const int64_t r = rows[m];
    if (r < 0 || r >= msrc) {
        if ((threadIdx.x & 31) == 0) record_status(status, W4_ERR_DEVICE_CHECK);
        return -1;
    }
    return r;
}


template <int NC>  // 16-byte chunks per thread held in registers
__global__ void __launch_bounds__(256) row_quant_kernel(const uint16_t *__restrict__ X, int64_t K, int group,
                                                        uint8_t *__restrict__ X8, uint16_t *__restrict__ x16,
                                                        float *__restrict__ row_scale,
                                                        float *__restrict__ gsum, uint16_t *__restrict__ gop,
                                                        int64_t KZ, const int32_t *__restrict__ rows, int64_t msrc,
                                                        int *status) {
    __shared__ uint32_t red[8];
    __shared__ float gsh[NC * 256 * 8 / 32];  // the row's group sums (K <= NC * 2048)
    const int64_t m = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t nchunk = K / 8;
    const int64_t srow = source_row(rows, m, msrc, status);
    const uint4 *src = reinterpret_cast<const uint4 *>(X + (srow < 0 ? 0 : srow) * K);
    uint4 v[NC];
    uint32_t mb = 0;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int64_t c = tid + 256 * i;
        v[i] = (c < nchunk && srow >= 0) ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        mb = absmax_bits(mb, v[i]);
    }
    mb = block_max_u32(__vmaxu2(mb, mb >> 16) & 0xFFFFu, red);
    const bool special = mb >= 0x7F80u;  // an infinity or a NaN in the row
    float amax = __uint_as_float(mb << 16);
    if (mb > 0x7F80u) {  // NaN: the maximum of the other values
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < NC; ++i) a = absmax_float(a, v[i]);
        amax = block_max_f32(a, red);
    }
    const float s = scale_of(amax);
    const float r = __frcp_rn(s);
    if (tid == 0) row_scale[m] = s;

    const bool sums = gsum || gop;
    int isum[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int64_t c = tid + 256 * i;
        isum[i] = 0;
        if (c < nchunk) {
            const uint2 o = special ? quantize8<true>(v[i], s, r) : quantize8<false>(v[i], s, r);
            store_chunk(X8, x16, m, K, c, o);
            if (sums) isum[i] = e4m3x8_sum_times512(o.x, o.y);
        }
    }
    if (sums) {
        // every chunk's group sum over the lanes that share its group, all chunks at once
        // (groups never straddle a 256-chunk stride: 256 * 8 is a multiple of the group)
        const int lanes_per_group = group / 8;
        for (int off = 1; off < lanes_per_group; off <<= 1) {
#pragma unroll
            for (int i = 0; i < NC; ++i) isum[i] += __shfl_xor_sync(FULL, isum[i], off);
        }
        if (tid % lanes_per_group == 0) {
#pragma unroll
            for (int i = 0; i < NC; ++i) {
                const int64_t c = tid + 256 * i;
                if (c < nchunk) gsh[(c * 8) / group] = __fmul_rn(__int2float_rn(isum[i]), 0.001953125f);
            }
        }
        __syncthreads();
        write_group_outputs(gsh, 0, (int)(K / group), K / group, m, gsum, gop, KZ, tid, 256);
        if (gop)
            for (int64_t t = 3 * (K / group) + tid; t < KZ; t += 256) gop[m * KZ + t] = 0;
    }
}

// Rows of at most 32 * NCW chunks (K <= 4096): one warp per row, 8 rows per block, the row in
// registers (chunk c of the row goes to lane c mod 32); every reduction is a warp operation.
template <int NCW>
__global__ void __launch_bounds__(256) row_quant_warp_kernel(const uint16_t *__restrict__ X, int64_t M, int64_t K,
                                                             int group, uint8_t *__restrict__ X8, uint16_t *__restrict__ x16,
                                                             float *__restrict__ row_scale, float *__restrict__ gsum,
                                                             uint16_t *__restrict__ gop, int64_t KZ,
                                                             const int32_t *__restrict__ rows, int64_t msrc,
                                                             int *status) {
    __shared__ float gsh_all[8][NCW * 8];  // per warp: its row's group sums (K / 32 at most)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m = (int64_t)blockIdx.x * 8 + warp;
    if (m >= M) return;  // no block-wide barrier below
    float *gsh = gsh_all[warp];
    const int64_t nchunk = K / 8;
    const int64_t srow = source_row(rows, m, msrc, status);
    const uint4 *src = reinterpret_cast<const uint4 *>(X + (srow < 0 ? 0 : srow) * K);
    uint4 v[NCW];
    uint32_t mb = 0;
#pragma unroll
    for (int i = 0; i < NCW; ++i) {
        const int64_t c = lane + 32 * i;
        v[i] = (c < nchunk && srow >= 0) ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        mb = absmax_bits(mb, v[i]);
    }
    mb = __reduce_max_sync(FULL, __vmaxu2(mb, mb >> 16) & 0xFFFFu);
    const bool special = mb >= 0x7F80u;  // an infinity or a NaN in the row
    float amax = __uint_as_float(mb << 16);
    if (mb > 0x7F80u) {  // NaN: the maximum of the other values (non-negative floats order as bits)
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < NCW; ++i) a = absmax_float(a, v[i]);
        amax = __uint_as_float(__reduce_max_sync(FULL, __float_as_uint(a)));
    }
    const float s = scale_of(amax);
    const float r = __frcp_rn(s);
    if (lane == 0) row_scale[m] = s;

    const bool sums = gsum || gop;
    int isum[NCW];
#pragma unroll
    for (int i = 0; i < NCW; ++i) {
        const int64_t c = lane + 32 * i;
        isum[i] = 0;
        if (c < nchunk) {
            const uint2 o = special ? quantize8<true>(v[i], s, r) : quantize8<false>(v[i], s, r);
            store_chunk(X8, x16, m, K, c, o);
            if (sums) isum[i] = e4m3x8_sum_times512(o.x, o.y);
        }
    }
    if (sums) {
        // groups never straddle a 32-chunk stride (32 * 8 is a multiple of the group)
        const int lanes_per_group = group / 8;
        for (int off = 1; off < lanes_per_group; off <<= 1) {
#pragma unroll
            for (int i = 0; i < NCW; ++i) isum[i] += __shfl_xor_sync(FULL, isum[i], off);
        }
        if (lane % lanes_per_group == 0) {
#pragma unroll
            for (int i = 0; i < NCW; ++i) {
                const int64_t c = lane + 32 * i;
                if (c < nchunk) gsh[(c * 8) / group] = __fmul_rn(__int2float_rn(isum[i]), 0.001953125f);
            }
        }
        __syncwarp();
        write_group_outputs(gsh, 0, (int)(K / group), K / group, m, gsum, gop, KZ, lane, 32);
        if (gop)
            for (int64_t t = 3 * (K / group) + lane; t < KZ; t += 32) gop[m * KZ + t] = 0;
    }
}

// Rows longer than the register budget: two passes over global memory.
__global__ void __launch_bounds__(256) row_quant_long_kernel(const uint16_t *__restrict__ X, int64_t K, int group,
                                                             uint8_t *__restrict__ X8, uint16_t *__restrict__ x16,
                                                             float *__restrict__ row_scale,
                                                             float *__restrict__ gsum, uint16_t *__restrict__ gop,
                                                             int64_t KZ, const int32_t *__restrict__ rows, int64_t msrc,
                                                        int *status) {
    __shared__ uint32_t red[8];
    __shared__ float gsh[256 * 8 / 32];  // group sums of one round of 256 chunks
    const int64_t m = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t nchunk = K / 8;
    const int64_t srow = source_row(rows, m, msrc, status);
    const uint4 *src = reinterpret_cast<const uint4 *>(X + (srow < 0 ? 0 : srow) * K);
    uint32_t mb = 0;
    for (int64_t c = tid; c < nchunk && srow >= 0; c += 256) mb = absmax_bits(mb, src[c]);
    mb = block_max_u32(__vmaxu2(mb, mb >> 16) & 0xFFFFu, red);
    const bool special = mb >= 0x7F80u;
    float amax = __uint_as_float(mb << 16);
    if (mb > 0x7F80u) {
        float a = 0.0f;
        for (int64_t c = tid; c < nchunk && srow >= 0; c += 256) a = absmax_float(a, src[c]);
        amax = block_max_f32(a, red);
    }
    const float s = scale_of(amax);
    const float r = __frcp_rn(s);
    if (tid == 0) row_scale[m] = s;
    const int64_t iters = (nchunk + 255) / 256;
    for (int64_t i = 0; i < iters; ++i) {
        const int64_t c = tid + 256 * i;
        const bool live = c < nchunk;
        uint2 o = make_uint2(0u, 0u);
        if (live) {
            const uint4 v = srow >= 0 ? src[c] : make_uint4(0u, 0u, 0u, 0u);
            o = special ? quantize8<true>(v, s, r) : quantize8<false>(v, s, r);
            store_chunk(X8, x16, m, K, c, o);
        }
        if (gsum || gop) {
            // this round's groups: [j0, j0 + nj)
            const int64_t j0 = i * 2048 / group;
            const int64_t jend = ((i + 1) * 2048 < K ? (i + 1) * 2048 : K) / group;
            group_sum(o, live, c, group, j0, gsh);
            __syncthreads();
            write_group_outputs(gsh, j0, (int)(jend - j0), K / group, m, gsum, gop, KZ, tid, 256);
            __syncthreads();  // gsh is reused by the next round
        }
    }
    if (gop)
        for (int64_t t = 3 * (K / group) + tid; t < KZ; t += 256) gop[m * KZ + t] = 0;
}

// SwiGLU between the expert projections, then the row quant of its result: row r of the
// gate_up output holds [gate (H) | up (H)] in bf16; h = gate * up / (1 + exp(-gate)) in fp32
// (expf, then a product, a sum and an IEEE division), amax over the row, s = max(amax, 1e-8)
// / 448 and codes e4m3(h / s) with the IEEE division (h is an fp32 value, so the bf16-domain
// reciprocal shortcut of the other kernels does not apply). One 256-thread block per row,
// the row's h held in registers (NC chunks of 8 per thread, H <= NC * 2048).
template <int NC>
__global__ void __launch_bounds__(256) swiglu_quant_kernel(const uint16_t *__restrict__ Y, int64_t H, int group,
                                                           uint8_t *__restrict__ X8, uint16_t *__restrict__ x16,
                                                           float *__restrict__ row_scale,
                                                           uint16_t *__restrict__ gop, int64_t KZ) {
    __shared__ uint32_t red[8];
    __shared__ float gsh[NC * 256 * 8 / 32];
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t nchunk = H / 8;
    const uint4 *gsrc = reinterpret_cast<const uint4 *>(Y + r * 2 * H);
    const uint4 *usrc = reinterpret_cast<const uint4 *>(Y + r * 2 * H + H);
    float h[NC][8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int64_t c = tid + 256 * i;
        const uint4 gv = c < nchunk ? gsrc[c] : make_uint4(0u, 0u, 0u, 0u);
        const uint4 uv = c < nchunk ? usrc[c] : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t g4[4] = {gv.x, gv.y, gv.z, gv.w}, u4[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float gj = (j & 1) ? bf16_hi(g4[j >> 1]) : bf16_lo(g4[j >> 1]);
            const float uj = (j & 1) ? bf16_hi(u4[j >> 1]) : bf16_lo(u4[j >> 1]);
            h[i][j] = __fdiv_rn(__fmul_rn(gj, uj), __fadd_rn(1.0f, expf(-gj)));
            amax = fmaxf(amax, fabsf(h[i][j]));
        }
    }
    amax = block_max_f32(amax, red);
    const float s = scale_of(amax);
    if (tid == 0) row_scale[r] = s;
    int isum[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int64_t c = tid + 256 * i;
        isum[i] = 0;
        if (c < nchunk) {
            uint32_t p[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) p[t] = cvt_e4m3x2(__fdiv_rn(h[i][2 * t], s), __fdiv_rn(h[i][2 * t + 1], s));
            const uint2 o = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
            store_chunk(X8, x16, r, H, c, o);
            if (gop) isum[i] = e4m3x8_sum_times512(o.x, o.y);
        }
    }
    if (gop) {
        const int lanes_per_group = group / 8;
        for (int off = 1; off < lanes_per_group; off <<= 1) {
#pragma unroll
            for (int i = 0; i < NC; ++i) isum[i] += __shfl_xor_sync(FULL, isum[i], off);
        }
        if (tid % lanes_per_group == 0) {
#pragma unroll
            for (int i = 0; i < NC; ++i) {
                const int64_t c = tid + 256 * i;
                if (c < nchunk) gsh[(c * 8) / group] = __fmul_rn(__int2float_rn(isum[i]), 0.001953125f);
            }
        }
        __syncthreads();
        write_group_outputs(gsh, 0, (int)(H / group), H / group, r, nullptr, gop, KZ, tid, 256);
        for (int64_t t = 3 * (H / group) + tid; t < KZ; t += 256) gop[r * KZ + t] = 0;
    }
}

}  // namespace w4

using namespace w4;

W4_API int64_t w4a8_gsum_op_cols(int64_t K, int group) {
    if (K < 1 || !valid_group(group) || K % group != 0) return 0;
    return zop_cols(K / group);
}

// Output row m is the quantization of source row rows[m] (rows == nullptr: row m).
static w4_status row_quant_launch(const void *X_bf16, const int32_t *rows, int64_t msrc, int64_t M, int64_t K,
                                  int group, uint8_t *X_e4m3, uint16_t *X_f16, float *row_scale, float *group_sums,
                                  uint16_t *gsum_op, cudaStream_t stream) {
    int *st = device_status_ptr();
    const bool sums = group_sums || gsum_op;
    const int g = sums ? group : 32;
    const int64_t KZ = gsum_op ? zop_cols(K / g) : 0;
    const int64_t nchunk = K / 8;
    const uint16_t *X = static_cast<const uint16_t *>(X_bf16);
    const dim3 grid((unsigned)M), wgrid((unsigned)((M + 7) / 8));
    if (nchunk <= 64) row_quant_warp_kernel<2><<<wgrid, 256, 0, stream>>>(X, M, K, g, X_e4m3, X_f16, row_scale, group_sums, gsum_op, KZ, rows, msrc, st);
    else if (nchunk <= 128) row_quant_warp_kernel<4><<<wgrid, 256, 0, stream>>>(X, M, K, g, X_e4m3, X_f16, row_scale, group_sums, gsum_op, KZ, rows, msrc, st);
    else if (nchunk <= 256) row_quant_warp_kernel<8><<<wgrid, 256, 0, stream>>>(X, M, K, g, X_e4m3, X_f16, row_scale, group_sums, gsum_op, KZ, rows, msrc, st);
    else if (nchunk <= 384) row_quant_warp_kernel<12><<<wgrid, 256, 0, stream>>>(X, M, K, g, X_e4m3, X_f16, row_scale, group_sums, gsum_op, KZ, rows, msrc, st);
    else if (nchunk <= 512) row_quant_warp_kernel<16><<<wgrid, 256, 0, stream>>>(X, M, K, g, X_e4m3, X_f16, row_scale, group_sums, gsum_op, KZ, rows, msrc, st);
    else if (nchunk <= 1024) row_quant_kernel<4><<<grid, 256, 0, stream>>>(X, K, g, X_e4m3, X_f16, row_scale, group_sums, gsum_op, KZ, rows, msrc, st);
    else if (nchunk <= 2048) row_quant_kernel<8><<<grid, 256, 0, stream>>>(X, K, g, X_e4m3, X_f16, row_scale, group_sums, gsum_op, KZ, rows, msrc, st);
    else row_quant_long_kernel<<<grid, 256, 0, stream>>>(X, K, g, X_e4m3, X_f16, row_scale, group_sums, gsum_op, KZ, rows, msrc, st);
    return launch_status();
}

W4_API w4_status fp8_row_quant(const void *X_bf16, int64_t M, int64_t K, int group, uint8_t *X_e4m3,
                               float *row_scale, float *group_sums, uint16_t *gsum_op, uint16_t *X_f16,
                               cudaStream_t stream) {
    if (!X_bf16 || !(X_e4m3 || X_f16) || !row_scale) return W4_ERR_NULL;
    if (M < 1 || M > 0x7fffffff || K < 16 || K % 16 != 0) return W4_ERR_SHAPE;
    const bool sums = group_sums || gsum_op;
    if (sums && (!valid_group(group) || K % group != 0)) return W4_ERR_GROUP;
    if (!aligned16(X_bf16) || !aligned16(X_e4m3) || !aligned16(X_f16) || !aligned16(row_scale) ||
        (group_sums && !aligned16(group_sums)) || (gsum_op && !aligned16(gsum_op)))
        return W4_ERR_ALIGN;
    return row_quant_launch(X_bf16, nullptr, M, M, K, group, X_e4m3, X_f16, row_scale, group_sums, gsum_op, stream);
}

W4_API w4_status fp8_row_quant_gather(const void *X_bf16, int64_t M_src, int64_t K, int group,
                                      const int32_t *row_index, int64_t M, uint8_t *X_e4m3, float *row_scale,
                                      float *group_sums, uint16_t *gsum_op, uint16_t *X_f16, cudaStream_t stream) {
    if (!X_bf16 || !row_index || !(X_e4m3 || X_f16) || !row_scale) return W4_ERR_NULL;
    if (M < 1 || M > 0x7fffffff || M_src < 1 || M_src > 0x7fffffff || K < 16 || K % 16 != 0) return W4_ERR_SHAPE;
    const bool sums = group_sums || gsum_op;
    if (sums && (!valid_group(group) || K % group != 0)) return W4_ERR_GROUP;
    if (!aligned16(X_bf16) || !aligned16(X_e4m3) || !aligned16(X_f16) || !aligned16(row_scale) ||
        (group_sums && !aligned16(group_sums)) || (gsum_op && !aligned16(gsum_op)) ||
        (reinterpret_cast<uintptr_t>(row_index) & 3))
        return W4_ERR_ALIGN;
    return row_quant_launch(X_bf16, row_index, M_src, M, K, group, X_e4m3, X_f16, row_scale, group_sums, gsum_op,
                            stream);
}

W4_API w4_status w4_moe_swiglu_quant(const void *gate_up_bf16, int64_t R, int64_t H, int group, uint8_t *X_e4m3,
                                     float *row_scale, uint16_t *gsum_op, uint16_t *X_f16, cudaStream_t stream) {
    if (!gate_up_bf16 || !(X_e4m3 || X_f16) || !row_scale) return W4_ERR_NULL;
    if (R < 1 || R > 0x7fffffff || H < 16 || H % 16 != 0 || H > 8 * 2048) return W4_ERR_SHAPE;
    if (gsum_op && (!valid_group(group) || H % group != 0)) return W4_ERR_GROUP;
    if (!aligned16(gate_up_bf16) || !aligned16(X_e4m3) || !aligned16(X_f16) || !aligned16(row_scale) ||
        (gsum_op && !aligned16(gsum_op)))
        return W4_ERR_ALIGN;
    const int g = gsum_op ? group : 32;
    const int64_t KZ = gsum_op ? zop_cols(H / g) : 0;
    const int64_t nchunk = H / 8;
    const uint16_t *Y = static_cast<const uint16_t *>(gate_up_bf16);
    if (nchunk <= 512) swiglu_quant_kernel<2><<<(unsigned)R, 256, 0, stream>>>(Y, H, g, X_e4m3, X_f16, row_scale, gsum_op, KZ);
    else if (nchunk <= 1024) swiglu_quant_kernel<4><<<(unsigned)R, 256, 0, stream>>>(Y, H, g, X_e4m3, X_f16, row_scale, gsum_op, KZ);
    else swiglu_quant_kernel<8><<<(unsigned)R, 256, 0, stream>>>(Y, H, g, X_e4m3, X_f16, row_scale, gsum_op, KZ);
    return launch_status();
}
