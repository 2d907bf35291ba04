// w4a16_gemv: weight-only INT4 GEMV for decode, dequantization fused into the product.
//
// "Quantizing LLMs Without Guesswork", The Problem & Context (decode reads every weight
// once and that read sets the pace) and Weight-only methods (4-bit weights, 16-bit
// activations, dequantized inside the matmul).
//
//   y[m, n] = sum_j s[n,j] * sum_{k in j} x[m,k] * (q[n,k] - z[n,j])
//
// HBM-bound streaming kernel on the CUDA cores (W4_LAYOUT_GEMV, see w4_layout.cuh):
//  * one CTA (8 warps) per octet of 8 weight rows; the warps take the octet's 128-wide
//    units round-robin, every lane streams one 16-byte word of codes per unit
//    (ld.global.nc.L1::no_allocate, a warp reads 512 contiguous bytes);
//  * the octet's scales/zeros and the activation rows are staged into shared memory by
//    one bulk copy (cp.async.bulk, completion on an mbarrier with a bounded wait);
//  * nibbles become bf16 pairs with one AND/OR: (w & 0x000F000F) | 0x43004300 is the pair
//    (128 + q_a, 128 + q_b), exact in bf16;
//  * fma.rn.f32.bf16 multiplies the bf16 activation by the bf16 (128 + q) exactly and
//    accumulates in fp32; per 32-wide chunk the offset is removed with the chunk's
//    activation sum: sum x*(q - z) = sum x*(128 + q) - (128 + z) * sum x;
//  * the chunk partial is scaled by the group's fp16 scale in fp32 and summed over the
//    row; the four chunk lanes of a row reduce by shuffles, the 8 warps through shared
//    memory in a fixed order (deterministic).
#include "w4_common.cuh"
#include "w4_layout.cuh"

namespace w4 {

__device__ __forceinline__ void fma2_bf16(float &a0, float &a1, uint32_t x, uint32_t q) {
    asm("{\n .reg .b16 xl, xh, ql, qh;\n mov.b32 {xl, xh}, %2;\n mov.b32 {ql, qh}, %3;\n"
        " fma.rn.f32.bf16 %0, xl, ql, %0;\n fma.rn.f32.bf16 %1, xh, qh, %1;\n}\n"
        : "+f"(a0), "+f"(a1)
        : "r"(x), "r"(q));
}

__device__ __forceinline__ uint32_t magic_pair(uint32_t w) { return (w & 0x000F000Fu) | 0x43004300u; }

struct GemvArgs {
    const uint16_t *x;
    const uint8_t *packed;
    void *y;
    int *status;
    int64_t N, K, Kpad, U;
    size_t codes_bytes;
    int M, g, out_fp32, stage_x;
    uint32_t slab_bytes;  // scales of one octet
};

template <int MT>
__global__ void __launch_bounds__(256) gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
    uint32_t *sz = reinterpret_cast<uint32_t *>(smem + 16);                    // scales slab
    float *sx = reinterpret_cast<float *>(smem + 16 + a.slab_bytes);           // [MT][Kpad/32]
    const int nck = (int)(a.Kpad / 32);
    float *red = sx + MT * nck;                                                // [8][8][MT]
    uint16_t *xs = reinterpret_cast<uint16_t *>(red + 64 * MT);                // [M][K] if staged

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = lane >> 2, c = lane & 3;
    const int64_t o = blockIdx.x;
    const int M = a.M;
    const int64_t K = a.K;

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        const uint32_t xbytes = a.stage_x ? (uint32_t)(M * K * 2) : 0u;
        mbar_arrive_expect_tx(bar, a.slab_bytes + xbytes);
        bulk_g2s(sz, a.packed + a.codes_bytes + (size_t)o * a.slab_bytes, a.slab_bytes, bar);
        if (a.stage_x) bulk_g2s(xs, a.x, xbytes, bar);
    }

    // first codes of this warp, issued before waiting on the staged data
    const uint8_t *octet_codes = a.packed + (size_t)o * (size_t)a.U * 512;
    constexpr int UNR = 4;
    uint4 q[UNR];
#pragma unroll
    for (int i = 0; i < UNR; ++i) {
        const int64_t u = warp + 8 * i;
        if (u < a.U) q[i] = ldg_stream(octet_codes + u * 512 + lane * 16);
    }

    if (!mbar_wait_bounded(bar, 0, a.status)) {
        mbar_wait_bounded(bar, 0, a.status);  // let copies in flight land before leaving
        return;
    }

    // activation sums of every 32-wide chunk (chunks past K are zero)
    for (int idx = tid; idx < MT * nck; idx += 256) {
        const int m = idx / nck, ck = idx - m * nck;
        float s = 0.0f;
        if (m < M && (int64_t)ck * 32 < K) {
            if (a.stage_x) {
                const uint32_t *xv = reinterpret_cast<const uint32_t *>(xs + (int64_t)m * K + ck * 32);
#pragma unroll
                for (int t = 0; t < 16; ++t) s = __fadd_rn(__fadd_rn(s, bf16_lo(xv[t])), bf16_hi(xv[t]));
            } else {
                const uint4 *xv = reinterpret_cast<const uint4 *>(a.x + (int64_t)m * K + ck * 32);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint4 v = __ldg(xv + t);
                    s = __fadd_rn(__fadd_rn(s, bf16_lo(v.x)), bf16_hi(v.x));
                    s = __fadd_rn(__fadd_rn(s, bf16_lo(v.y)), bf16_hi(v.y));
                    s = __fadd_rn(__fadd_rn(s, bf16_lo(v.z)), bf16_hi(v.z));
                    s = __fadd_rn(__fadd_rn(s, bf16_lo(v.w)), bf16_hi(v.w));
                }
            }
        }
        sx[idx] = s;
    }
    __syncthreads();

    float y[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) y[m] = 0.0f;
    const int per_unit = 128 / a.g;

    for (int64_t u0 = warp; u0 < a.U; u0 += 8 * UNR) {
#pragma unroll
        for (int i = 0; i < UNR; ++i) {
            const int64_t u = u0 + 8 * i;
            if (u >= a.U) break;
            const uint4 w4v = q[i];
            // prefetch the unit UNR rounds ahead into the slot just consumed
            const int64_t un = u + 8 * UNR;
            if (un < a.U) q[i] = ldg_stream(octet_codes + un * 512 + lane * 16);
            const int64_t k0 = u * 128 + c * 32;
            if (k0 >= K) continue;
            const uint32_t e = sz[(u * 8 + r) * per_unit + (c * 32) / a.g];
            const float s = __half2float(__ushort_as_half((unsigned short)(e & 0xFFFF)));
            const float cz = (float)(128 + (int)(int16_t)(e >> 16));
            const uint32_t wv[4] = {w4v.x, w4v.y, w4v.z, w4v.w};
            uint32_t p[4][4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                p[t][0] = magic_pair(wv[t]);
                p[t][1] = magic_pair(wv[t] >> 4);
                p[t][2] = magic_pair(wv[t] >> 8);
                p[t][3] = magic_pair(wv[t] >> 12);
            }
            const int ck = (int)(k0 >> 5);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= M) break;
                float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    uint4 xv;
                    if (a.stage_x)
                        xv = *reinterpret_cast<const uint4 *>(xs + (int64_t)m * K + k0 + 8 * t);
                    else
                        xv = __ldg(reinterpret_cast<const uint4 *>(a.x + (int64_t)m * K + k0 + 8 * t));
                    fma2_bf16(a0, a1, xv.x, p[t][0]);
                    fma2_bf16(a0, a1, xv.y, p[t][1]);
                    fma2_bf16(a0, a1, xv.z, p[t][2]);
                    fma2_bf16(a0, a1, xv.w, p[t][3]);
                }
                const float part = fmaf(-cz, sx[m * nck + ck], a0 + a1);
                y[m] = fmaf(s, part, y[m]);
            }
        }
    }

#pragma unroll
    for (int m = 0; m < MT; ++m) {
        y[m] += __shfl_xor_sync(FULL, y[m], 1);
        y[m] += __shfl_xor_sync(FULL, y[m], 2);
    }
    if (c == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) red[(warp * 8 + r) * MT + m] = y[m];
    }
    __syncthreads();
    if (tid < 8 * MT) {
        const int rr = tid / MT, m = tid % MT;
        const int64_t n = o * 8 + rr;
        if (m < M && n < a.N) {
            float acc = red[rr * MT + m];
#pragma unroll
            for (int w = 1; w < 8; ++w) acc += red[(w * 8 + rr) * MT + m];
            if (a.out_fp32) static_cast<float *>(a.y)[(int64_t)m * a.N + n] = acc;
            else static_cast<__nv_bfloat16 *>(a.y)[(int64_t)m * a.N + n] = __float2bfloat16_rn(acc);
        }
    }
}

template <int MT>
static w4_status launch_gemv(GemvArgs a, cudaStream_t stream, int64_t N8) {
    const int nck = (int)(a.Kpad / 32);
    const size_t base = 16 + a.slab_bytes + (size_t)MT * nck * 4 + (size_t)64 * MT * 4;
    const size_t xbytes = (size_t)a.M * a.K * 2;
    a.stage_x = (xbytes <= 48 * 1024) ? 1 : 0;
    const size_t smem = base + (a.stage_x ? xbytes : 0);
    if (smem > 200 * 1024) return W4_ERR_SHAPE;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(gemv_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return W4_ERR_CUDA;
    gemv_kernel<MT><<<(unsigned)N8, 256, smem, stream>>>(a);
    return launch_status();
}

}  // namespace w4

using namespace w4;

W4_API w4_status w4a16_gemv(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K, int group,
                            int mode, void *y, int out_fp32, cudaStream_t stream) {
    if (!x_bf16 || !packed || !y) return W4_ERR_NULL;
    if (!valid_mode(mode) || (out_fp32 != 0 && out_fp32 != 1)) return W4_ERR_ARG;
    if (M < 1 || M > 16 || N < 1 || N > (int64_t)0x7fffffff * 8 || K < 32 || K % 32 != 0) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(y)) return W4_ERR_ALIGN;
    const GemvLayout L = gemv_layout(N, K, group);
    GemvArgs a;
    a.x = static_cast<const uint16_t *>(x_bf16);
    a.packed = static_cast<const uint8_t *>(packed);
    a.y = y;
    a.status = device_status_ptr();
    a.N = N; a.K = K; a.Kpad = L.Kpad; a.U = L.U;
    a.codes_bytes = L.codes_bytes;
    a.M = (int)M; a.g = group; a.out_fp32 = out_fp32; a.stage_x = 0;
    a.slab_bytes = (uint32_t)(L.scales_bytes / (size_t)L.N8);
    if (M <= 1) return launch_gemv<1>(a, stream, L.N8);
    if (M <= 2) return launch_gemv<2>(a, stream, L.N8);
    if (M <= 4) return launch_gemv<4>(a, stream, L.N8);
    if (M <= 8) return launch_gemv<8>(a, stream, L.N8);
    return launch_gemv<16>(a, stream, L.N8);
}
