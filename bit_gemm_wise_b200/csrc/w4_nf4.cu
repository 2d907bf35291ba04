// NF4 comparator: the normal-quantile 4-bit format the pages set against their W4A8 path
// ("Quantizing LLMs Without Guesswork", NF4 paragraph: 16 levels that are quantiles of a
// normal distribution, blocks of 64, dequantized to 16-bit before the matmul; "Four-bit
// inference ... Tahoma": the NF4 operating point the W4A8 path is measured against).
//
// Levels: the QLoRA construction (the pages leave it open) -- with delta = (1/32 + 1/30)/2,
// eight positive quantiles Phi^-1(p) at p = 1 - delta + i (delta - 1/2) / 8 (i = 0..7), seven
// negative ones at p = 1 - delta + i (delta - 1/2) / 7 (i = 0..6), an exact zero, all divided
// by Phi^-1(1 - delta). They are computed once on the host here: Phi^-1 by a rational first
// guess (Acklam's approximation of the normal quantile) refined by Halley steps on
// erfc(-x / sqrt(2)) / 2 - p in double precision, then rounded to fp32.
//
//  * w4_nf4_quantize: one warp per block of 64 (two weights per lane): a = max|w| by
//    shuffles, t = w / a (IEEE), code = the level nearest to t (fp32 distances, ties to the
//    lower level); a zero block takes the zero level. Codes are packed like the INT4 ones.
//  * w4_nf4_gemv: y[m, n] = sum_k x[m, k] * level[q[n, k]] * a[n, k / 64]. Activations are
//    staged once per block as fp32; the code bytes are looked up in a 256-entry table of level
//    pairs and multiplied with packed fp32 FMAs; each warp takes whole rows (16 bytes of codes
//    per lane per step), the block's partial sums are scaled by the block's absmax, and the
//    row is reduced over the warp in a fixed order.
#include "w4_common.cuh"

#include <math.h>
#include <mutex>

namespace w4 {
namespace nf4 {

struct Levels {
    float v[16];
    int zero_code;
};

// Acklam's rational approximation to the normal quantile (relative error ~1e-9), then two
// Halley steps on Phi(x) - p with Phi(x) = erfc(-x / sqrt(2)) / 2.
static double normal_quantile(double p) {
    static const double a[6] = {-3.969683028665376e+01, 2.209460984245205e+02, -2.759285104469687e+02,
                                1.383577518672690e+02, -3.066479806614716e+01, 2.506628277459239e+00};
    static const double b[5] = {-5.447609879822406e+01, 1.615858368580409e+02, -1.556989798598866e+02,
                                6.680131188771972e+01, -1.328068155288572e+01};
    static const double c[6] = {-7.784894002430293e-03, -3.223964580411365e-01, -2.400758277161838e+00,
                                -2.549732539343734e+00, 4.374664141464968e+00, 2.938163982698783e+00};
    static const double d[4] = {7.784695709041462e-03, 3.224671290700398e-01, 2.445134137142996e+00,
                                3.754408661907416e+00};
    const double pl = 0.02425, ph = 1.0 - pl;
    double x;
    if (p < pl) {
        const double q = sqrt(-2.0 * log(p));
        x = (((((c[0] * q + c[1]) * q + c[2]) * q + c[3]) * q + c[4]) * q + c[5]) /
            ((((d[0] * q + d[1]) * q + d[2]) * q + d[3]) * q + 1.0);
    } else if (p <= ph) {
        const double q = p - 0.5, r = q * q;
        x = (((((a[0] * r + a[1]) * r + a[2]) * r + a[3]) * r + a[4]) * r + a[5]) * q /
            (((((b[0] * r + b[1]) * r + b[2]) * r + b[3]) * r + b[4]) * r + 1.0);
    } else {
        const double q = sqrt(-2.0 * log(1.0 - p));
        x = -(((((c[0] * q + c[1]) * q + c[2]) * q + c[3]) * q + c[4]) * q + c[5]) /
            ((((d[0] * q + d[1]) * q + d[2]) * q + d[3]) * q + 1.0);
    }
    for (int it = 0; it < 2; ++it) {
        const double e = 0.5 * erfc(-x / sqrt(2.0)) - p;
        const double u = e * sqrt(2.0 * M_PI) * exp(0.5 * x * x);
        x = x - u / (1.0 + 0.5 * x * u);
    }
    return x;
}

static const Levels &levels() {
    static Levels L;
    static std::once_flag once;
    std::call_once(once, [] {
        const double delta = 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
        const double top = normal_quantile(1.0 - delta);
        double v[16];
        int n = 0;
        for (int i = 0; i < 7; ++i) v[n++] = -normal_quantile(1.0 - delta + i * (delta - 0.5) / 7.0) / top;
        L.zero_code = n;
        v[n++] = 0.0;
        for (int i = 7; i >= 0; --i) v[n++] = normal_quantile(1.0 - delta + i * (delta - 0.5) / 8.0) / top;
        for (int i = 0; i < 16; ++i) L.v[i] = (float)v[i];
        L.v[0] = -1.0f;  // -Phi^-1(1 - delta) / Phi^-1(1 - delta)
        L.v[15] = 1.0f;
    });
    return L;
}

__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t *__restrict__ W, int64_t K, int64_t blocks,
                                                       Levels L, uint8_t *__restrict__ codes,
                                                       float *__restrict__ absmax) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t b = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); b < blocks; b += nwarps) {
        const int64_t n = b / (K / 64), j = b - n * (K / 64);
        const uint32_t v = reinterpret_cast<const uint32_t *>(W + n * K + j * 64)[lane];
        const float w0 = bf16_lo(v), w1 = bf16_hi(v);
        float a = fmaxf(fabsf(w0), fabsf(w1));
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
        int q[2] = {L.zero_code, L.zero_code};
        if (a > 0.0f) {
            const float t[2] = {__fdiv_rn(w0, a), __fdiv_rn(w1, a)};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                int best = 0;
                float bd = fabsf(__fsub_rn(t[h], L.v[0]));
#pragma unroll
                for (int c = 1; c < 16; ++c) {
                    const float d = fabsf(__fsub_rn(t[h], L.v[c]));
                    if (d < bd) { bd = d; best = c; }
                }
                q[h] = best;
            }
        }
        codes[n * (K / 2) + j * 32 + lane] = (uint8_t)(q[0] | (q[1] << 4));
        if (lane == 0) absmax[n * (K / 64) + j] = a;
    }
}

constexpr int GEMV_THREADS = 256;

// M activation rows (1..4), rows of W strided over all warps of the grid
template <int M>
__global__ void __launch_bounds__(GEMV_THREADS, 1) gemv_kernel(const uint16_t *__restrict__ x,
                                                            const uint8_t *__restrict__ codes,
                                                            const float *__restrict__ absmax, int64_t N, int64_t K,
                                                            Levels L, void *y, int out_fp32, int pdl) {
    extern __shared__ __align__(16) uint8_t smem[];
    float2 *lut = reinterpret_cast<float2 *>(smem);                 // [256]: levels of a code byte
    float *xs = reinterpret_cast<float *>(smem + 256 * sizeof(float2));  // [M][K]
    for (int i = threadIdx.x; i < 256; i += blockDim.x) lut[i] = make_float2(L.v[i & 15], L.v[i >> 4]);
    if (pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int64_t i = threadIdx.x; i < (int64_t)M * K / 2; i += blockDim.x) {
        const uint32_t v = reinterpret_cast<const uint32_t *>(x)[i];
        reinterpret_cast<float2 *>(xs)[i] = make_float2(bf16_lo(v), bf16_hi(v));
    }
    __syncthreads();
    if (pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t nch = K / 32;  // 16-byte chunks of a row (32 weights, half an NF4 block)
    for (int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N; n += nwarps) {
        const uint4 *crow = reinterpret_cast<const uint4 *>(codes + n * (K / 2));
        const float *arow = absmax + n * (K / 64);
        float acc[M];
#pragma unroll
        for (int m = 0; m < M; ++m) acc[m] = 0.0f;
        for (int64_t c0 = 0; c0 < nch; c0 += 64) {
            // two chunks per lane in flight
            const int64_t ca = c0 + lane, cb = c0 + 32 + lane;
            const uint4 va = ca < nch ? __ldg(crow + ca) : make_uint4(0u, 0u, 0u, 0u);
            const uint4 vb = cb < nch ? __ldg(crow + cb) : make_uint4(0u, 0u, 0u, 0u);
            const float aa = ca < nch ? __ldg(arow + ca / 2) : 0.0f, ab = cb < nch ? __ldg(arow + cb / 2) : 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t c = h ? cb : ca;
                if (c >= nch) break;
                const uint4 v = h ? vb : va;
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    float2 s = make_float2(0.0f, 0.0f);
                    const float2 *xr = reinterpret_cast<const float2 *>(xs + (int64_t)m * K + c * 32);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 w = lut[(wv[i >> 2] >> (8 * (i & 3))) & 0xFFu];
                        s = __ffma2_rn(xr[i], w, s);
                    }
                    acc[m] = __fmaf_rn(__fadd_rn(s.x, s.y), h ? ab : aa, acc[m]);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < M; ++m) {
            float r = acc[m];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) r += __shfl_xor_sync(FULL, r, off);
            if (lane == 0) {
                if (out_fp32) static_cast<float *>(y)[m * N + n] = r;
                else static_cast<__nv_bfloat16 *>(y)[m * N + n] = __float2bfloat16_rn(r);
            }
        }
    }
}


// M = 1 with K a multiple of 1024 up to 16384: one block per SM owns a contiguous run of rows;
// thread (slot, sl) takes the 16-byte code chunk sl (32 weights, half an NF4 block) of the rows
// slot, slot + nslot, ... and holds its 32 activations in registers. The code chunks and block
// scales of the next PF rows are loaded ahead in registers (issued before the dependency wait
// under programmatic launch), and the chunks PF rows beyond those are prefetched into L2, so
// that the register loads find them there. Each code is looked up in a 16-entry fp32 table in shared
// memory (one entry per bank, so any lookup pattern is conflict-free) and multiplied into one
// of four fp32 sums; the chunk's sum times the block scale is reduced over the warp, then over
// the row's warps in order.
constexpr int RT = 512;
constexpr int PF = 4;
constexpr int MAX_RPB = 256;

__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float lut_at(const float *lut, uint32_t byte_off) {
    return *reinterpret_cast<const float *>(reinterpret_cast<const char *>(lut) + byte_off);
}

__global__ void __launch_bounds__(RT, 1) gemv_rows_kernel(const uint16_t *__restrict__ x,
                                                          const uint8_t *__restrict__ codes,
                                                          const float *__restrict__ absmax, int64_t N, int64_t K,
                                                          Levels L, void *y, int out_fp32, int pdl, int rpb) {
    __shared__ float lut[16];
    __shared__ float red[MAX_RPB * 16];  // [row][warp of the row]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wpr = (int)(K / 1024);          // warps per row
    const int nslot = (RT / 32) / wpr;        // rows in flight
    const int slot = warp / wpr, ws = warp - slot * wpr;
    const int sl = ws * 32 + lane;            // 16-byte chunk of the row
    const bool active = slot < nslot;
    const int64_t row0 = (int64_t)blockIdx.x * rpb;
    const int rows = (int)((N - row0) < rpb ? (N - row0) : rpb);
    const int nr = active && slot < rows ? (rows - slot + nslot - 1) / nslot : 0;  // rows of this slot
    const int64_t rb = K / 2, ab = K / 64;    // code bytes and block scales per row
    if (tid < 16) lut[tid] = L.v[tid];
    uint4 cq[PF];
    float aq[PF];
#pragma unroll
    for (int p = 0; p < PF; ++p) {
        const int64_t n = row0 + slot + (int64_t)p * nslot;
        const bool ok = p < nr;
        cq[p] = ok ? __ldg(reinterpret_cast<const uint4 *>(codes + n * rb) + sl) : make_uint4(0u, 0u, 0u, 0u);
        aq[p] = ok ? __ldg(absmax + n * ab + (sl >> 1)) : 0.0f;
        if (p + PF < nr) prefetch_l2(reinterpret_cast<const uint4 *>(codes + (n + (int64_t)PF * nslot) * rb) + sl);
    }
    __syncthreads();
    if (pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    float xr[32];
    {
        const uint4 *xs = reinterpret_cast<const uint4 *>(x) + (int64_t)sl * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = active ? __ldg(xs + q) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xr[8 * q + 2 * i] = bf16_lo(u[i]);
                xr[8 * q + 2 * i + 1] = bf16_hi(u[i]);
            }
        }
    }
    if (pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int i = 0; i < nr; ++i) {
        const uint4 c = cq[0];
        const float am = aq[0];
#pragma unroll
        for (int p = 0; p + 1 < PF; ++p) {
            cq[p] = cq[p + 1];
            aq[p] = aq[p + 1];
        }
        {
            const int64_t n = row0 + slot + (int64_t)(i + PF) * nslot;
            const bool ok = i + PF < nr;
            cq[PF - 1] = ok ? __ldg(reinterpret_cast<const uint4 *>(codes + n * rb) + sl) : make_uint4(0u, 0u, 0u, 0u);
            aq[PF - 1] = ok ? __ldg(absmax + n * ab + (sl >> 1)) : 0.0f;
            if (i + 2 * PF < nr) prefetch_l2(reinterpret_cast<const uint4 *>(codes + (n + (int64_t)PF * nslot) * rb) + sl);
        }
        const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint32_t lo = (wv[w] & 0x0F0F0F0Fu) << 2;  // byte b: 4 q[8w + 2b]
            const uint32_t hi = (wv[w] >> 2) & 0x3C3C3C3Cu;  // byte b: 4 q[8w + 2b + 1]
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t sel = 0x4440u | (uint32_t)b;
                acc[(2 * b) & 3] = __fmaf_rn(lut_at(lut, __byte_perm(lo, 0u, sel)), xr[8 * w + 2 * b], acc[(2 * b) & 3]);
                acc[(2 * b + 1) & 3] =
                    __fmaf_rn(lut_at(lut, __byte_perm(hi, 0u, sel)), xr[8 * w + 2 * b + 1], acc[(2 * b + 1) & 3]);
            }
        }
        float r = __fmul_rn(__fadd_rn(__fadd_rn(acc[0], acc[1]), __fadd_rn(acc[2], acc[3])), am);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) r += __shfl_xor_sync(FULL, r, off);
        if (lane == 0) red[(slot + i * nslot) * 16 + ws] = r;
    }
    __syncthreads();
    for (int rl = tid; rl < rows; rl += RT) {
        float acc = 0.0f;
        for (int w = 0; w < wpr; ++w) acc += red[rl * 16 + w];
        const int64_t n = row0 + rl;
        if (out_fp32) static_cast<float *>(y)[n] = acc;
        else static_cast<__nv_bfloat16 *>(y)[n] = __float2bfloat16_rn(acc);
    }
}

}  // namespace nf4
}  // namespace w4

using namespace w4;

W4_API w4_status w4_nf4_levels(float *levels_host) {
    if (!levels_host) return W4_ERR_NULL;
    for (int i = 0; i < 16; ++i) levels_host[i] = nf4::levels().v[i];
    return W4_OK;
}

W4_API w4_status w4_nf4_quantize(const void *W_bf16, int64_t N, int64_t K, uint8_t *codes, float *absmax,
                                 cudaStream_t stream) {
    if (!W_bf16 || !codes || !absmax) return W4_ERR_NULL;
    if (N < 1 || K < 64 || K % 64 != 0) return W4_ERR_SHAPE;
    if (!aligned16(W_bf16) || !aligned16(codes) || !aligned16(absmax)) return W4_ERR_ALIGN;
    const int64_t blocks = N * (K / 64);
    const int64_t want = (blocks + 7) / 8;
    const int grid = (int)(want < (int64_t)num_sms() * 32 ? want : (int64_t)num_sms() * 32);
    nf4::quantize_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(W_bf16), K, blocks, nf4::levels(),
                                                   codes, absmax);
    return launch_status();
}

W4_API w4_status w4_nf4_gemv(const void *x_bf16, int64_t M, const uint8_t *codes, const float *absmax, int64_t N,
                             int64_t K, void *y, int flags, cudaStream_t stream) {
    if (!x_bf16 || !codes || !absmax || !y) return W4_ERR_NULL;
    if ((flags & ~(W4_OUT_FP32 | W4_OVERLAP_PREVIOUS))) return W4_ERR_ARG;
    if (M < 1 || M > 4 || N < 1 || K < 64 || K % 64 != 0) return W4_ERR_SHAPE;
    const size_t smem = 256 * sizeof(float2) + (size_t)M * K * sizeof(float);
    if (smem > 227 * 1024) return W4_ERR_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(absmax) || !aligned16(y)) return W4_ERR_ALIGN;
    const int out_fp32 = (flags & W4_OUT_FP32) ? 1 : 0, pdl = (flags & W4_OVERLAP_PREVIOUS) ? 1 : 0;
    if (M == 1 && K % 1024 == 0 && K <= 16384) {
        // one block per SM, contiguous row runs of at most MAX_RPB rows
        const int64_t sms = num_sms();
        int64_t grid = sms < N ? sms : N;
        if ((N + grid - 1) / grid > nf4::MAX_RPB) grid = (N + nf4::MAX_RPB - 1) / nf4::MAX_RPB;
        const int rpb = (int)((N + grid - 1) / grid);
        grid = (N + rpb - 1) / rpb;
        if (grid > 0x7fffffffLL) return W4_ERR_SHAPE;
        const nf4::Levels L = nf4::levels();
        const uint16_t *xp = static_cast<const uint16_t *>(x_bf16);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(nf4::RT);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = pdl;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        void *args[] = {(void *)&xp, (void *)&codes, (void *)&absmax, (void *)&N, (void *)&K, (void *)&L, &y,
                        (void *)&out_fp32, (void *)&pdl, (void *)&rpb};
        if (cudaLaunchKernelExC(&cfg, reinterpret_cast<void *>(nf4::gemv_rows_kernel), args) != cudaSuccess)
            return W4_ERR_CUDA;
        return launch_status();
    }
    const int64_t want = (N + 7) / 8;  // a warp per row, 8 warps per block
    const int grid = (int)(want < (int64_t)num_sms() * 2 ? want : (int64_t)num_sms() * 2);
    void *fn = M == 1 ? reinterpret_cast<void *>(nf4::gemv_kernel<1>)
             : M == 2 ? reinterpret_cast<void *>(nf4::gemv_kernel<2>)
             : M == 3 ? reinterpret_cast<void *>(nf4::gemv_kernel<3>) : reinterpret_cast<void *>(nf4::gemv_kernel<4>);
    static int attr_done[64][4] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev][M - 1]) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev][M - 1] = 1;
    }
    const nf4::Levels L = nf4::levels();
    const uint16_t *xp = static_cast<const uint16_t *>(x_bf16);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(nf4::GEMV_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[] = {(void *)&xp, (void *)&codes, (void *)&absmax, (void *)&N, (void *)&K, (void *)&L, &y,
                    (void *)&out_fp32, (void *)&pdl};
    if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}
