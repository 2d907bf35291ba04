// w4_prepack: canonical quantized weight -> kernel layout (lossless move of codes,
// scales and zeros; see w4_layout.cuh). One thread per output 32-bit word.
#include "w4_common.cuh"
#include "w4_layout.cuh"

namespace w4 {

__device__ __forceinline__ uint32_t nib_at(const uint8_t *codes, int64_t N, int64_t K, int64_t n, int64_t k) {
    if (n >= N || k >= K) return 0;
    const uint8_t b = codes[n * (K / 2) + (k >> 1)];
    return (k & 1) ? (b >> 4) : (b & 0xF);
}

__device__ __forceinline__ uint32_t scale_entry(const uint16_t *scales, const int16_t *zeros, int64_t N, int64_t J,
                                                int64_t n, int64_t j) {
    if (n >= N || j >= J) return 0;
    const uint32_t s = scales[n * J + j];
    const uint32_t z = zeros ? (uint16_t)zeros[n * J + j] : 8u;
    return s | (z << 16);
}

// W4_LAYOUT_GEMV: one thread per 32-bit word of the row records
__global__ void prepack_gemv_rows(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ scales,
                                  const int16_t *__restrict__ zeros, int64_t N, int64_t K, int g,
                                  int64_t row_words, int64_t nwords, uint32_t *__restrict__ out) {
    const int64_t J = K / g, cw = K / 8;  // code words per row
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < nwords;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = idx / row_words, w = idx - n * row_words;
        uint32_t v;
        if (w < cw) v = reinterpret_cast<const uint32_t *>(codes + n * (K / 2))[w];
        else v = scale_entry(scales, zeros, N, J, n, w - cw);
        out[idx] = v;
    }
}

__global__ void prepack_gemm_codes(const uint8_t *__restrict__ codes, int64_t N, int64_t K, int64_t Kpad,
                                   int64_t nwords, uint32_t *__restrict__ out) {
    const int64_t wpr = Kpad / 8;  // words per row
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < nwords;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = idx / wpr;
        const int64_t k0 = (idx % wpr) * 8;
        uint32_t word = 0;
        for (int p = 0; p < 8; ++p) word |= nib_at(codes, N, K, n, k0 + p / 2 + 4 * (p % 2)) << (4 * p);
        out[idx] = word;
    }
}

__global__ void prepack_gemm_scales(const uint16_t *__restrict__ scales, const int16_t *__restrict__ zeros,
                                    int64_t N, int64_t K, int g, int64_t Npad, int64_t nent,
                                    uint32_t *__restrict__ out) {
    const int64_t J = K / g;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < nent;
         idx += (int64_t)gridDim.x * blockDim.x)
        out[idx] = scale_entry(scales, zeros, N, J, idx % Npad, idx / Npad);
}

// bf16 round-to-nearest-even bit pattern of a finite fp32 value
__device__ __forceinline__ uint32_t bf16_rn_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// zero-point operand: one thread per 32-bit word (two bf16 columns) of [Npad][KZ]
__global__ void prepack_gemm_zop(const uint16_t *__restrict__ scales, const int16_t *__restrict__ zeros, int64_t N,
                                 int64_t Jr, int64_t KZ, int64_t nwords, uint32_t *__restrict__ out) {
    const int64_t wpr = KZ / 2;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < nwords;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = idx / wpr;
        uint32_t word = 0;
        for (int h = 0; h < 2; ++h) {
            const int64_t c = (idx % wpr) * 2 + h;
            const int64_t part = c / Jr, j = c - part * Jr;
            uint32_t v = 0;
            if (n < N && part < 3) {
                const float sc = __half2float(__ushort_as_half(scales[n * Jr + j]));
                const float z = zeros ? (float)zeros[n * Jr + j] : 8.0f;
                const float sz = __fmul_rn(sc, z);
                const uint32_t hi = bf16_rn_bits(sz);
                v = (part < 2) ? hi : bf16_rn_bits(__fsub_rn(sz, __uint_as_float(hi << 16)));
            }
            word |= v << (16 * h);
        }
        out[idx] = word;
    }
}

// W4_LAYOUT_TC: one thread per 32-bit word of the unit records
__global__ void prepack_tc(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ scales,
                           const int16_t *__restrict__ zeros, int64_t N, int64_t K, int g, int64_t NKB,
                           int64_t nwords, uint32_t *__restrict__ out) {
    const int ks = TcLayoutGeo::ks(g);
    const int64_t rec_words = TcLayoutGeo::record_bytes(g) / 4, code_words = TcLayoutGeo::code_bytes(g) / 4;
    const int64_t J = K / g;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < nwords;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t u = idx / rec_words, wr = idx - u * rec_words;
        const int64_t t = u / NKB, kb = u - t * NKB;
        uint32_t v = 0;
        if (wr < code_words) {
            const int64_t c = wr / (128 * 4), r = (wr / 4) % 128, i = wr % 4;
            const int64_t n = t * 128 + r, k0 = kb * ks + c * 32 + i * 8;
            for (int p = 0; p < 8; ++p) v |= nib_at(codes, N, K, n, k0 + (p < 4 ? 2 * p : 2 * (p - 4) + 1)) << (4 * p);
        } else {
            const int64_t e = wr - code_words, gg = e / 128, r = e % 128;
            v = scale_entry(scales, zeros, N, J, t * 128 + r, kb * (ks / g) + gg);
        }
        out[idx] = v;
    }
}

static int grid_for(int64_t n) {
    const int64_t b = (n + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 32;
    return (int)(b < cap ? (b > 0 ? b : 1) : cap);
}

}  // namespace w4

using namespace w4;

W4_API size_t w4_prepack_bytes(int64_t N, int64_t K, int group, int layout) {
    if (N < 1 || K < 32 || K % 32 != 0 || !valid_group(group) || K % group != 0) return 0;
    if (layout == W4_LAYOUT_GEMV) return gemv_layout(N, K, group).total;
    if (layout == W4_LAYOUT_GEMM) return gemm_layout(N, K, group).total;
    if (layout == W4_LAYOUT_TC) return tc_layout(N, K, group).total;
    return 0;
}

W4_API w4_status w4_prepack(const uint8_t *codes, const uint16_t *scales_fp16, const int16_t *zeros, int64_t N,
                            int64_t K, int group, int mode, int layout, void *packed, cudaStream_t stream) {
    if (!codes || !scales_fp16 || !packed) return W4_ERR_NULL;
    if (!valid_mode(mode)) return W4_ERR_ARG;
    if (mode == W4_ASYM && !zeros) return W4_ERR_NULL;
    if (mode == W4_SYM && zeros) return W4_ERR_ARG;
    if (N < 1 || K < 32 || K % 32 != 0) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (layout != W4_LAYOUT_GEMV && layout != W4_LAYOUT_GEMM && layout != W4_LAYOUT_TC) return W4_ERR_ARG;
    if (!aligned16(codes) || !aligned16(scales_fp16) || (zeros && !aligned16(zeros)) || !aligned16(packed))
        return W4_ERR_ALIGN;
    uint8_t *base = static_cast<uint8_t *>(packed);
    if (layout == W4_LAYOUT_GEMV) {
        const GemvLayout L = gemv_layout(N, K, group);
        const int64_t row_words = (int64_t)(L.row_bytes / 4);
        const int64_t nwords = (int64_t)(L.total / 4);
        prepack_gemv_rows<<<grid_for(nwords), 256, 0, stream>>>(codes, scales_fp16, zeros, N, K, group, row_words,
                                                                nwords, reinterpret_cast<uint32_t *>(base));
    } else if (layout == W4_LAYOUT_TC) {
        const TcLayout L = tc_layout(N, K, group);
        const int64_t nwords = (int64_t)(L.total / 4);
        prepack_tc<<<grid_for(nwords), 256, 0, stream>>>(codes, scales_fp16, zeros, N, K, group, L.NKB, nwords,
                                                         reinterpret_cast<uint32_t *>(base));
    } else {
        const GemmLayout L = gemm_layout(N, K, group);
        const int64_t nwords = (int64_t)(L.codes_bytes / 4);
        const int64_t nent = (int64_t)(L.scales_bytes / 4);
        prepack_gemm_codes<<<grid_for(nwords), 256, 0, stream>>>(codes, N, K, L.Kpad, nwords,
                                                                 reinterpret_cast<uint32_t *>(base));
        prepack_gemm_scales<<<grid_for(nent), 256, 0, stream>>>(scales_fp16, zeros, N, K, group, L.Npad, nent,
                                                                reinterpret_cast<uint32_t *>(base + L.codes_bytes));
        const int64_t zwords = (int64_t)(L.zop_bytes / 4);
        prepack_gemm_zop<<<grid_for(zwords), 256, 0, stream>>>(
            scales_fp16, zeros, N, L.Jr, L.KZ, zwords, reinterpret_cast<uint32_t *>(base + L.codes_bytes + L.scales_bytes));
    }
    return launch_status();
}
