// Mixture-of-experts plumbing around the grouped W4A8 GEMM: the router and the weighted
// combine ("4-bit by default": MoE expert weights, as in gpt-oss, are the 4-bit target; the
// pages leave the router and the combine open).
//
//  * w4_moe_route: per token the k largest logits (descending; equal logits in ascending
//    expert order), gate weights = softmax of the k selected logits, and the expert-grouped
//    row layout the grouped GEMM takes: rows of expert e are [off[e], off[e+1]), holding
//    its tokens in ascending order; row_of[t, i] is the row of token t's i-th expert.
//    One block: every thread routes tokens and counts them per expert in shared memory;
//    then one warp per expert walks the tokens in order with ballots to give each routed
//    token its rank (so the layout is deterministic).
//  * w4_moe_combine: y[t] = sum_i gates[t, i] * rows[row_of[t, i]] in fp32 (i in order),
//    rounded once to bf16. One block per token, 16-byte chunks.
#include "w4_common.cuh"

namespace w4 {
namespace moe {

constexpr int ROUTE_THREADS = 1024;
constexpr int MAX_E = 1024;
constexpr int MAX_K = 8;
constexpr int ROUTE_SMEM = 96 * 1024;  // membership bits: T * ceil(E / 32) words

__global__ void __launch_bounds__(ROUTE_THREADS) route_kernel(const float *__restrict__ logits, int T, int E, int k,
                                                              int32_t *__restrict__ experts, float *__restrict__ gates,
                                                              int32_t *__restrict__ off, int32_t *__restrict__ tor,
                                                              int32_t *__restrict__ row_of) {
    extern __shared__ uint32_t member[];  // [T][EW]
    __shared__ int cnt[MAX_E];
    __shared__ int base[MAX_E + 1];
    const int EW = (E + 31) / 32;
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    for (int i = threadIdx.x; i < T * EW; i += blockDim.x) member[i] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
        const float *l = logits + (int64_t)t * E;
        int sel[MAX_K];
        for (int i = 0; i < k; ++i) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                bool taken = false;
                for (int j = 0; j < i; ++j) taken |= sel[j] == e;
                if (!taken && (best < 0 || l[e] > l[best])) best = e;
            }
            sel[i] = best;
            experts[(int64_t)t * k + i] = best;
            atomicOr(&member[t * EW + (best >> 5)], 1u << (best & 31));
            atomicAdd(&cnt[best], 1);
        }
        const float mx = l[sel[0]];
        float den = 0.0f, ev[MAX_K];
        for (int i = 0; i < k; ++i) {
            ev[i] = expf(l[sel[i]] - mx);
            den += ev[i];
        }
        for (int i = 0; i < k; ++i) gates[(int64_t)t * k + i] = ev[i] / den;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int e = 0; e < E; ++e) {
            base[e] = acc;
            off[e] = acc;
            acc += cnt[e];
        }
        base[E] = acc;
        off[E] = acc;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int e = warp; e < E; e += nw) {
        int run = base[e];
        for (int t0 = 0; t0 < T; t0 += 32) {
            const int t = t0 + lane;
            const bool in = t < T && ((member[t * EW + (e >> 5)] >> (e & 31)) & 1u);
            const uint32_t m = __ballot_sync(FULL, in);
            if (in) {
                const int r = run + __popc(m & ((1u << lane) - 1u));
                tor[r] = t;
                for (int i = 0; i < k; ++i)
                    if (experts[(int64_t)t * k + i] == e) row_of[(int64_t)t * k + i] = r;
            }
            run += __popc(m);
        }
    }
}

__global__ void __launch_bounds__(256) combine_kernel(const uint16_t *__restrict__ rows, int64_t N, int64_t R,
                                                      const int32_t *__restrict__ row_of,
                                                      const float *__restrict__ gates, int k,
                                                      uint16_t *__restrict__ y, int *status) {
    const int64_t t = blockIdx.x;
    int64_t ri[MAX_K];
    float gi[MAX_K];
    for (int i = 0; i < k; ++i) {
        ri[i] = row_of[t * k + i];
        gi[i] = gates[t * k + i];
        if (ri[i] < 0 || ri[i] >= R) {
            if (threadIdx.x == 0) record_status(status, W4_ERR_DEVICE_CHECK);
            ri[i] = -1;
        }
    }
    const int64_t nch = N / 8;
    for (int64_t c = threadIdx.x; c < nch; c += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
        for (int i = 0; i < k; ++i) {
            if (ri[i] < 0) continue;
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(rows + ri[i] * N) + c);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[2 * j] = __fmaf_rn(gi[i], bf16_lo(u[j]), acc[2 * j]);
                acc[2 * j + 1] = __fmaf_rn(gi[i], bf16_hi(u[j]), acc[2 * j + 1]);
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
            o[j] = *reinterpret_cast<const uint32_t *>(&b);
        }
        reinterpret_cast<uint4 *>(y + t * N)[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace moe
}  // namespace w4

using namespace w4;

W4_API w4_status w4_moe_route(const float *logits, int64_t T, int E, int k, int32_t *experts, float *gates,
                              int32_t *expert_row_offsets, int32_t *token_of_row, int32_t *row_of,
                              cudaStream_t stream) {
    if (!logits || !experts || !gates || !expert_row_offsets || !token_of_row || !row_of) return W4_ERR_NULL;
    if (E < 1 || E > moe::MAX_E || k < 1 || k > moe::MAX_K || k > E || T < 1) return W4_ERR_SHAPE;
    const int64_t words = T * ((E + 31) / 32);
    if (words * 4 > moe::ROUTE_SMEM || T * k > 0x7fffffffLL) return W4_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(experts) |
         reinterpret_cast<uintptr_t>(gates) | reinterpret_cast<uintptr_t>(expert_row_offsets) |
         reinterpret_cast<uintptr_t>(token_of_row) | reinterpret_cast<uintptr_t>(row_of)) & 3)
        return W4_ERR_ALIGN;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(moe::route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, moe::ROUTE_SMEM) !=
            cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev] = 1;
    }
    moe::route_kernel<<<1, moe::ROUTE_THREADS, (size_t)words * 4, stream>>>(
        logits, (int)T, E, k, experts, gates, expert_row_offsets, token_of_row, row_of);
    return launch_status();
}

W4_API w4_status w4_moe_combine(const void *rows_bf16, int64_t N, int64_t R, const int32_t *row_of,
                                const float *gates, int64_t T, int k, void *y_bf16, cudaStream_t stream) {
    if (!rows_bf16 || !row_of || !gates || !y_bf16) return W4_ERR_NULL;
    if (N < 8 || N % 8 != 0 || R < 1 || T < 1 || T > 0x7fffffffLL || k < 1 || k > moe::MAX_K) return W4_ERR_SHAPE;
    if (!aligned16(rows_bf16) || !aligned16(y_bf16) ||
        ((reinterpret_cast<uintptr_t>(row_of) | reinterpret_cast<uintptr_t>(gates)) & 3))
        return W4_ERR_ALIGN;
    moe::combine_kernel<<<(unsigned)T, 256, 0, stream>>>(static_cast<const uint16_t *>(rows_bf16), N, R, row_of, gates,
                                                         k, static_cast<uint16_t *>(y_bf16), device_status_ptr());
    return launch_status();
}
