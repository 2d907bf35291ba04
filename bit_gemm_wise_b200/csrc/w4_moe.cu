// Mixture-of-experts plumbing around the grouped W4A8 GEMM: the router and the weighted
// combine ("4-bit by default": MoE expert weights, as in gpt-oss, are the 4-bit target; the
// pages leave the router and the combine open).
//
//  * w4_moe_route: per token the k largest logits (descending; equal logits in ascending
//    expert order), gate weights = softmax of the k selected logits, and the expert-grouped
//    row layout the grouped GEMM takes: rows of expert e are [off[e], off[e+1]), holding
//    its tokens in ascending order; row_of[t, i] is the row of token t's i-th expert.
//    Two launches over blocks of TPB consecutive tokens. Select: one warp per token picks
//    the experts by k rounds of a warp arg-max (value, then lower index), computes the gates,
//    counts the block's tokens per expert into the workspace (cnt[block][e]) and gives every
//    (token, expert) its rank among the block's earlier tokens of that expert. Place: every
//    block sums the counts of the blocks before it and of all blocks, scans the totals into
//    the expert offsets and writes its tokens' rows. No step depends on thread timing.
//  * w4_moe_combine: y[t] = sum_i gates[t, i] * rows[row_of[t, i]] in fp32 (i in order),
//    rounded once to bf16. One block per token, 16-byte chunks.
#include "w4_common.cuh"

namespace w4 {
namespace moe {

constexpr int RT = 256;        // threads of the placement launch
constexpr int TPB = 32;        // tokens per block (one warp each in the selection launch)
constexpr int MAX_E = 1024;
constexpr int MAX_K = 8;

// The oracle's sequential scan (best = first untaken expert, replaced by a strictly larger
// logit) as a warp reduction: if the first untaken logit is NaN it stays the choice;
// otherwise the largest non-NaN untaken logit wins, ties to the lower index. EPL = logits
// per lane (E <= 32 EPL).
template <int EPL>
__global__ void __launch_bounds__(TPB * 32) route_select_kernel(const float *__restrict__ logits, int T, int E, int k,
                                                                int32_t *__restrict__ experts,
                                                                float *__restrict__ gates,
                                                                int32_t *__restrict__ rank,
                                                                int32_t *__restrict__ cnt) {
    __shared__ int sel[TPB][MAX_K];
    __shared__ int cnt_s[MAX_E];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * TPB;
    const int ntok = (int)((T - t0) < TPB ? (T - t0) : TPB);
    for (int e = threadIdx.x; e < E; e += TPB * 32) cnt_s[e] = 0;
    __syncthreads();
    if (warp < ntok) {
        const int tb = warp;
        const float *l = logits + (t0 + tb) * E;
        float v[EPL];
        uint32_t taken = 0;  // bit j: expert lane + 32 j is taken (or does not exist)
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            v[j] = e < E ? __ldg(l + e) : 0.0f;
            if (e >= E) taken |= 1u << j;
        }
        float val[MAX_K];
        int ex[MAX_K];
#pragma unroll
        for (int i = 0; i < MAX_K; ++i) {
            if (i >= k) break;
            // this lane's first untaken expert and its best non-NaN untaken logit
            int first = 0x7fffffff, bi = 0x7fffffff;
            bool first_nan = false;
            float bv = 0.0f;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                if ((taken >> j) & 1u) continue;
                const int e = lane + 32 * j;
                if (first == 0x7fffffff) {
                    first = e;
                    first_nan = v[j] != v[j];
                }
                if (v[j] == v[j] && (bi == 0x7fffffff || v[j] > bv)) {
                    bv = v[j];
                    bi = e;
                }
            }
            const int e0 = (int)__reduce_min_sync(FULL, (unsigned)first);
            const bool nan0 = __ballot_sync(FULL, first == e0 && first_nan) != 0;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                const float ov = __shfl_xor_sync(FULL, bv, off);
                const int oi = __shfl_xor_sync(FULL, bi, off);
                if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
                    bv = ov;
                    bi = oi;
                }
            }
            int best;
            float bval;
            if (nan0 || bi == 0x7fffffff) {  // the second case: every untaken logit is NaN
                best = e0;
                bval = __int_as_float(0x7fc00000);
            } else {
                best = bi;
                bval = bv;
            }
            if ((best & 31) == lane) taken |= 1u << (best >> 5);
            ex[i] = best;
            val[i] = bval;
        }
        // softmax over the selected logits (fp32; every lane computes it, lane i writes slot i)
        const float mx = val[0];
        float den = 0.0f, ev[MAX_K];
#pragma unroll
        for (int i = 0; i < MAX_K; ++i) {
            if (i >= k) break;
            ev[i] = expf(val[i] - mx);
            den += ev[i];
        }
#pragma unroll
        for (int i = 0; i < MAX_K; ++i)
            if (i < k && lane == i) {
                experts[(t0 + tb) * k + i] = ex[i];
                gates[(t0 + tb) * k + i] = ev[i] / den;
                sel[tb][i] = ex[i];
                atomicAdd(&cnt_s[ex[i]], 1);
            }
    }
    __syncthreads();
    // rank of (token, i) among the block's earlier tokens routed to the same expert
    for (int idx = threadIdx.x; idx < ntok * k; idx += TPB * 32) {
        const int tb = idx / k, e = sel[tb][idx - tb * k];
        int r = 0;
        for (int u = 0; u < tb; ++u)
            for (int i = 0; i < k; ++i) r += sel[u][i] == e;
        rank[(t0 + tb) * k + (idx - tb * k)] = r;
    }
    for (int e = threadIdx.x; e < E; e += TPB * 32) cnt[(int64_t)blockIdx.x * E + e] = cnt_s[e];
}

__global__ void __launch_bounds__(RT) route_place_kernel(int T, int E, int k, const int32_t *__restrict__ cnt,
                                                         const int32_t *__restrict__ experts,
                                                         int32_t *__restrict__ off, int32_t *__restrict__ tor,
                                                         int32_t *__restrict__ row_of) {
    __shared__ int before[MAX_E], total[MAX_E], base[MAX_E + 1];
    __shared__ int pb[RT / 32][32], pt[RT / 32][32];
    const int nblk = (T + TPB - 1) / TPB;
    const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // counts of the blocks before this one and of all blocks, 32 experts at a time: lane <->
    // expert, warps stride over the blocks, then the warps' sums are added in warp order
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        int sb = 0, st = 0;
        if (e < E)
            for (int bb = warp; bb < nblk; bb += RT / 32) {
                const int c = __ldg(cnt + (int64_t)bb * E + e);
                st += c;
                if (bb < b) sb += c;
            }
        pb[warp][lane] = sb;
        pt[warp][lane] = st;
        __syncthreads();
        if (warp == 0 && e < E) {
            int a0 = 0, a1 = 0;
            for (int w = 0; w < RT / 32; ++w) {
                a0 += pb[w][lane];
                a1 += pt[w][lane];
            }
            before[e] = a0;
            total[e] = a1;
        }
        __syncthreads();
    }
    // exclusive scan of the totals (one warp, 32 experts at a time)
    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int v = e < E ? total[e] : 0;
            int incl = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int o = __shfl_up_sync(FULL, incl, d);
                if (lane >= d) incl += o;
            }
            if (e < E) base[e] = run + incl - v;
            run += __shfl_sync(FULL, incl, 31);
        }
        if (lane == 0) base[E] = run;
    }
    __syncthreads();
    if (b == 0)
        for (int e = threadIdx.x; e <= E; e += RT) off[e] = base[e];
    const int64_t t0 = (int64_t)b * TPB;
    const int ntok = (int)((T - t0) < TPB ? (T - t0) : TPB);
    for (int idx = threadIdx.x; idx < ntok * k; idx += RT) {
        const int64_t j = t0 * k + idx;
        const int e = experts[j];
        const int r = base[e] + before[e] + row_of[j];
        row_of[j] = r;
        tor[r] = (int32_t)(t0 + idx / k);
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

W4_API int64_t w4_moe_route_workspace_bytes(int64_t T, int E) {
    if (T < 1 || E < 1) return 0;
    return (T + moe::TPB - 1) / moe::TPB * (int64_t)E * 4;
}

W4_API w4_status w4_moe_route(const float *logits, int64_t T, int E, int k, int32_t *experts, float *gates,
                              int32_t *expert_row_offsets, int32_t *token_of_row, int32_t *row_of, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
    if (!logits || !experts || !gates || !expert_row_offsets || !token_of_row || !row_of || !workspace)
        return W4_ERR_NULL;
    if (E < 1 || E > moe::MAX_E || k < 1 || k > moe::MAX_K || k > E || T < 1 || T * k > 0x7fffffffLL)
        return W4_ERR_SHAPE;
    if ((int64_t)workspace_bytes < w4_moe_route_workspace_bytes(T, E)) return W4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(experts) |
         reinterpret_cast<uintptr_t>(gates) | reinterpret_cast<uintptr_t>(expert_row_offsets) |
         reinterpret_cast<uintptr_t>(token_of_row) | reinterpret_cast<uintptr_t>(row_of) |
         reinterpret_cast<uintptr_t>(workspace)) & 3)
        return W4_ERR_ALIGN;
    const unsigned nblk = (unsigned)((T + moe::TPB - 1) / moe::TPB);
    int32_t *cnt = static_cast<int32_t *>(workspace);
    const int epl = (E + 31) / 32;
    auto sel = epl <= 1 ? moe::route_select_kernel<1> : epl <= 2 ? moe::route_select_kernel<2>
             : epl <= 4 ? moe::route_select_kernel<4> : epl <= 8 ? moe::route_select_kernel<8>
             : epl <= 16 ? moe::route_select_kernel<16> : moe::route_select_kernel<32>;
    sel<<<nblk, moe::TPB * 32, 0, stream>>>(logits, (int)T, E, k, experts, gates, row_of, cnt);
    if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
    moe::route_place_kernel<<<nblk, moe::RT, 0, stream>>>((int)T, E, k, cnt, experts, expert_row_offsets,
                                                         token_of_row, row_of);
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
