// w4a16_gemv: weight-only INT4 GEMV for decode, dequantization fused into the product.
//
// "Quantizing LLMs Without Guesswork", The Problem & Context (decode reads every weight
// once and that read sets the pace) and Weight-only methods (4-bit weights, 16-bit
// activations, dequantized inside the matmul).
//
//   y[m, n] = sum_j s[n,j] * sum_{k in j} x[m,k] * (q[n,k] - z[n,j])
//
// HBM-bound streaming kernel on the CUDA cores (W4_LAYOUT_GEMV, see w4_layout.cuh).
//  * Persistent stream-K: the weight is a sequence of T = (N/8) * (Kpad/128) units of
//    512 bytes (8 rows x 128 k) in octet-major order; CTA c of P (one per SM) owns the
//    contiguous unit range [t0, t1) with |t1 - t0| differing by at most one between CTAs,
//    so every SM streams the same number of bytes whatever N and K are.
//  * Warp w of a CTA takes units t0 + w, t0 + w + W, ... (so the W warps read W
//    consecutive 512-byte units, i.e. contiguous memory) and keeps a queue of the next
//    units' codes and scales in registers (128-bit streaming loads that bypass L1), so
//    each SM keeps ~64 KB of loads in flight. The activations (and the per-32-chunk
//    activation sums) are staged once per CTA in shared memory with a bulk copy
//    (cp.async.bulk, bounded mbarrier wait).
//  * A lane (row r = lane/4, chunk c = lane%4) turns a 16-byte word of codes into bf16
//    pairs with one AND/OR each
//    ((w & 0x000F000F) | 0x43004300 is the exact pair 128 + q), multiplies them into fp32
//    with fma.rn.f32.bf16, and removes the offset per 32-wide chunk with the chunk's
//    activation sum: sum x*(q - z) = sum x*(128 + q) - (128 + z) * sum x. The chunk
//    partial times the fp16 group scale is accumulated per octet in registers.
//  * Octets wholly inside a CTA's range are reduced in shared memory (fixed warp order)
//    and written. An octet split between CTAs is finished by the last of its CTAs to
//    arrive on a per-octet counter: it adds the CTAs' partials in CTA order (so results are
//    deterministic) and resets the counter. Partials and counters live in the caller's
//    workspace, which every call leaves zero-filled.
#include "w4_common.cuh"
#include "w4_layout.cuh"

#include <mutex>

namespace w4 {
namespace gemv {

constexpr int SMEM_LIMIT = 100 * 1024;
constexpr int PF = 4;  // units queued per warp

__device__ __forceinline__ void fma2_bf16(float &a0, float &a1, uint32_t x, uint32_t q) {
    asm("{\n .reg .b16 xl, xh, ql, qh;\n mov.b32 {xl, xh}, %2;\n mov.b32 {ql, qh}, %3;\n"
        " fma.rn.f32.bf16 %0, xl, ql, %0;\n fma.rn.f32.bf16 %1, xh, qh, %1;\n}\n"
        : "+f"(a0), "+f"(a1)
        : "r"(x), "r"(q));
}

__device__ __forceinline__ uint32_t magic_pair(uint32_t w) { return (w & 0x000F000Fu) | 0x43004300u; }

// Division of 32-bit unsigned values by an invariant divisor d (Granlund & Montgomery,
// "Division by invariant integers using multiplication", 1994): with l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (t + ((n - t) >> min(l,1))) >> max(l-1,0)
// where t = mulhi(m, n). Exact for every n < 2^32.
struct FastDiv {
    uint32_t d, m, s1, s2;
};

inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while (l < 32 && (1ull << l) < d) ++l;
    FastDiv f;
    f.d = d;
    f.m = (uint32_t)((((1ull << 32) * ((1ull << l) - d)) / d) + 1);
    f.s1 = l < 1 ? l : 1;
    f.s2 = l > 1 ? l - 1 : 0;
    return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f) {
    const uint32_t t = __umulhi(f.m, n);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

struct Args {
    const uint16_t *x;
    const uint8_t *codes;      // packed codes
    const uint8_t *scales;     // packed scales (u32 entries)
    void *y;
    float *ws_part;            // [P][2][8][MT] partials of boundary octets
    int *ws_count;             // [N8] arrival counters (zero between calls)
    int *status;
    int64_t N, K;
    uint32_t U, T;             // U = units per octet, T = total units (< 2^31)
    FastDiv divU;
    uint32_t base, rem, step;  // range of CTA c starts at c*base + min(c, rem)*step
    FastDiv divB1, divB;       // division by base + step and by base
    int M, g, out_fp32, nol, pdl;
    uint32_t sub;              // scale bytes per unit
    uint32_t off_sx, off_slot;
    uint32_t off_xf;           // M = 1 kernel: padded bf16 copy of x
    uint32_t off_ring, off_bars;  // M = 1 kernel: per-warp stage rings and their mbarriers
};

__device__ __forceinline__ uint32_t range_start(const Args &a, uint32_t c) {
    return c * a.base + (c < a.rem ? c : a.rem) * a.step;
}

__device__ __forceinline__ uint32_t cta_of_unit(const Args &a, uint32_t t) {
    const uint32_t big = (a.base + a.step) * a.rem;
    return t < big ? fdiv(t, a.divB1) : a.rem + fdiv(t - big, a.divB);
}

template <int MT, int W>
__device__ __forceinline__ void flush_octet(uint32_t ol, float (&y)[MT], float *slot, int warp, int lane) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        y[m] += __shfl_xor_sync(FULL, y[m], 1);
        y[m] += __shfl_xor_sync(FULL, y[m], 2);
    }
    if ((lane & 3) == 0) {
        float *d = slot + (ol * W + warp) * 8 * MT + (lane >> 2) * MT;
#pragma unroll
        for (int m = 0; m < MT; ++m) d[m] = y[m];
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) y[m] = 0.0f;
}

template <int MT> struct Warps { static constexpr int value = MT == 1 ? 32 : (MT <= 4 ? 16 : 8); };

__device__ __forceinline__ void store_y(const Args &a, int m, int64_t n, float v) {
    if (a.out_fp32) static_cast<float *>(a.y)[(int64_t)m * a.N + n] = v;
    else static_cast<__nv_bfloat16 *>(a.y)[(int64_t)m * a.N + n] = __float2bfloat16_rn(v);
}

// Per-octet reduction of the warps' partials (fixed warp order) and, for octets cut by a
// range boundary (stream-K partitions only), the cross-CTA fixup: the last CTA to arrive on
// the octet's counter adds all CTAs' partials in CTA order and resets the counter.
template <int MT, int W>
__device__ __forceinline__ void finish(const Args &a, const float *slot, int *flags, uint32_t c, uint32_t t0,
                                       uint32_t t1, uint32_t o_first, uint32_t o_last, int tid) {
    constexpr int THREADS = W * 32;
    const int M = a.M;
    const uint32_t Uc = a.U;
    const int nol = (int)(o_last - o_first + 1);
    for (int idx = tid; idx < nol * 8 * MT; idx += THREADS) {
        const int ol = idx / (8 * MT), rm = idx - ol * 8 * MT;
        const int rr = rm / MT, m = rm - rr * MT;
        float acc = 0.0f;
        for (int w = 0; w < W; ++w) acc += slot[(ol * W + w) * 8 * MT + rm];
        const uint32_t o = o_first + ol;
        const bool inside = o * Uc >= t0 && (o + 1) * Uc <= t1;
        if (inside) {
            const int64_t n = (int64_t)o * 8 + rr;
            if (m < M && n < a.N) store_y(a, m, n, acc);
        } else {
            const int which = (o == o_first) ? 0 : 1;
            a.ws_part[(((int64_t)c * 2 + which) * 8 + rr) * MT + m] = acc;
        }
    }
    // boundary octets (stream-K partitions only): the last CTA to arrive adds all partials
    // in CTA order and resets the counter
    const bool b0 = !(o_first * Uc >= t0 && (o_first + 1) * Uc <= t1);
    const bool b1 = (o_last != o_first) && !(o_last * Uc >= t0 && (o_last + 1) * Uc <= t1);
    if (!b0 && !b1) return;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        flags[1] = 0;
        flags[2] = 0;
        for (int which = 0; which < 2; ++which) {
            if (!(which == 0 ? b0 : b1)) continue;
            const uint32_t o = which == 0 ? o_first : o_last;
            const uint32_t cnt = cta_of_unit(a, (o + 1) * Uc - 1) - cta_of_unit(a, o * Uc) + 1;
            const int prev = atomicAdd(&a.ws_count[o], 1);
            flags[1 + which] = (prev == (int)cnt - 1) ? 1 : 0;
        }
        __threadfence();
    }
    __syncthreads();
    for (int which = 0; which < 2; ++which) {
        if (!flags[1 + which]) continue;
        const uint32_t o = which == 0 ? o_first : o_last;
        const uint32_t cf = cta_of_unit(a, o * Uc), cl = cta_of_unit(a, (o + 1) * Uc - 1);
        for (int rm = tid; rm < 8 * MT; rm += THREADS) {
            const int rr = rm / MT, m = rm - rr * MT;
            float acc = 0.0f;
            for (uint32_t k = cf; k <= cl; ++k) {
                const int wk = (fdiv(range_start(a, k), a.divU) == o) ? 0 : 1;
                acc += __ldcg(a.ws_part + (((int64_t)k * 2 + wk) * 8 + rr) * MT + m);
            }
            const int64_t n = (int64_t)o * 8 + rr;
            if (m < M && n < a.N) store_y(a, m, n, acc);
        }
        if (tid == 0) a.ws_count[o] = 0;
    }
}

template <int MT>
__global__ void __launch_bounds__(Warps<MT>::value * 32, 1) gemv_kernel(const Args a) {
    constexpr int W = Warps<MT>::value;
    constexpr int THREADS = W * 32;
    extern __shared__ __align__(16) uint8_t smem[];
    int *flags = reinterpret_cast<int *>(smem);   // [1..2] last-arriver flags
    float *sx = reinterpret_cast<float *>(smem + a.off_sx);
    float *slot = reinterpret_cast<float *>(smem + a.off_slot);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = lane >> 2, cc = lane & 3;
    const uint32_t c = blockIdx.x;
    const uint32_t t0 = range_start(a, c), t1 = range_start(a, c + 1);
    const uint32_t o_first = fdiv(t0, a.divU), o_last = fdiv(t1 - 1, a.divU);
    const int M = a.M;
    const uint32_t Kc = (uint32_t)a.K, Uc = a.U;
    const int nck = (int)(Uc * 4);  // 32-wide chunks per row (padded)

    // ---- the weight stream does not depend on earlier kernels: start it first
    const uint32_t tb = t0 + (uint32_t)warp;
    const int per_unit = 128 / a.g;
    const uint32_t sc_lane = (uint32_t)(r * per_unit + (cc * 32) / a.g) * 4;
    const uint8_t *cp = a.codes + (size_t)tb * 512 + lane * 16;
    const uint8_t *sp = a.scales + (size_t)tb * a.sub + sc_lane;
    const size_t cstep = (size_t)W * 512, sstep = (size_t)W * a.sub;
    uint4 qv[PF];
    uint32_t ev[PF];
#pragma unroll
    for (int i = 0; i < PF; ++i) {
        if (tb + (uint32_t)(i * W) < t1) {
            qv[i] = ldg_stream(cp + i * cstep);
            ev[i] = __ldg(reinterpret_cast<const uint32_t *>(sp + i * sstep));
        }
    }
    cp += PF * cstep;
    sp += PF * sstep;

    for (int i = tid; i < a.nol * W * 8 * MT; i += THREADS) slot[i] = 0.0f;
    // activations may be written by the previous kernel in the stream
    if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    // activation sums of every 32-wide chunk (chunks past K are zero)
    for (int idx = tid; idx < MT * nck; idx += THREADS) {
        const int m = idx / nck, ck = idx - m * nck;
        float s = 0.0f;
        if (m < M && (uint32_t)ck * 32 < Kc) {
            const uint4 *xv = reinterpret_cast<const uint4 *>(a.x + (int64_t)m * a.K + ck * 32);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint4 v = __ldg(xv + t);
                s = __fadd_rn(__fadd_rn(s, bf16_lo(v.x)), bf16_hi(v.x));
                s = __fadd_rn(__fadd_rn(s, bf16_lo(v.y)), bf16_hi(v.y));
                s = __fadd_rn(__fadd_rn(s, bf16_lo(v.z)), bf16_hi(v.z));
                s = __fadd_rn(__fadd_rn(s, bf16_lo(v.w)), bf16_hi(v.w));
            }
        }
        sx[idx] = s;
    }
    __syncthreads();
    if (a.pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    float y[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) y[m] = 0.0f;
    uint32_t cur_ol = 0xffffffffu;  // octet of the accumulated partial, relative to o_first
    for (uint32_t tq = tb; tq < t1; tq += (uint32_t)(PF * W)) {
#pragma unroll
        for (int i = 0; i < PF; ++i) {
            const uint32_t t = tq + (uint32_t)(i * W);
            if (t >= t1) break;
            const uint4 wq = qv[i];
            const uint32_t e = ev[i];
            if (t + (uint32_t)(PF * W) < t1) {
                qv[i] = ldg_stream(cp);
                ev[i] = __ldg(reinterpret_cast<const uint32_t *>(sp));
            }
            cp += cstep;
            sp += sstep;
            const uint32_t o = fdiv(t, a.divU);
            const uint32_t ol = o - o_first;
            if (ol != cur_ol) {
                if (cur_ol != 0xffffffffu) flush_octet<MT, W>(cur_ol, y, slot, warp, lane);
                cur_ol = ol;
            }
            const uint32_t k0 = (t - o * Uc) * 128u + (uint32_t)cc * 32u;
            if (k0 >= Kc) continue;
            const float scl = __half2float(__ushort_as_half((unsigned short)(e & 0xFFFF)));
            const float cz = (float)(int)(int16_t)(e >> 16) + 128.0f;
            uint32_t p[4][4];
            const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                p[q][0] = magic_pair(wv[q]);
                p[q][1] = magic_pair(wv[q] >> 4);
                p[q][2] = magic_pair(wv[q] >> 8);
                p[q][3] = magic_pair(wv[q] >> 12);
            }
            const uint32_t ck = k0 >> 5;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= M) break;
                float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
                const uint4 *xp = reinterpret_cast<const uint4 *>(a.x + (int64_t)m * a.K + k0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 xv = __ldg(xp + q);
                    fma2_bf16(a0, a1, xv.x, p[q][0]);
                    fma2_bf16(a2, a3, xv.y, p[q][1]);
                    fma2_bf16(a0, a1, xv.z, p[q][2]);
                    fma2_bf16(a2, a3, xv.w, p[q][3]);
                }
                y[m] = fmaf(scl, fmaf(-cz, sx[m * nck + ck], (a0 + a1) + (a2 + a3)), y[m]);
            }
        }
    }
    if (cur_ol != 0xffffffffu) flush_octet<MT, W>(cur_ol, y, slot, warp, lane);
    __syncthreads();

    finish<MT, W>(a, slot, flags, c, t0, t1, o_first, o_last, tid);
}

// ---------------------------------------------------------------- M = 1 kernel
//
// Each warp streams a contiguous run of 512-byte units through its own ring of shared-memory
// stages filled by 1-D bulk copies (one copy of codes and one of scales per stage of SU
// units, issued by the warp's lane 0, completion on an mbarrier), so loading costs almost no
// instructions; lanes read their 16 bytes of codes and their scale entry from shared memory.
// x is staged once per CTA as bf16 with 16 bytes of padding after every 32 values, so the
// four 32-wide chunks a warp reads at once start in different banks.
constexpr int W1 = 16;   // warps of the M = 1 kernel
constexpr int SU = 8;    // units per stage
constexpr int NS = 2;    // stages per warp

__device__ __forceinline__ uint32_t xb_index(uint32_t k) { return k + (k >> 5) * 8; }

// One unit for one lane: 16 bytes of codes (32 weights of row r, chunk at k0) against the
// padded bf16 x at xp, offset removed with the chunk sum sxc, times the group scale.
__device__ __forceinline__ void unit_m1(float &y, const uint4 wq, uint32_t e, const uint4 *xp, float sxc) {
    const float scl = __half2float(__ushort_as_half((unsigned short)(e & 0xFFFF)));
    const float cz = (float)(int)(int16_t)(e >> 16) + 128.0f;
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
    const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 xv = xp[q];
        fma2_bf16(a0, a1, xv.x, magic_pair(wv[q]));
        fma2_bf16(a2, a3, xv.y, magic_pair(wv[q] >> 4));
        fma2_bf16(a0, a1, xv.z, magic_pair(wv[q] >> 8));
        fma2_bf16(a2, a3, xv.w, magic_pair(wv[q] >> 12));
    }
    y = fmaf(scl, fmaf(-cz, sxc, (a0 + a1) + (a2 + a3)), y);
}

// shared-memory bytes of the M = 1 kernel's regions
inline uint32_t xb_bytes(uint32_t U) { return U * 4 * 40 * 2; }              // padded bf16 x
inline uint32_t ring_bytes(uint32_t sub) { return W1 * NS * SU * (512 + sub); }

__global__ void __launch_bounds__(W1 * 32, 1) gemv1_kernel(const Args a) {
    constexpr int W = W1, THREADS = W1 * 32;
    extern __shared__ __align__(16) uint8_t smem[];
    int *flags = reinterpret_cast<int *>(smem);
    float *sx = reinterpret_cast<float *>(smem + a.off_sx);
    uint16_t *xb = reinterpret_cast<uint16_t *>(smem + a.off_xf);
    float *slot = reinterpret_cast<float *>(smem + a.off_slot);
    uint8_t *ring = smem + a.off_ring;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + a.off_bars);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = lane >> 2, cc = lane & 3;
    const uint32_t c = blockIdx.x;
    const uint32_t t0 = range_start(a, c), t1 = range_start(a, c + 1);
    const uint32_t o_first = fdiv(t0, a.divU), o_last = fdiv(t1 - 1, a.divU);
    const uint32_t Kc = (uint32_t)a.K, Uc = a.U;
    const int nck = (int)(Uc * 4);
    const uint32_t sub = a.sub, stage_bytes = SU * (512 + sub);

    // this warp's contiguous run [wt0, wt1) of the CTA's units, cut into stages of at most SU
    // units that never cross an octet boundary (so a stage has one octet and one flush)
    const uint32_t n = t1 - t0;
    const uint32_t wt0 = t0 + (uint32_t)(((uint64_t)n * warp) / W);
    const uint32_t wt1 = t0 + (uint32_t)(((uint64_t)n * (warp + 1)) / W);
    uint8_t *wring = ring + (size_t)warp * NS * stage_bytes;
    uint64_t *wbar = bars + warp * NS;
    struct Cursor {
        uint32_t t, o, u;  // next unit, its octet and its position in the octet
    };
    auto stage_len = [&](const Cursor &q) {
        uint32_t cnt = wt1 - q.t;
        cnt = cnt < (uint32_t)SU ? cnt : (uint32_t)SU;
        return cnt < Uc - q.u ? cnt : Uc - q.u;
    };
    auto advance = [&](Cursor &q, uint32_t cnt) {
        q.t += cnt;
        q.u += cnt;
        if (q.u == Uc) { q.u = 0; ++q.o; }
    };
    Cursor cons;
    cons.t = wt0;
    cons.o = fdiv(wt0, a.divU);
    cons.u = wt0 - cons.o * Uc;
    Cursor prod = cons;
    uint32_t jp = 0;  // stages issued
    // lane 0 fills the producer cursor's next stage into ring slot jp % NS
    auto issue = [&]() {
        const uint32_t cnt = stage_len(prod);
        uint8_t *dst = wring + (jp % NS) * stage_bytes;
        uint64_t *bar = wbar + (jp % NS);
        mbar_arrive_expect_tx(bar, cnt * (512 + sub));
        bulk_g2s(dst, a.codes + (size_t)prod.t * 512, cnt * 512, bar);
        bulk_g2s(dst + SU * 512, a.scales + (size_t)prod.t * sub, cnt * sub, bar);
    };
    // ---- the weight stream does not depend on earlier kernels: start it first
    if (lane == 0) {
        for (int j = 0; j < NS; ++j) mbar_init(wbar + j, 1);
        fence_mbar_init();
    }
    for (int j = 0; j < NS && prod.t < wt1; ++j) {  // warp-uniform cursor, lane 0 issues
        if (lane == 0) issue();
        advance(prod, stage_len(prod));
        ++jp;
    }
    for (int i = tid; i < a.nol * W * 8; i += THREADS) slot[i] = 0.0f;
    // activations may be written by the previous kernel in the stream
    if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    // x as padded bf16 and the sum of every 32-wide chunk (chunks past K are zero)
    for (int ck = tid; ck < nck; ck += THREADS) {
        float s = 0.0f;
        const bool live = (uint32_t)ck * 32 < Kc;
        const uint4 *xv = reinterpret_cast<const uint4 *>(a.x + ck * 32);
        uint4 *dst = reinterpret_cast<uint4 *>(xb + xb_index((uint32_t)ck * 32));
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint4 u4 = live ? __ldg(xv + t) : make_uint4(0u, 0u, 0u, 0u);
            s = __fadd_rn(__fadd_rn(s, bf16_lo(u4.x)), bf16_hi(u4.x));
            s = __fadd_rn(__fadd_rn(s, bf16_lo(u4.y)), bf16_hi(u4.y));
            s = __fadd_rn(__fadd_rn(s, bf16_lo(u4.z)), bf16_hi(u4.z));
            s = __fadd_rn(__fadd_rn(s, bf16_lo(u4.w)), bf16_hi(u4.w));
            dst[t] = u4;
        }
        sx[ck] = s;
    }
    __syncthreads();
    if (a.pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int per_unit = 128 / a.g;
    const uint32_t sc_lane = (uint32_t)(r * per_unit + (cc * 32) / a.g);  // u32 index in a unit's scales
    float y[1] = {0.0f};
    uint32_t cur_ol = 0xffffffffu;
    const bool kpad = (Kc & 127u) != 0;
    bool ok = true;
    uint32_t j = 0;  // stages consumed
    for (; cons.t < wt1; ++j) {
        const uint32_t sl = j % NS;
        // lane 0 polls; every lane then takes the (now immediate) wait for its own acquire
        bool got = true;
        if (lane == 0) got = mbar_wait_bounded(wbar + sl, (j / NS) & 1u, a.status);
        got = __shfl_sync(FULL, got ? 1 : 0, 0) != 0;
        if (!got) { ok = false; break; }
        (void)mbar_try_wait(wbar + sl, (j / NS) & 1u);
        const uint32_t cnt = stage_len(cons);
        const uint32_t ol = cons.o - o_first;
        if (ol != cur_ol) {
            if (cur_ol != 0xffffffffu) flush_octet<1, W>(cur_ol, y, slot, warp, lane);
            cur_ol = ol;
        }
        const uint8_t *st = wring + sl * stage_bytes;
        const uint4 *cw = reinterpret_cast<const uint4 *>(st) + lane;
        const uint32_t *sw = reinterpret_cast<const uint32_t *>(st + SU * 512) + sc_lane;
        const uint32_t k0 = cons.u * 128u + (uint32_t)cc * 32u;
        const uint4 *xp = reinterpret_cast<const uint4 *>(xb + xb_index(k0));
        const float *sxp = sx + (k0 >> 5);
#pragma unroll
        for (int i = 0; i < SU; ++i)
            if ((uint32_t)i < cnt && (!kpad || k0 + (uint32_t)i * 128u < Kc))
                unit_m1(y[0], cw[i * 32], sw[i * (sub >> 2)], xp + i * 20, sxp[i * 4]);
        advance(cons, cnt);
        // every lane has read the slot: lane 0 refills it with the next stage
        __syncwarp();
        if (prod.t < wt1) {
            if (lane == 0) issue();
            advance(prod, stage_len(prod));
            ++jp;
        }
    }
    if (cur_ol != 0xffffffffu) flush_octet<1, W>(cur_ol, y, slot, warp, lane);
    // no bulk copy may still be in flight when the CTA exits: after a failed wait, wait
    // (bounded) for every stage this warp issued and did not consume
    if (!ok && lane == 0)
        for (uint32_t q = j; q < jp; ++q) (void)mbar_wait_bounded(wbar + q % NS, (q / NS) & 1u, a.status);
    __syncthreads();
    finish<1, W>(a, slot, flags, c, t0, t1, o_first, o_last, tid);
}

// ------------------------------------------------------------------ host side

struct Plan {
    Args a;
    int P, smem;
    bool aligned;  // whole octets per block
};

static int sm_count_cached() {
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return num_sms();
    if (!cache[dev]) cache[dev] = num_sms();
    return cache[dev];
}

// Work partition. With N8 octets of U units each and S SMs: if whole octets split evenly
// enough (fewer octets than SMs; the busiest SM at most ~8% above the mean; or its extra
// units cheaper than the cross-CTA fixup), every CTA gets whole octets and no partial sum
// crosses CTAs; otherwise the unit stream is split evenly (stream-K) and octets cut by a
// range boundary are finished through the workspace.
constexpr int SMEM_LIMIT_M1 = 227 * 1024;

// xf: plan for the M = 1 kernel (padded bf16 x, per-warp stage rings, W1 warps)
template <int MT>
static bool make_plan(Plan &p, int64_t M, int64_t N, int64_t K, int g, bool xf, int64_t S) {
    const int W = xf ? W1 : Warps<MT>::value;
    const size_t limit = xf ? (size_t)SMEM_LIMIT_M1 : (size_t)SMEM_LIMIT;
    const GemvLayout L = gemv_layout(N, K, g);
    Args &a = p.a;
    const int64_t T = L.N8 * L.U;
    if (T >= (1LL << 31)) return false;
    a.N = N; a.K = K; a.U = (uint32_t)L.U; a.T = (uint32_t)T;
    a.divU = make_fastdiv(a.U);
    a.M = (int)M; a.g = g;
    a.sub = (uint32_t)(8 * (128 / g) * 4);
    a.off_sx = 64;
    a.off_slot = a.off_sx + (uint32_t)(MT * L.U * 4 * 4);
    a.off_xf = a.off_ring = a.off_bars = 0;
    if (xf) {
        a.off_xf = a.off_slot;
        a.off_ring = a.off_xf + xb_bytes((uint32_t)L.U);
        a.off_bars = a.off_ring + ring_bytes(a.sub);
        a.off_slot = a.off_bars + W1 * NS * 8;
    }
    a.pdl = 0;
    int64_t P;
    bool aligned;
    if (L.N8 <= S) {
        P = L.N8;
        aligned = true;
    } else {
        // whole octets when the busiest CTA's extra units cost less than the cross-CTA
        // fixup of an even split (measured at about 3 us, the time of ~160 units at M = 1
        // and proportionally fewer for more rows), or when they are within 8% of the mean
        const int64_t per = (L.N8 + S - 1) / S;
        aligned = (double)per <= 1.08 * (double)L.N8 / (double)S ||
                  (double)(per * L.U) <= (double)T / (double)S + 160.0 / MT;
        P = aligned ? (L.N8 + per - 1) / per : (S < T ? S : T);
    }
    while (true) {
        if (aligned) {
            a.base = (uint32_t)((L.N8 / P) * L.U);
            a.rem = (uint32_t)(L.N8 % P);
            a.step = a.U;
        } else {
            a.base = (uint32_t)(T / P);
            a.rem = (uint32_t)(T % P);
            a.step = 1;
        }
        const int64_t maxr = (int64_t)a.base + (a.rem ? a.step : 0);
        const int64_t nol = (maxr + L.U - 1) / L.U + 1;
        const size_t smem = a.off_slot + (size_t)nol * W * 8 * MT * 4;
        if (smem <= limit) {
            a.nol = (int)nol;
            p.P = (int)P;
            p.smem = (int)smem;
            p.aligned = aligned;
            break;
        }
        if (P >= T) return false;
        aligned = false;
        P = P * 2 < T ? P * 2 : T;
    }
    a.divB1 = make_fastdiv(a.base + a.step);
    a.divB = make_fastdiv(a.base);
    return true;
}

// The plan a call of M rows will use: the M = 1 kernel's when it applies and its shared
// memory (which grows with K) fits, else the general kernel's.
template <int MT>
static bool plan_for(Plan &p, int64_t M, int64_t N, int64_t K, int g, bool &xf, int64_t S = 0) {
    if (S <= 0) S = sm_count_cached();
    xf = MT == 1;
    if (xf && make_plan<MT>(p, M, N, K, g, true, S)) return true;
    xf = false;
    return make_plan<MT>(p, M, N, K, g, false, S);
}

// Host-only view of a plan for `sms` SMs: out = {units, octets, blocks, whole octets (0/1),
// dynamic shared memory bytes per block, M = 1 ring kernel (0/1)}.
template <int MT>
static bool describe_plan(int64_t M, int64_t N, int64_t K, int g, int64_t sms, int64_t *out) {
    Plan p;
    bool xf;
    if (!plan_for<MT>(p, M, N, K, g, xf, sms)) return false;
    const GemvLayout L = gemv_layout(N, K, g);
    out[0] = (int64_t)p.a.T;
    out[1] = L.N8;
    out[2] = p.P;
    out[3] = p.aligned ? 1 : 0;
    out[4] = p.smem;
    out[5] = xf ? 1 : 0;
    return true;
}

template <int MT>
static size_t ws_need(int64_t N, int64_t K, int g) {
    Plan p;
    bool xf;
    if (!plan_for<MT>(p, MT, N, K, g, xf)) return 0;
    return (size_t)p.P * 2 * 8 * MT * 4;
}

template <int MT>
static w4_status run(const void *x, int64_t M, const void *packed, int64_t N, int64_t K, int g, void *y, int out_fp32,
                     void *ws, size_t ws_bytes, int pdl, cudaStream_t stream) {
    constexpr int W = Warps<MT>::value;
    Plan p;
    bool xf;
    if (!plan_for<MT>(p, M, N, K, g, xf)) return W4_ERR_SHAPE;
    const GemvLayout L = gemv_layout(N, K, g);
    const size_t need = (size_t)p.P * 2 * 8 * MT * 4 + (size_t)L.N8 * 4;
    if (!ws || ws_bytes < need) return W4_ERR_WORKSPACE;
    Args &a = p.a;
    a.x = static_cast<const uint16_t *>(x);
    a.codes = static_cast<const uint8_t *>(packed);
    a.scales = static_cast<const uint8_t *>(packed) + L.codes_bytes;
    a.y = y;
    a.out_fp32 = out_fp32;
    a.ws_part = static_cast<float *>(ws);
    a.ws_count = reinterpret_cast<int *>(static_cast<uint8_t *>(ws) + (size_t)p.P * 2 * 8 * MT * 4);
    a.status = device_status_ptr();
    a.pdl = pdl;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(gemv_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_LIMIT) !=
            cudaSuccess)
            return W4_ERR_CUDA;
        if (MT == 1 && cudaFuncSetAttribute(gemv1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            SMEM_LIMIT_M1) != cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.P);
    cfg.blockDim = dim3(xf ? W1 * 32 : W * 32);
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = xf ? cudaLaunchKernelEx(&cfg, gemv1_kernel, a) : cudaLaunchKernelEx(&cfg, gemv_kernel<MT>, a);
    if (e != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}

size_t workspace_bytes(int64_t N, int64_t K, int g) {
    const GemvLayout L = gemv_layout(N, K, g);
    size_t worst = 0;
    const size_t cand[5] = {ws_need<1>(N, K, g), ws_need<2>(N, K, g), ws_need<4>(N, K, g), ws_need<8>(N, K, g),
                            ws_need<16>(N, K, g)};
    for (size_t v : cand) worst = v > worst ? v : worst;
    return (worst + (size_t)L.N8 * 4 + 255) / 256 * 256;
}

}  // namespace gemv
}  // namespace w4

using namespace w4;

W4_API size_t w4a16_gemv_workspace_bytes(int64_t N, int64_t K, int group) {
    if (N < 1 || K < 32 || K % 32 != 0 || !valid_group(group) || K % group != 0) return 0;
    return gemv::workspace_bytes(N, K, group);
}

W4_API w4_status w4a16_gemv_schedule(int64_t M, int64_t N, int64_t K, int group, int sms, int64_t *out) {
    if (!out) return W4_ERR_NULL;
    if (M < 1 || M > 16 || N < 1 || N > (int64_t)0x7fffffff * 8 || K < 32 || K % 32 != 0 || sms < 1 || sms > 4096)
        return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    bool ok;
    if (M <= 1) ok = gemv::describe_plan<1>(M, N, K, group, sms, out);
    else if (M <= 2) ok = gemv::describe_plan<2>(M, N, K, group, sms, out);
    else if (M <= 4) ok = gemv::describe_plan<4>(M, N, K, group, sms, out);
    else if (M <= 8) ok = gemv::describe_plan<8>(M, N, K, group, sms, out);
    else ok = gemv::describe_plan<16>(M, N, K, group, sms, out);
    return ok ? W4_OK : W4_ERR_SHAPE;
}

W4_API w4_status w4a16_gemv(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K, int group,
                            int mode, void *y, int flags, void *workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
    if (!x_bf16 || !packed || !y) return W4_ERR_NULL;
    if (!valid_mode(mode) || (flags & ~(W4_OUT_FP32 | W4_OVERLAP_PREVIOUS))) return W4_ERR_ARG;
    const int out_fp32 = (flags & W4_OUT_FP32) ? 1 : 0;
    const int pdl = (flags & W4_OVERLAP_PREVIOUS) ? 1 : 0;
    if (M < 1 || M > 16 || N < 1 || N > (int64_t)0x7fffffff * 8 || K < 32 || K % 32 != 0) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(y) || (workspace && !aligned16(workspace)))
        return W4_ERR_ALIGN;
    if (M <= 1) return gemv::run<1>(x_bf16, M, packed, N, K, group, y, out_fp32, workspace, workspace_bytes, pdl, stream);
    if (M <= 2) return gemv::run<2>(x_bf16, M, packed, N, K, group, y, out_fp32, workspace, workspace_bytes, pdl, stream);
    if (M <= 4) return gemv::run<4>(x_bf16, M, packed, N, K, group, y, out_fp32, workspace, workspace_bytes, pdl, stream);
    if (M <= 8) return gemv::run<8>(x_bf16, M, packed, N, K, group, y, out_fp32, workspace, workspace_bytes, pdl, stream);
    return gemv::run<16>(x_bf16, M, packed, N, K, group, y, out_fp32, workspace, workspace_bytes, pdl, stream);
}

// ------------------------------------------------------------------ allocation-free variant
//
// Callers that must not allocate device memory on the hot path -- a plug-in running inside
// another runtime that owns all device memory, or a latency-critical decode loop where
// cudaMalloc's implicit device synchronisation is not acceptable -- can call
// w4a16_gemv_noalloc. Its scratch (the partial sums and arrival counters of the stream-K
// fixup) is a fixed array in this library's device memory, reserved when the library loads
// on a GPU and held until the process exits.

namespace w4 {
namespace gemv {

constexpr size_t kNoAllocScratchBytes = (size_t)1 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void *g_noalloc_ptr[64];

// Device address of the scratch array on the current device. Host code must not use the
// symbol itself (that is a host-side stand-in, not a device address); the address is looked
// up once per device, with that device current.
static void *noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}

template <int MT>
static w4_status run_noalloc(const void *x, int64_t M, const void *packed, int64_t N, int64_t K, int g, void *y,
                             int out_fp32, int pdl, cudaStream_t stream) {
    Plan p;
    bool xf;
    if (!plan_for<MT>(p, M, N, K, g, xf)) return W4_ERR_SHAPE;
    const GemvLayout L = gemv_layout(N, K, g);
    const size_t part = (size_t)p.P * 2 * 8 * MT * 4;
    const size_t need = part + (size_t)L.N8 * 4;
    if (need > kNoAllocScratchBytes) return W4_ERR_SCRATCH_LIMIT;
    uint8_t *ws = static_cast<uint8_t *>(noalloc_scratch());
    if (!ws) return W4_ERR_CUDA;
    // the arrival counters must start at zero; a call normally leaves them at zero, but the
    // array outlives every call, so clear them on the caller's stream first
    if (cudaMemsetAsync(ws + part, 0, (size_t)L.N8 * 4, stream) != cudaSuccess) return W4_ERR_CUDA;
    return run<MT>(x, M, packed, N, K, g, y, out_fp32, ws, kNoAllocScratchBytes, pdl, stream);
}

}  // namespace gemv
}  // namespace w4

W4_API size_t w4a16_gemv_noalloc_scratch_limit(void) { return w4::gemv::kNoAllocScratchBytes; }

W4_API w4_status w4a16_gemv_noalloc(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K,
                                    int group, int mode, void *y, int flags, cudaStream_t stream) {
    if (!x_bf16 || !packed || !y) return W4_ERR_NULL;
    if (!valid_mode(mode) || (flags & ~(W4_OUT_FP32 | W4_OVERLAP_PREVIOUS))) return W4_ERR_ARG;
    if (M < 1 || M > 16 || N < 1 || N > (int64_t)0x7fffffff * 8 || K < 32 || K % 32 != 0) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(y)) return W4_ERR_ALIGN;
    const int out_fp32 = (flags & W4_OUT_FP32) ? 1 : 0;
    const int pdl = (flags & W4_OVERLAP_PREVIOUS) ? 1 : 0;
    if (M <= 1) return gemv::run_noalloc<1>(x_bf16, M, packed, N, K, group, y, out_fp32, pdl, stream);
    if (M <= 2) return gemv::run_noalloc<2>(x_bf16, M, packed, N, K, group, y, out_fp32, pdl, stream);
    if (M <= 4) return gemv::run_noalloc<4>(x_bf16, M, packed, N, K, group, y, out_fp32, pdl, stream);
    if (M <= 8) return gemv::run_noalloc<8>(x_bf16, M, packed, N, K, group, y, out_fp32, pdl, stream);
    return gemv::run_noalloc<16>(x_bf16, M, packed, N, K, group, y, out_fp32, pdl, stream);
}
