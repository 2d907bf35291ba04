// w4a16_gemv: weight-only INT4 GEMV for decode, dequantization fused into the product.
//
// "Quantizing LLMs Without Guesswork", The Problem & Context (decode reads every weight
// once and that read sets the pace) and Weight-only methods (4-bit weights, 16-bit
// activations, dequantized inside the matmul).
//
//   y[m, n] = sum_j s[n,j] * sum_{k in j} x[m,k] * (q[n,k] - z[n,j])
//
// A streaming kernel on the CUDA cores, layout W4_LAYOUT_GEMV (one record of codes and
// scales per weight row, see w4_layout.cuh).
//
// Integer dot products. The codes are 4-bit integers, so the inner product runs on the
// integer dot-product unit (dp4a: four 8-bit products and a 32-bit sum per instruction, on
// a different pipe from the bit operations that unpack the codes). Each thread owns a slice
// of KC = 128/MT consecutive k and keeps the activations of that slice in registers as
// 24-bit fixed point with one exponent per slice: X[k] = rint(x[k] * 2^S), |X| < 2^19, with
// S chosen from the slice's largest |x| (exact for every x within 2^11 of that maximum;
// smaller ones are rounded to 2^-S, i.e. 2^-19 of the maximum). Three byte planes of 16X
// (even k) and of X (odd k) meet the code bytes w & 0x0F0F0F0F (q of the even k) and
// w & 0xF0F0F0F0 (16 q of the odd k), so six dp4a per 8 weights give the exact integer
// D = 16 * sum X q; per group segment the planes' sums are combined in fp32:
//   sum x (q - z) = 2^-S (D / 16 - z sum X),  partial += s * that.
// Every integer sum is exact; the fp32 roundings are those of the per-segment combine and
// of the row sum, so the result is within a few fp32 roundings of the exact product of the
// fixed-point activations.
//
// Data movement. One persistent block per SM owns a contiguous run of rows. A producer warp
// streams the block's rows through a ring of shared-memory stages with 1-D bulk copies
// (consecutive rows are consecutive records: a stage is one range, copied in 4 KB pieces), so
// the whole ring (~150 KB per SM) is in flight from the first instruction. The activations are converted
// to byte planes once per block (all threads cooperate, each element once) into an area at
// the end of the ring that the producer fills only after every thread has loaded its planes
// into registers. A stage holds one row per "slot" of threads; each thread adds its
// slice's partial for that row and stores it in shared memory; after the last stage the
// row sums are formed in a fixed order (bit-identical results run to run).
//
// Rows longer than a block's threads can cover (K > 448 KC) are split along K over several
// blocks; their partial sums go through the caller's workspace and the last block of a row
// range to arrive adds them in a fixed order. M > MT activation rows run as ceil(M/MT)
// sweeps over the weights (the launch's second grid dimension).
#include "w4_common.cuh"
#include "w4_layout.cuh"

#include <mutex>

namespace w4 {
namespace gemv {

constexpr int NCW = 14;                 // consumer warps
constexpr int NCT = NCW * 32;           // consumer threads
constexpr int THREADS = NCT + 32;       // + one producer warp
constexpr int SMEM_MAX = 227 * 1024;
constexpr int RED_BUDGET = 48 * 1024;   // row-partial buffer
constexpr int MAX_STAGES = 16;
constexpr uint32_t SLACK = 64;          // bytes after the ring (reads past a short last slice)
constexpr uint64_t PF_PIECE = 32 * 1024; // bytes per L2 prefetch instruction
constexpr uint32_t STREAM_PIECE = 4096;  // bytes per bulk copy of the weight stream (a multiple of 16)

struct Args {
    const uint16_t *x;   // [M, K] bf16
    const uint8_t *w;    // packed row records
    void *y;             // [M, N]
    float *ws_part;      // [kparts][M][N] partial sums (K split only)
    int *ws_count;       // [sweeps][nrb] arrival counters (K split only; zero between calls)
    int *status;
    int64_t N, K;
    int M, J, g;
    uint32_t RS;         // row record bytes
    uint32_t RSp;        // bytes of one row in a stage
    uint32_t KPB;        // code bytes of one row in a stage (the scales follow)
    int tpr;             // slices of the whole row
    int spp;             // slices per K part (threads per row)
    int kparts;
    int nslot;           // thread slots (each takes rpt rows of a stage)
    int rpt;             // rows per thread and stage
    int rpc;             // rows per block (last block may have fewer)
    int nrb;             // row blocks
    int NS, NS_early;    // ring stages; stages issued before the planes are loaded
    uint32_t SB;         // stage bytes
    uint32_t off_sx, off_pp, off_red, off_ring, off_planes;
    int warpred;         // MT > 1 with spp a multiple of 32: partials reduced over the warp first
    int direct;          // MT = 1, one warp per row (spp = 32, whole rows, one stage per block):
                         // the warp adds the row's partials and its lane 0 stores y
    int nred;            // partials per (row, m): spp, or spp / 32 with warpred
    int rstr;            // words between the partials of consecutive (row, m) (nred, padded)
    int lpr;             // lanes that add one (row, m)'s partials in the final reduction
    int out_fp32, pdl;
    const uint8_t *pf;   // bytes to bring into L2 once the block's own stream is issued (or null)
    uint64_t pf_bytes;   // their count (a multiple of 16)
    uint64_t pf_chunk;   // per block (a multiple of 16)
};

__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int32_t dp4a_su(uint32_t a, uint32_t b, int32_t c) {
    int32_t d;
    asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// two fp32 lanes per instruction (sm_100): lane 0 in the low word
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t pair(uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; }

// 2^e as an fp32 (0 below the subnormal range); e <= 127
__device__ __forceinline__ float exp2i(int e) {
    if (e >= -126) return __int_as_float((e + 127) << 23);
    if (e >= -149) return __int_as_float(1 << (e + 149));
    return 0.0f;
}

// Sum of v[m] over the warp for MT values at once: after the exchange at distance 16 (MT >= 2)
// and 8 (MT = 4) each lane keeps the partial sums of one m, then a butterfly over the
// remaining distances; lane l ends with the sum for m = l / (32 / MT). Fixed order.
template <int MT>
__device__ __forceinline__ float warp_transpose_sum(const float (&v)[MT], int lane) {
    float r;
    if constexpr (MT == 1) {
        r = v[0];
    } else if constexpr (MT == 2) {
        const bool b4 = lane & 16;
        r = (b4 ? v[1] : v[0]) + __shfl_xor_sync(FULL, b4 ? v[0] : v[1], 16);
    } else {
        const bool b4 = lane & 16, b3 = lane & 8;
        const float k0 = (b4 ? v[2] : v[0]) + __shfl_xor_sync(FULL, b4 ? v[0] : v[2], 16);
        const float k1 = (b4 ? v[3] : v[1]) + __shfl_xor_sync(FULL, b4 ? v[1] : v[3], 16);
        r = (b3 ? k1 : k0) + __shfl_xor_sync(FULL, b3 ? k0 : k1, 8);
    }
#pragma unroll
    for (int off = 32 / MT / 2; off >= 1; off >>= 1) r += __shfl_xor_sync(FULL, r, off);
    return r;
}

// Geometry shared by host and device for a slice width KC.
template <int MT> struct Geo {
    static constexpr int KC = 128 / MT;       // k per slice
    static constexpr int NCH = KC / 32;       // 16-byte code chunks per slice
    static constexpr int WPS = KC / 8;        // code words per slice
    static constexpr int PW = 6 * WPS;        // plane words per slice and activation row
    // A slice's planes are stored load-major: the 16-byte load q (q = 0..5) of chunk c sits at
    // word 4 (q NCH + c), so the loads a thread issues for its chunks in rotated order, with
    // slices PSTRIDE words apart, fall in distinct banks for every 8 lanes when PSTRIDE / 4 is
    // congruent to NCH modulo 8 (lanes 2r, 2r+1 share the rotation r when NCH = 4, lanes
    // 4r..4r+3 when NCH = 2). With one chunk any odd PSTRIDE / 4 does.
    static constexpr int PSTRIDE = NCH == 1 ? PW + 4 : PW + ((4 * NCH - PW % 32) % 32 + 32) % 32;
    static constexpr int RPT = MT == 1 ? 2 : 1;  // rows per thread and stage (registers allow two at MT = 1)
};

// Byte planes of activation row m0 + m for the tasks t0 + r NCT (r < XBN) of this thread (one
// task = 8 consecutive k of a slice; a slice's WPS tasks are consecutive lanes). X = rint(x 2^S)
// with S from the slice's largest |x| (|X| < 2^19); planes: even k as 16 X, odd k as X, byte p
// of each in 4-byte words, stored load-major (see Geo); per chunk the sum of X, per slice 2^-S.
template <int MT, int XBN>
__device__ __forceinline__ void xprep_rounds(const Args &a, uint32_t *planes, int *sx, float *pp, int m, int m0,
                                             int64_t k0, int nsl, int t0) {
    using GE_ = Geo<MT>;
    constexpr int KC = GE_::KC, NCH = GE_::NCH, WPS = GE_::WPS, PSTRIDE = GE_::PSTRIDE;
    const int tasks = a.spp * WPS;
    uint4 xv[XBN];
#pragma unroll
    for (int r = 0; r < XBN; ++r) {
        const int t = t0 + r * NCT;
        const int tsl = t / WPS, wi = t - tsl * WPS;
        const int64_t k = k0 + (int64_t)tsl * KC + wi * 8;
        const bool live = t < tasks && tsl < nsl && m0 + m < a.M && k < a.K;
        xv[r] = live ? __ldg(reinterpret_cast<const uint4 *>(a.x + (int64_t)(m0 + m) * a.K + k))
                     : make_uint4(0u, 0u, 0u, 0u);
    }
    // largest magnitude pattern of each slice (bf16 bits order like magnitudes): a 16-bit
    // SIMD max over the magnitude bits of both halves, then the larger half
    uint32_t mx[XBN];
#pragma unroll
    for (int r = 0; r < XBN; ++r) {
        const uint32_t m2 = __vmaxu2(__vmaxu2(xv[r].x & 0x7FFF7FFFu, xv[r].y & 0x7FFF7FFFu),
                                     __vmaxu2(xv[r].z & 0x7FFF7FFFu, xv[r].w & 0x7FFF7FFFu));
        mx[r] = max(m2 & 0xFFFFu, m2 >> 16);
    }
#pragma unroll
    for (int off = WPS / 2; off >= 1; off >>= 1)
#pragma unroll
        for (int r = 0; r < XBN; ++r) mx[r] = max(mx[r], __shfl_xor_sync(FULL, mx[r], off));
    int xs[XBN];
#pragma unroll
    for (int r = 0; r < XBN; ++r) {
        const uint32_t e[4] = {xv[r].x, xv[r].y, xv[r].z, xv[r].w};
        // exponent of the largest |x|: |x| in [2^ex, 2^(ex+1)); every step below is a select,
        // not a branch, so that the rounds of a thread interleave
        const int ex = mx[r] >= 0x80u ? (int)(mx[r] >> 7) - 127 : (31 - __clz((int)(mx[r] | 1u))) - 133;
        const int S = 18 - ex;  // -109 <= S <= 151
        // x 2^S as two exact power-of-two products (2^S alone leaves the fp32 range when the
        // slice's largest |x| is below 2^-109): 2^min(S, 127), then 2^max(S - 127, 0)
        const uint32_t f1 = (uint32_t)((S < 127 ? S : 127) + 127) << 23;
        const uint32_t f2 = (uint32_t)((S > 127 ? S - 127 : 0) + 127) << 23;
        // rint by the 1.5 * 2^23 shift, two elements per instruction. A slice of zeros gives
        // X = 0; in a slice holding an infinity or a NaN the values are meaningless, and its
        // 2^-S below is a NaN, which makes the rows' sums NaN
        const uint64_t F1 = pair(f1, f1), F2 = pair(f2, f2), RND = pair(0x4B400000u, 0x4B400000u);
        int X[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const uint64_t v = add_f32x2(mul_f32x2(mul_f32x2(pair(e[h] << 16, e[h] & 0xFFFF0000u), F1), F2), RND);
            X[2 * h] = (int)(uint32_t)v - 0x4B400000;
            X[2 * h + 1] = (int)(uint32_t)(v >> 32) - 0x4B400000;
        }
        uint32_t pw[6];
#pragma unroll
        for (int par = 0; par < 2; ++par) {
            const uint32_t sh = par ? 0u : 4u;
            const uint32_t V0 = (uint32_t)X[par] << sh, V1 = (uint32_t)X[2 + par] << sh;
            const uint32_t V2 = (uint32_t)X[4 + par] << sh, V3 = (uint32_t)X[6 + par] << sh;
            // plane pl = byte pl of V0..V3: pairs of bytes first, then the planes
            const uint32_t t01l = __byte_perm(V0, V1, 0x5140u), t01h = __byte_perm(V0, V1, 0x0062u);
            const uint32_t t23l = __byte_perm(V2, V3, 0x5140u), t23h = __byte_perm(V2, V3, 0x0062u);
            pw[par * 3 + 0] = __byte_perm(t01l, t23l, 0x5410u);
            pw[par * 3 + 1] = __byte_perm(t01l, t23l, 0x7632u);
            pw[par * 3 + 2] = __byte_perm(t01h, t23h, 0x5410u);
        }
        xs[r] = X[0] + X[1] + X[2] + X[3] + X[4] + X[5] + X[6] + X[7];
        const int t = t0 + r * NCT;
        const int tsl = t / WPS, wi = t - tsl * WPS;
        if (t < tasks) {
            // word u = 6 (wi % 4) + i of chunk wi / 4 goes to load u / 4, lane u % 4
            uint32_t *dst = planes + tsl * PSTRIDE + (wi >> 2) * 4;
#pragma unroll
            for (int h = 0; h < 3; ++h) {
                const int u = (wi & 3) * 6 + 2 * h;
                *reinterpret_cast<uint2 *>(dst + (u >> 2) * 4 * NCH + (u & 3)) = make_uint2(pw[2 * h], pw[2 * h + 1]);
            }
            // 2^-S: normal for S <= 126, subnormal up to S = 149 (0 beyond)
            const float p2 = S <= 126 ? __int_as_float((127 - S) << 23) : (S <= 149 ? __int_as_float(1 << (149 - S)) : 0.0f);
            if (wi == 0)
                pp[m * a.spp + tsl] = (mx[r] >= 0x7F80u) ? __int_as_float(0x7FC00000) : (mx[r] == 0u ? 0.0f : p2);
        }
    }
    // sums of X per chunk of 32 k (4 tasks)
#pragma unroll
    for (int r = 0; r < XBN; ++r) xs[r] += __shfl_xor_sync(FULL, xs[r], 1);
#pragma unroll
    for (int r = 0; r < XBN; ++r) xs[r] += __shfl_xor_sync(FULL, xs[r], 2);
#pragma unroll
    for (int r = 0; r < XBN; ++r) {
        const int t = t0 + r * NCT;
        const int tsl = t / WPS, wi = t - tsl * WPS;
        if (t < tasks && (wi & 3) == 0) sx[(m * a.spp + tsl) * NCH + (wi >> 2)] = xs[r];
    }
}

// The work of one block: row block bx (and K part), activation rows by * MT ... of the
// problem a.
template <int MT, int G>
__device__ __forceinline__ void gemv_block(const Args &a, const int bx, const int by) {
    using GE_ = Geo<MT>;
    constexpr int KC = GE_::KC, NCH = GE_::NCH, WPS = GE_::WPS, PSTRIDE = GE_::PSTRIDE;
    constexpr int GS = G < KC ? G : KC;       // k per combine segment
    constexpr int NSEG = KC / GS;             // segments per slice
    constexpr int CPS = GS / 32;              // chunks per segment
    constexpr int RPT = GE_::RPT;             // rows per thread and stage
    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + MAX_STAGES;
    uint64_t *planes_done = empty + MAX_STAGES;
    int *abort_flag = reinterpret_cast<int *>(planes_done + 1);
    int *last_flag = abort_flag + 1;
    int *sx = reinterpret_cast<int *>(smem + a.off_sx);          // [MT][spp][NCH] sums of X per chunk
    float *pp = reinterpret_cast<float *>(smem + a.off_pp);      // [MT][spp] 2^-S per slice
    float *red = reinterpret_cast<float *>(smem + a.off_red);    // [rpc][MT][spp] row partials
    const uint32_t ring = smem_addr(smem + a.off_ring);
    uint32_t *planes = reinterpret_cast<uint32_t *>(smem + a.off_planes);  // [spp][PSTRIDE], one row m at a time

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kp = (int)((unsigned)bx % (unsigned)a.kparts);
    const int rb = (int)((unsigned)bx / (unsigned)a.kparts);
    const int m0 = by * MT;
    const int64_t row0 = (int64_t)rb * a.rpc;
    const int rows = (int)((a.N - row0) < a.rpc ? (a.N - row0) : a.rpc);
    const int nstages = (rows + a.nslot * a.rpt - 1) / (a.nslot * a.rpt);
    const int sl0 = kp * a.spp;                                    // first slice of this part
    const int nsl = (a.tpr - sl0) < a.spp ? (a.tpr - sl0) : a.spp;  // slices of this part
    const int64_t k0 = (int64_t)sl0 * KC;                          // first k of this part
    const int gsh = __ffs(a.g) - 1;                                // log2 of the group (a power of two)
    const int J0 = (int)(k0 >> gsh);                               // first group of this part

    if (tid == 0) {
        for (int i = 0; i < a.NS; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, NCW);
        }
        mbar_init(planes_done, NCW);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == NCW) {
        // ------------------------------------------------ producer: stream the rows
        if (a.pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        if (lane == 0) {
            const uint8_t *src0 = a.w + (size_t)row0 * a.RS;
            int issued = 0;
            bool ok = true;
            for (int s = 0; s < nstages && ok; ++s) {
                const int slot = s % a.NS;
                if (s >= a.NS) {
                    ok = mbar_wait_abortable(empty + slot, ((s / a.NS) - 1) & 1, abort_flag, a.status, 2000000000ull);
                } else if (s == a.NS_early) {
                    ok = mbar_wait_abortable(planes_done, 0, abort_flag, a.status, 2000000000ull);
                }
                if (!ok) break;
                const int r0 = s * a.nslot * a.rpt;
                const int nr = (rows - r0) < a.nslot * a.rpt ? (rows - r0) : a.nslot * a.rpt;
                uint8_t *dst = smem + a.off_ring + (size_t)slot * a.SB;
                if (a.kparts == 1) {
                    // the stage's rows are consecutive records: copied in pieces of STREAM_PIECE
                    // bytes, so that the activation loads the consumers issue meanwhile are not
                    // queued behind one long copy in the SM's inbound traffic
                    const uint32_t tot = (uint32_t)nr * a.RS;
                    mbar_arrive_expect_tx(full + slot, tot);
                    for (uint32_t o = 0; o < tot; o += STREAM_PIECE) {
                        const uint32_t n = tot - o < STREAM_PIECE ? tot - o : STREAM_PIECE;
                        bulk_g2s_stream(dst + o, src0 + (size_t)r0 * a.RS + o, n, full + slot);
                    }
                } else {
                    // this part's codes and scales of each row
                    const uint32_t cb = (uint32_t)(((k0 + (int64_t)nsl * KC < a.K ? k0 + (int64_t)nsl * KC : a.K) - k0) / 2);
                    const uint32_t scb0 = (uint32_t)(a.K / 2) + 4u * (uint32_t)J0;
                    const uint32_t scb = (kp == a.kparts - 1) ? a.RS - scb0 : 4u * (uint32_t)(nsl * KC / a.g);
                    mbar_arrive_expect_tx(full + slot, (uint32_t)nr * (cb + scb));
                    for (int r = 0; r < nr; ++r) {
                        const uint8_t *rs = src0 + (size_t)(r0 + r) * a.RS;
                        bulk_g2s_stream(dst + (size_t)r * a.RSp, rs + k0 / 2, cb, full + slot);
                        bulk_g2s_stream(dst + (size_t)r * a.RSp + a.KPB, rs + scb0, scb, full + slot);
                    }
                }
                ++issued;
            }
            // the next GEMV's weights: once this block's rows are all requested, its share of
            // them goes into L2, so that HBM reads them while this launch converts, sums and
            // exits and the next launch finds them there
            if (a.pf && ok) {
                const uint64_t lb = (uint64_t)by * gridDim.x + (uint64_t)bx;
                const uint64_t b0 = lb * a.pf_chunk;
                const uint64_t b1 = b0 + a.pf_chunk < a.pf_bytes ? b0 + a.pf_chunk : a.pf_bytes;
                for (uint64_t o = b0; o < b1; o += PF_PIECE) {
                    const uint64_t n = b1 - o < PF_PIECE ? b1 - o : PF_PIECE;
                    bulk_prefetch_l2(a.pf + o, (uint32_t)n);
                }
            }
            // no bulk copy may be in flight when the block exits
            for (int s = issued - a.NS > 0 ? issued - a.NS : 0; s < issued; ++s)
                (void)mbar_wait_bounded(full + (s % a.NS), (s / a.NS) & 1, a.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ consumers
        // activations may be written by the previous kernel in the stream
        if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");

        // this thread's slice; its chunks are visited in an order rotated per lane so that
        // the 16-byte code loads of a warp hit distinct banks (planes are loaded in that order)
        const int slot = tid / a.spp, sl = tid - slot * a.spp;
        const bool active = slot < a.nslot && sl < nsl;
        constexpr int ROT_DIV = 8 / NCH;          // lanes sharing a rotation
        const int rraw = (lane / ROT_DIV) % NCH;
        const int rot = NSEG == 1 ? rraw : rraw / CPS * CPS;   // segments keep their chunks together
        const int srot = NSEG == 1 ? 0 : rot / CPS;          // rotation in segments
        uint32_t xp[MT][NCH][4][6];
        float q16[MT], q16x256[MT], q16x65536[MT], sxf[MT][NSEG];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            // (1) byte planes of activation row m0 + m, one task per 8 consecutive k; a thread
            // takes up to 4 rounds of tasks at once, every step done for all its rounds together
            // so that the rounds' latencies (loads, shuffle chains) overlap
            const int tasks = a.spp * WPS;
            for (int tb = 0; tb < tasks; tb += 4 * NCT) {
                // rounds in which this warp has a task (warp-uniform; a warp with none skips)
                const int nr = (tasks - tb - warp * 32 + NCT - 1) / NCT;
                if (nr <= 0) continue;
                if (nr >= 4) xprep_rounds<MT, 4>(a, planes, sx, pp, m, m0, k0, nsl, tb + warp * 32 + lane);
                else if (nr == 3) xprep_rounds<MT, 3>(a, planes, sx, pp, m, m0, k0, nsl, tb + warp * 32 + lane);
                else if (nr == 2) xprep_rounds<MT, 2>(a, planes, sx, pp, m, m0, k0, nsl, tb + warp * 32 + lane);
                else xprep_rounds<MT, 1>(a, planes, sx, pp, m, m0, k0, nsl, tb + warp * 32 + lane);
            }
            named_bar_sync(1, NCT);
            // (2) this thread's planes of row m into registers
            const uint32_t pb = smem_addr(planes + (active ? sl : 0) * PSTRIDE);
#pragma unroll
            for (int j = 0; j < NCH; ++j) {
                const int c = (j + rot) % NCH;
#pragma unroll
                for (int q = 0; q < 6; ++q) {  // 24 words of chunk c: 6 loads of 4
                    const uint4 v = lds128(pb + (uint32_t)(q * 4 * NCH + c * 4) * 4u);
                    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int r = 0; r < 4; ++r) xp[m][j][(q * 4 + r) / 6][(q * 4 + r) % 6] = vv[r];
                }
            }
            const float p = active ? pp[m * a.spp + sl] : 0.0f;
            q16[m] = __fmul_rn(p, 0.0625f);
            q16x256[m] = __fmul_rn(p, 16.0f);
            q16x65536[m] = __fmul_rn(p, 4096.0f);
#pragma unroll
            for (int js = 0; js < NSEG; ++js) {
                const int seg = (js + srot) % NSEG;
                int sum = 0;
#pragma unroll
                for (int c = 0; c < CPS; ++c) sum += active ? sx[(m * a.spp + sl) * NCH + seg * CPS + c] : 0;
                sxf[m][js] = __fmul_rn((float)sum, p);
            }
            if (m + 1 < MT) named_bar_sync(1, NCT);  // the next row's tasks overwrite the planes
        }
        if (a.pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(planes_done);

        // (3) the rows: RPT per thread and stage (rows slot, slot + nslot, ... of the stage)
        const uint32_t code_off = (uint32_t)sl * (KC / 2);
        uint32_t sc_off[NSEG];  // byte offset of each segment's scale word in a row
        bool seg_live[NSEG];
#pragma unroll
        for (int js = 0; js < NSEG; ++js) {
            const int seg = (js + srot) % NSEG;
            const int jg = (int)((k0 + (int64_t)sl * KC + seg * GS) >> gsh);
            seg_live[js] = jg < a.J;
            sc_off[js] = a.KPB + 4u * (uint32_t)(jg - J0);
        }
        const int SR = a.nslot * RPT;  // rows per stage
        bool ok = true;
        for (int s = 0; s < nstages; ++s) {
            const int slot_s = s % a.NS;
            bool got = true;
            if (lane == 0) got = mbar_wait_abortable(full + slot_s, (s / a.NS) & 1, abort_flag, a.status, 2000000000ull);
            got = __shfl_sync(FULL, got ? 1 : 0, 0) != 0;
            if (!got) { ok = false; break; }
            // lane 0's wait acquired the stage's bytes; the warp barrier orders the other lanes'
            // reads after it (a try_wait by every lane of every warp costs the barrier unit
            // hundreds of cycles a stage)
            __syncwarp();
            const uint32_t sbase = ring + (uint32_t)slot_s * a.SB;
            float yv[RPT][MT];
            bool live[RPT];
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                live[i] = active && s * SR + slot + i * a.nslot < rows;
#pragma unroll
                for (int m = 0; m < MT; ++m) yv[i][m] = 0.0f;
            }
            if (live[0]) {
                uint32_t rbase[RPT];
#pragma unroll
                for (int i = 0; i < RPT; ++i) rbase[i] = sbase + (uint32_t)(slot + i * a.nslot) * a.RSp;
#pragma unroll
                for (int js = 0; js < NSEG; ++js) {
                    // independent accumulators per row and plane
                    uint32_t A0[RPT][MT], A1[RPT][MT];
                    int32_t A2[RPT][MT];
#pragma unroll
                    for (int i = 0; i < RPT; ++i)
#pragma unroll
                        for (int m = 0; m < MT; ++m) { A0[i][m] = 0u; A1[i][m] = 0u; A2[i][m] = 0; }
#pragma unroll
                    for (int jc = 0; jc < CPS; ++jc) {
                        const int j = js * CPS + jc;
                        const uint32_t coff = code_off + (uint32_t)(((j + rot) % NCH) * 16);
                        uint4 cj[RPT];
#pragma unroll
                        for (int i = 0; i < RPT; ++i)
                            cj[i] = (i == 0 || live[i]) ? lds128(rbase[i] + coff) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
#pragma unroll
                            for (int i = 0; i < RPT; ++i) {
                                const uint32_t wv = w == 0 ? cj[i].x : w == 1 ? cj[i].y : w == 2 ? cj[i].z : cj[i].w;
                                const uint32_t L = wv & 0x0F0F0F0Fu, H = wv & 0xF0F0F0F0u;
#pragma unroll
                                for (int m = 0; m < MT; ++m) {
                                    A0[i][m] = dp4a_uu(xp[m][j][w][0], L, A0[i][m]);
                                    A1[i][m] = dp4a_uu(xp[m][j][w][1], L, A1[i][m]);
                                    A2[i][m] = dp4a_su(xp[m][j][w][2], L, A2[i][m]);
                                    A0[i][m] = dp4a_uu(xp[m][j][w][3], H, A0[i][m]);
                                    A1[i][m] = dp4a_uu(xp[m][j][w][4], H, A1[i][m]);
                                    A2[i][m] = dp4a_su(xp[m][j][w][5], H, A2[i][m]);
                                }
                            }
                        }
                    }
                    if (seg_live[js]) {
#pragma unroll
                        for (int i = 0; i < RPT; ++i) {
                            if (i > 0 && !live[i]) continue;
                            const uint32_t e = lds32(rbase[i] + sc_off[js]);
                            const float scl = __half2float(__ushort_as_half((unsigned short)(e & 0xFFFFu)));
                            const float zf = (float)(int)(int16_t)(e >> 16);
#pragma unroll
                            for (int m = 0; m < MT; ++m) {
                                // (D / 16) 2^-S with D = A0 + 256 A1 + 65536 A2
                                float d = __fmul_rn((float)A0[i][m], q16[m]);
                                d = __fmaf_rn((float)A1[i][m], MT == 1 ? q16x256[m] : __fmul_rn(q16[m], 256.0f), d);
                                d = __fmaf_rn((float)A2[i][m], MT == 1 ? q16x65536[m] : __fmul_rn(q16[m], 65536.0f), d);
                                yv[i][m] = __fmaf_rn(scl, __fmaf_rn(-zf, sxf[m][js], d), yv[i][m]);
                            }
                        }
                    }
                }
                if (a.direct) {
                    // the warp holds the row's 32 slices: a butterfly over the warp, in a
                    // fixed order, and lane 0 stores the sum
#pragma unroll
                    for (int i = 0; i < RPT; ++i) {
                        float r = yv[i][0];
#pragma unroll
                        for (int off = 16; off >= 1; off >>= 1) r += __shfl_xor_sync(FULL, r, off);
                        if (lane == 0 && live[i]) {
                            const int64_t n = row0 + s * SR + slot + i * a.nslot;
                            if (a.out_fp32) static_cast<float *>(a.y)[(int64_t)m0 * a.N + n] = r;
                            else static_cast<__nv_bfloat16 *>(a.y)[(int64_t)m0 * a.N + n] = __float2bfloat16_rn(r);
                        }
                    }
                } else if (!a.warpred) {
#pragma unroll
                    for (int i = 0; i < RPT; ++i) {
                        if (!live[i]) continue;
                        const uint32_t rl = (uint32_t)(s * SR + slot + i * a.nslot);
#pragma unroll
                        for (int m = 0; m < MT; ++m) red[(rl * MT + m) * (uint32_t)a.rstr + sl] = yv[i][m];
                    }
                }
            }
            if (MT > 1 && a.warpred) {
                // the warp's 32 slices belong to one row: transpose-reduce its MT partials so
                // that lane l ends with the warp's sum for m = l / (32 / MT)
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const float r = warp_transpose_sum<MT>(yv[i], lane);
                    const int rl = s * SR + slot + i * a.nslot;
                    if (slot < a.nslot && rl < rows && (lane & (32 / MT - 1)) == 0)
                        red[((uint32_t)rl * MT + lane / (32 / MT)) * (uint32_t)a.rstr + sl / 32] = r;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot_s);
        }
        if (!ok) *(volatile int *)abort_flag = 1;
        if (a.direct) return;  // every row was stored in the stage loop

        // (4) row sums in a fixed order: lpr lanes per (row, m), each adding every lpr-th
        // partial in turn, then a butterfly over the lpr lanes
        named_bar_sync(1, NCT);
        const bool aborted = *(volatile int *)abort_flag != 0;
        float *outp = nullptr;
        if (a.kparts > 1) outp = a.ws_part + (size_t)kp * a.M * a.N;
        {
            const int lpr = a.lpr, opw = 32 / lpr;  // outputs per warp
            const int nv = a.warpred ? (nsl + 31) / 32 : nsl;
            const int j = lane & (lpr - 1);
            for (int ob = warp * opw; ob < rows * MT; ob += NCW * opw) {
                const int o = ob + lane / lpr;
                float acc = 0.0f;
                if (o < rows * MT)
                    for (int i = j; i < nv; i += lpr) acc += red[(size_t)o * a.rstr + i];
                for (int off = lpr >> 1; off >= 1; off >>= 1) acc += __shfl_xor_sync(FULL, acc, off);
                const int rl = o / MT, m = o - rl * MT;
                const int64_t n = row0 + rl;
                if (j == 0 && o < rows * MT && m0 + m < a.M && !aborted) {
                    if (outp) outp[(int64_t)(m0 + m) * a.N + n] = acc;
                    else if (a.out_fp32) static_cast<float *>(a.y)[(int64_t)(m0 + m) * a.N + n] = acc;
                    else static_cast<__nv_bfloat16 *>(a.y)[(int64_t)(m0 + m) * a.N + n] = __float2bfloat16_rn(acc);
                }
            }
        }
        if (a.kparts > 1) {
            // the last block of the row range to arrive adds the parts in order and resets the counter
            __threadfence();
            named_bar_sync(1, NCT);
            int *cnt = a.ws_count + (size_t)by * a.nrb + rb;
            if (tid == 0) {
                const int prev = atomicAdd(cnt, 1);
                *last_flag = (prev == a.kparts - 1) ? 1 : 0;
                __threadfence();
            }
            named_bar_sync(1, NCT);
            if (*last_flag) {
                for (int o = tid; o < rows * MT; o += NCT) {
                    const int rl = o / MT, m = o - rl * MT;
                    if (m0 + m >= a.M) continue;
                    const int64_t n = row0 + rl, idx = (int64_t)(m0 + m) * a.N + n;
                    float acc = 0.0f;
                    for (int p = 0; p < a.kparts; ++p) acc += __ldcg(a.ws_part + (size_t)p * a.M * a.N + idx);
                    if (aborted) continue;
                    if (a.out_fp32) static_cast<float *>(a.y)[idx] = acc;
                    else static_cast<__nv_bfloat16 *>(a.y)[idx] = __float2bfloat16_rn(acc);
                }
                if (tid == 0) *cnt = 0;
            }
        }
    }
}

template <int MT, int G>
__global__ void __launch_bounds__(THREADS, 1) gemv_kernel(const __grid_constant__ Args a) {
    gemv_block<MT, G>(a, (int)blockIdx.x, (int)blockIdx.y);
}

// Several independent problems in one launch: blocks [first[j], first[j+1]) work on problem j
// (whole rows, one K part each), so the per-launch phases (activation conversion, first
// stage, row sums) are paid once for the group.
constexpr int MAX_GROUP = 8;
struct GroupArgs {
    Args m[MAX_GROUP];
    int first[MAX_GROUP + 1];
    int count;
};

template <int MT, int G>
__global__ void __launch_bounds__(THREADS, 1) gemv_grouped_kernel(const __grid_constant__ GroupArgs ga) {
    int j = 0;
    while (j + 1 < ga.count && (int)blockIdx.x >= ga.first[j + 1]) ++j;
    gemv_block<MT, G>(ga.m[j], (int)blockIdx.x - ga.first[j], (int)blockIdx.y);
}

// ------------------------------------------------------------------ host side

struct Plan {
    Args a;
    int MT, sweeps, grid_x, smem;
};

static int sm_count_cached() {
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return num_sms();
    if (!cache[dev]) cache[dev] = num_sms();
    return cache[dev];
}

template <int MT>
static bool make_plan_parts(Plan &p, int64_t M, int64_t N, int64_t K, int g, int64_t S, int want_parts,
                            int64_t red_budget = RED_BUDGET) {
    using GE_ = Geo<MT>;
    const GemvLayout L = gemv_layout(N, K, g);
    Args &a = p.a;
    a = Args{};
    a.N = N; a.K = K; a.M = (int)M; a.J = (int)(K / g); a.g = g;
    a.RS = (uint32_t)L.row_bytes;
    a.tpr = (int)((K + GE_::KC - 1) / GE_::KC);
    // K parts: whole rows when the slices fit the consumer threads, else parts of a multiple
    // of 512 k (so that every part's scales start on a 16-byte boundary)
    const int unit = 512 / GE_::KC;
    if (want_parts == 1) {
        if (a.tpr > NCT) return false;
        a.kparts = 1;
        a.spp = a.tpr;
    } else {
        a.spp = (a.tpr + want_parts - 1) / want_parts;
        a.spp = (a.spp + unit - 1) / unit * unit;
        if (a.spp > NCT) return false;
        a.kparts = (a.tpr + a.spp - 1) / a.spp;
        if (a.kparts == 1) return false;
    }
    if (a.kparts == 1) {
        a.RSp = a.RS;
        a.KPB = (uint32_t)(K / 2);
    } else {
        a.KPB = (uint32_t)a.spp * (GE_::KC / 2);
        a.RSp = a.KPB + (uint32_t)(4 * a.spp * GE_::KC / g);
        a.RSp = (a.RSp + 15) / 16 * 16;
    }
    a.nslot = NCT / a.spp;
    a.rpt = GE_::RPT;
    const uint32_t planes_bytes = (uint32_t)(a.spp * GE_::PSTRIDE * 4);  // one activation row at a time
    const uint32_t sx_bytes = (uint32_t)(MT * a.spp * GE_::NCH * 4);
    const uint32_t pp_bytes = (uint32_t)(MT * a.spp * 4);
    a.SB = (uint32_t)(a.nslot * a.rpt) * a.RSp;
    a.warpred = (MT > 1 && a.spp % 32 == 0) ? 1 : 0;
    a.nred = a.warpred ? a.spp / 32 : a.spp;
    // rows per block: N spread over the SMs, capped by the row-partial buffer (sized for the
    // widest padding of a (row, m)'s partials, nred + 31 words)
    int64_t nrb = S < N ? S : N;
    int64_t rpc = (N + nrb - 1) / nrb;
    const int64_t rpc_cap = red_budget / ((int64_t)MT * (a.nred + 31) * 4);
    if (rpc_cap < 1) return false;
    if (rpc > rpc_cap) rpc = rpc_cap;
    a.rpc = (int)rpc;
    // (only for blocks whose rows fit one stage: in a longer stream the butterfly of every row
    // lengthens the dot-product-bound loop more than the final pass costs)
    a.direct = (MT == 1 && a.kparts == 1 && a.spp == 32 && rpc <= (int64_t)a.nslot * a.rpt) ? 1 : 0;
    // final reduction: as many lanes per (row, m) as the consumer threads allow (a power of
    // two up to 32); partials of consecutive (row, m) are rstr = lpr (mod 32) words apart, so
    // a warp's loads hit distinct banks
    a.lpr = 32;
    while (a.lpr > 1 && (int64_t)rpc * MT * a.lpr > NCT) a.lpr >>= 1;
    a.rstr = a.lpr == 32 ? a.nred : a.nred + ((a.lpr - a.nred % 32) % 32 + 32) % 32;
    a.nrb = (int)((N + rpc - 1) / rpc);
    a.off_sx = 512;
    a.off_pp = a.off_sx + (sx_bytes + 15) / 16 * 16;
    a.off_red = a.off_pp + (pp_bytes + 15) / 16 * 16;
    a.off_ring = a.off_red + (uint32_t)((rpc * MT * a.rstr * 4 + 15) / 16 * 16);
    const int64_t avail = (int64_t)SMEM_MAX - a.off_ring - SLACK;
    int NS = (int)(avail / a.SB);
    if (NS > MAX_STAGES) NS = MAX_STAGES;
    if ((int64_t)NS * a.SB >= (int64_t)planes_bytes + 2 * (int64_t)a.SB) {
        // the planes sit at the end of the ring; the stages below them are issued at once
        const int64_t ring_bytes = (int64_t)NS * a.SB;
        const int64_t p0 = (ring_bytes - planes_bytes) / 16 * 16;
        a.off_planes = (uint32_t)(a.off_ring + p0);
        a.NS_early = (int)(p0 / a.SB);
        p.smem = (int)(a.off_ring + ring_bytes + SLACK);
    } else {
        // too little room for that: the planes follow the ring
        NS = (int)((avail - planes_bytes) / a.SB);
        if (NS > MAX_STAGES) NS = MAX_STAGES;
        if (NS < 2) return false;
        a.off_planes = (uint32_t)(a.off_ring + (int64_t)NS * a.SB);
        a.NS_early = NS;
        p.smem = (int)(a.off_planes + planes_bytes + SLACK);
    }
    a.NS = NS;
    p.MT = MT;
    p.sweeps = (int)((M + MT - 1) / MT);
    p.grid_x = a.nrb * a.kparts;
    return true;
}

// Whole rows per block when they fit (threads and shared memory), else the fewest K parts
// that do.
template <int MT>
static bool make_plan_mt(Plan &p, int64_t M, int64_t N, int64_t K, int g, int64_t S) {
    const int tpr = (int)((K + Geo<MT>::KC - 1) / Geo<MT>::KC);
    for (int parts = 1; parts <= tpr; ++parts)
        if (make_plan_parts<MT>(p, M, N, K, g, S, parts)) return true;
    return false;
}

// MT = activation rows per sweep: as many as the registers hold for this K (4, 2 or 1),
// with whole rows per block when possible
// Whole rows per block with MT rows per sweep. When the row-partial buffer of the default size
// caps a block's rows so low that the blocks outnumber the SMs (a second, mostly empty wave),
// a larger buffer (up to four times) is taken if shared memory still holds the ring.
template <int MT>
static bool make_plan_whole(Plan &p, int64_t M, int64_t N, int64_t K, int g, int64_t S) {
    if (!make_plan_parts<MT>(p, M, N, K, g, S, 1)) return false;
    for (int64_t rb = 2 * RED_BUDGET; rb <= 4 * RED_BUDGET && p.grid_x > S; rb += RED_BUDGET) {
        Plan q;
        if (make_plan_parts<MT>(q, M, N, K, g, S, 1, rb) && q.grid_x < p.grid_x) p = q;
    }
    return true;
}

static bool make_plan(Plan &p, int64_t M, int64_t N, int64_t K, int g, int64_t S) {
    const int want = M >= 3 ? 4 : (int)M;
    if (want >= 4 && make_plan_whole<4>(p, M, N, K, g, S)) return true;
    if (want >= 2 && make_plan_whole<2>(p, M, N, K, g, S)) return true;
    return make_plan_mt<1>(p, M, N, K, g, S);
}

template <int MT, int G>
static void *kernel_ptr() { return reinterpret_cast<void *>(gemv_kernel<MT, G>); }

static void *pick_kernel(int MT, int g) {
    // groups of 128 or more: every slice (at most 128 k) lies in one group, one kernel serves
    if (MT == 4) return g == 32 ? kernel_ptr<4, 32>() : (g == 64 ? kernel_ptr<4, 64>() : kernel_ptr<4, 128>());
    if (MT == 2) return g == 32 ? kernel_ptr<2, 32>() : (g == 64 ? kernel_ptr<2, 64>() : kernel_ptr<2, 128>());
    return g == 32 ? kernel_ptr<1, 32>() : (g == 64 ? kernel_ptr<1, 64>() : kernel_ptr<1, 128>());
}

static size_t ws_need(const Plan &p) {
    if (p.a.kparts == 1) return 0;
    const size_t part = (size_t)p.a.kparts * p.a.M * p.a.N * 4;
    return (part + 255) / 256 * 256 + (size_t)p.sweeps * p.a.nrb * 4;
}

static w4_status run(const void *x, int64_t M, const void *packed, int64_t N, int64_t K, int g, void *y, int out_fp32,
                     void *ws, size_t ws_bytes, int pdl, cudaStream_t stream, const void *next = nullptr,
                     size_t next_bytes = 0) {
    Plan p;
    if (!make_plan(p, M, N, K, g, sm_count_cached())) return W4_ERR_SHAPE;
    Args &a = p.a;
    const size_t need = ws_need(p);
    if (need) {
        if (!ws || ws_bytes < need) return W4_ERR_WORKSPACE;
        a.ws_part = static_cast<float *>(ws);
        a.ws_count = reinterpret_cast<int *>(static_cast<uint8_t *>(ws) + (need - (size_t)p.sweeps * a.nrb * 4));
    }
    a.x = static_cast<const uint16_t *>(x);
    a.w = static_cast<const uint8_t *>(packed);
    a.y = y;
    a.out_fp32 = out_fp32;
    a.status = device_status_ptr();
    a.pdl = pdl;
    if (next && next_bytes >= 16) {
        const uint64_t nblk = (uint64_t)p.grid_x * (uint64_t)p.sweeps;
        a.pf = static_cast<const uint8_t *>(next);
        a.pf_bytes = (uint64_t)next_bytes / 16 * 16;
        a.pf_chunk = (a.pf_bytes + nblk - 1) / nblk;
        a.pf_chunk = (a.pf_chunk + 15) / 16 * 16;
    }
    void *fn = pick_kernel(p.MT, g);
    static int attr_done[64][3][3] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int mi = p.MT == 4 ? 2 : p.MT - 1, gi = g == 32 ? 0 : (g == 64 ? 1 : 2);
    if (dev >= 0 && dev < 64 && !attr_done[dev][mi][gi]) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_MAX) != cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev][mi][gi] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.grid_x, (unsigned)p.sweeps);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[] = {&a};
    if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}

// Plans of a group of problems launched together: problem j gets a share of the SMs in
// proportion to its bytes, whole rows per block and one K part; blocks may hold more rows than
// in a single launch (a larger row-partial buffer, at least two ring stages), so that the group
// fits one wave. All problems must take the same activation rows per sweep.
static bool make_group_plan(int count, int64_t M, const int64_t *N, const int64_t *K, int g, int64_t sms, Plan *pl,
                            int *first) {
    double total = 0.0;
    for (int j = 0; j < count; ++j) total += (double)N[j] * (double)K[j] * (0.5 + 4.0 / g);
    first[0] = 0;
    for (int j = 0; j < count; ++j) {
        const double share = (double)N[j] * (double)K[j] * (0.5 + 4.0 / g) / total;
        int64_t S = (int64_t)(share * (double)sms);
        if (S < 1) S = 1;
        bool ok = false;
        const int want = M >= 3 ? 4 : (int)M;
        for (int64_t rb = 3 * RED_BUDGET; rb >= RED_BUDGET && !ok; rb -= RED_BUDGET / 2) {
            if (want >= 4) ok = make_plan_parts<4>(pl[j], M, N[j], K[j], g, S, 1, rb);
            else if (want == 2) ok = make_plan_parts<2>(pl[j], M, N[j], K[j], g, S, 1, rb);
            else ok = make_plan_parts<1>(pl[j], M, N[j], K[j], g, S, 1, rb);
        }
        if (!ok || pl[j].a.kparts != 1 || pl[j].MT != pl[0].MT || pl[j].sweeps != pl[0].sweeps)
            return false;
        first[j + 1] = first[j] + pl[j].grid_x;
    }
    return true;
}

template <int MT>
static void *grouped_kernel_ptr(int g) {
    return g == 32 ? reinterpret_cast<void *>(gemv_grouped_kernel<MT, 32>)
         : g == 64 ? reinterpret_cast<void *>(gemv_grouped_kernel<MT, 64>)
                   : reinterpret_cast<void *>(gemv_grouped_kernel<MT, 128>);
}

static w4_status run_grouped(int count, const void *const *x, int64_t M, const void *const *packed, const int64_t *N,
                             const int64_t *K, int g, void *const *y, int out_fp32, int pdl, cudaStream_t stream) {
    Plan pl[MAX_GROUP];
    GroupArgs ga{};
    if (!make_group_plan(count, M, N, K, g, sm_count_cached(), pl, ga.first)) return W4_ERR_UNSUPPORTED;
    int smem = 0;
    for (int j = 0; j < count; ++j) {
        Args &a = pl[j].a;
        a.x = static_cast<const uint16_t *>(x[j]);
        a.w = static_cast<const uint8_t *>(packed[j]);
        a.y = y[j];
        a.out_fp32 = out_fp32;
        a.status = device_status_ptr();
        a.pdl = pdl;
        ga.m[j] = a;
        if (pl[j].smem > smem) smem = pl[j].smem;
    }
    ga.count = count;
    const int MT = pl[0].MT;
    void *fn = MT == 4 ? grouped_kernel_ptr<4>(g) : MT == 2 ? grouped_kernel_ptr<2>(g) : grouped_kernel_ptr<1>(g);
    static int attr_done[64][3][3] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int mi = MT == 4 ? 2 : MT - 1, gi = g == 32 ? 0 : (g == 64 ? 1 : 2);
    if (dev >= 0 && dev < 64 && !attr_done[dev][mi][gi]) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_MAX) != cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev][mi][gi] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ga.first[count], (unsigned)pl[0].sweeps);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[] = {&ga};
    if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}

// Host-only view of a plan: out = {activation rows per sweep, sweeps, K parts, row blocks,
// rows per block, dynamic shared memory bytes, ring stages, workspace bytes}.
static bool describe_plan(int64_t M, int64_t N, int64_t K, int g, int64_t sms, int64_t *out) {
    Plan p;
    if (!make_plan(p, M, N, K, g, sms)) return false;
    out[0] = p.MT;
    out[1] = p.sweeps;
    out[2] = p.a.kparts;
    out[3] = p.a.nrb;
    out[4] = p.a.rpc;
    out[5] = p.smem;
    out[6] = p.a.NS;
    out[7] = (int64_t)ws_need(p);
    return true;
}

// The workspace a call may need: the largest over M = 1..16 on this device's SM count.
size_t workspace_bytes(int64_t N, int64_t K, int g) {
    size_t worst = 0;
    const int64_t S = sm_count_cached();
    for (int64_t M = 1; M <= 16; ++M) {
        Plan p;
        if (make_plan(p, M, N, K, g, S)) {
            const size_t v = ws_need(p);
            worst = v > worst ? v : worst;
        }
    }
    return worst;
}

}  // namespace gemv
}  // namespace w4

using namespace w4;

static bool gemv_shape_ok(int64_t M, int64_t N, int64_t K) {
    return M >= 1 && M <= 16 && N >= 1 && N <= ((int64_t)1 << 31) && K >= 32 && K % 32 == 0 && K <= ((int64_t)1 << 24);
}

W4_API size_t w4a16_gemv_workspace_bytes(int64_t N, int64_t K, int group) {
    if (!gemv_shape_ok(1, N, K) || !valid_group(group) || K % group != 0) return 0;
    return gemv::workspace_bytes(N, K, group);
}

W4_API w4_status w4a16_gemv_schedule(int64_t M, int64_t N, int64_t K, int group, int sms, int64_t *out) {
    if (!out) return W4_ERR_NULL;
    if (!gemv_shape_ok(M, N, K) || sms < 1 || sms > 4096) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    return gemv::describe_plan(M, N, K, group, sms, out) ? W4_OK : W4_ERR_SHAPE;
}

W4_API w4_status w4a16_gemv(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K, int group,
                            int mode, void *y, int flags, void *workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
    if (!x_bf16 || !packed || !y) return W4_ERR_NULL;
    if (!valid_mode(mode) || (flags & ~(W4_OUT_FP32 | W4_OVERLAP_PREVIOUS))) return W4_ERR_ARG;
    const int out_fp32 = (flags & W4_OUT_FP32) ? 1 : 0;
    const int pdl = (flags & W4_OVERLAP_PREVIOUS) ? 1 : 0;
    if (!gemv_shape_ok(M, N, K)) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(y) || (workspace && !aligned16(workspace)))
        return W4_ERR_ALIGN;
    return gemv::run(x_bf16, M, packed, N, K, group, y, out_fp32, workspace, workspace_bytes, pdl, stream);
}

W4_API w4_status w4a16_gemv_prefetch_next(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K,
                                          int group, int mode, void *y, int flags, void *workspace,
                                          size_t workspace_bytes, const void *next, size_t next_bytes,
                                          cudaStream_t stream) {
    if (!x_bf16 || !packed || !y || (!next && next_bytes)) return W4_ERR_NULL;
    if (!valid_mode(mode) || (flags & ~(W4_OUT_FP32 | W4_OVERLAP_PREVIOUS))) return W4_ERR_ARG;
    const int out_fp32 = (flags & W4_OUT_FP32) ? 1 : 0;
    const int pdl = (flags & W4_OVERLAP_PREVIOUS) ? 1 : 0;
    if (!gemv_shape_ok(M, N, K)) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(y) || (workspace && !aligned16(workspace)) ||
        (next && !aligned16(next)))
        return W4_ERR_ALIGN;
    return gemv::run(x_bf16, M, packed, N, K, group, y, out_fp32, workspace, workspace_bytes, pdl, stream, next,
                     next_bytes);
}

W4_API w4_status w4a16_gemv_grouped(int count, const void *const *x_bf16, int64_t M, const void *const *packed,
                                    const int64_t *N, const int64_t *K, int group, int mode, void *const *y,
                                    int flags, cudaStream_t stream) {
    if (!x_bf16 || !packed || !N || !K || !y) return W4_ERR_NULL;
    if (count < 1 || count > gemv::MAX_GROUP) return W4_ERR_SHAPE;
    if (!valid_mode(mode) || (flags & ~(W4_OUT_FP32 | W4_OVERLAP_PREVIOUS))) return W4_ERR_ARG;
    if (!valid_group(group)) return W4_ERR_GROUP;
    for (int j = 0; j < count; ++j) {
        if (!x_bf16[j] || !packed[j] || !y[j]) return W4_ERR_NULL;
        if (!gemv_shape_ok(M, N[j], K[j])) return W4_ERR_SHAPE;
        if (K[j] % group != 0) return W4_ERR_GROUP;
        if (!aligned16(x_bf16[j]) || !aligned16(packed[j]) || !aligned16(y[j])) return W4_ERR_ALIGN;
    }
    return gemv::run_grouped(count, x_bf16, M, packed, N, K, group, y, (flags & W4_OUT_FP32) ? 1 : 0,
                             (flags & W4_OVERLAP_PREVIOUS) ? 1 : 0, stream);
}

// Host-only: the blocks of each problem of a grouped launch on `sms` SMs (0 if the group is not
// supported).
W4_API w4_status w4a16_gemv_grouped_schedule(int count, int64_t M, const int64_t *N, const int64_t *K, int group,
                                             int sms, int64_t *blocks) {
    if (!N || !K || !blocks) return W4_ERR_NULL;
    if (count < 1 || count > gemv::MAX_GROUP || sms < 1 || sms > 4096) return W4_ERR_SHAPE;
    if (!valid_group(group)) return W4_ERR_GROUP;
    for (int j = 0; j < count; ++j)
        if (!gemv_shape_ok(M, N[j], K[j]) || K[j] % group != 0) return W4_ERR_SHAPE;
    gemv::Plan pl[gemv::MAX_GROUP];
    int first[gemv::MAX_GROUP + 1];
    if (!gemv::make_group_plan(count, M, N, K, group, sms, pl, first)) return W4_ERR_UNSUPPORTED;
    for (int j = 0; j < count; ++j) blocks[j] = first[j + 1] - first[j];
    return W4_OK;
}

// ------------------------------------------------------------------ allocation-free variant
//
// Callers that must not allocate device memory on the hot path -- a plug-in running inside
// another runtime that owns all device memory, or a latency-critical decode loop where
// cudaMalloc's implicit device synchronisation is not acceptable -- can call
// w4a16_gemv_noalloc. Its scratch (the partial sums and arrival counters of rows split along
// K over several blocks) is a fixed array in this library's device memory, reserved when the
// library loads on a GPU and held until the process exits.

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

static w4_status run_noalloc(const void *x, int64_t M, const void *packed, int64_t N, int64_t K, int g, void *y,
                             int out_fp32, int pdl, cudaStream_t stream) {
    Plan p;
    if (!make_plan(p, M, N, K, g, sm_count_cached())) return W4_ERR_SHAPE;
    const size_t need = ws_need(p);
    if (need > kNoAllocScratchBytes) return W4_ERR_SCRATCH_LIMIT;
    uint8_t *ws = nullptr;
    if (need) {
        ws = static_cast<uint8_t *>(noalloc_scratch());
        if (!ws) return W4_ERR_CUDA;
        // the arrival counters must start at zero; a call normally leaves them at zero, but
        // the array outlives every call, so clear them on the caller's stream first
        const size_t cnt = (size_t)p.sweeps * p.a.nrb * 4;
        if (cudaMemsetAsync(ws + need - cnt, 0, cnt, stream) != cudaSuccess) return W4_ERR_CUDA;
    }
    return run(x, M, packed, N, K, g, y, out_fp32, ws, kNoAllocScratchBytes, pdl, stream);
}

}  // namespace gemv
}  // namespace w4

W4_API size_t w4a16_gemv_noalloc_scratch_limit(void) { return w4::gemv::kNoAllocScratchBytes; }

W4_API w4_status w4a16_gemv_noalloc(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K,
                                    int group, int mode, void *y, int flags, cudaStream_t stream) {
    if (!x_bf16 || !packed || !y) return W4_ERR_NULL;
    if (!valid_mode(mode) || (flags & ~(W4_OUT_FP32 | W4_OVERLAP_PREVIOUS))) return W4_ERR_ARG;
    if (!gemv_shape_ok(M, N, K)) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(y)) return W4_ERR_ALIGN;
    const int out_fp32 = (flags & W4_OUT_FP32) ? 1 : 0;
    const int pdl = (flags & W4_OVERLAP_PREVIOUS) ? 1 : 0;
    return gemv::run_noalloc(x_bf16, M, packed, N, K, group, y, out_fp32, pdl, stream);
}
