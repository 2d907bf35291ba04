// w4a16_gemm_tc: the W4A16 product for a few activation rows (1 <= M <= 16) on the sm_100a
// tensor cores (tcgen05.mma, TMEM operands and accumulators, TMA activation tiles).
//
//   y[m, n] = sum_j s[n,j] * sum_{k in group j} (q[n,k] - z[n,j]) * x[m,k]
//           = sum_j s[n,j] * ( P_j[m,n] - (z[n,j] - 8) X_j[m] ),
//   P_j[m,n] = sum_{k in j} (q[n,k] - 8) x[m,k],      X_j[m] = sum_{k in j} x[m,k]
//
// "Four-bit inference ... Tahoma", the W4A16 path (weights stay 4-bit in HBM and are expanded
// next to the arithmetic, activations stay bf16, accumulation is fp32, one fp16 scale per
// group) and "4-bit by default" (small-batch decode is bound by reading the weights). The
// CUDA-core GEMV (w4a16_gemv) forms integer dot products per weight and activation row, so its
// instruction count grows with M; here one expansion per weight feeds all M rows at once.
//
// Design (one persistent CTA per SM):
//  * swap-AB: 128 weight rows are the MMA's M (one TMEM lane per weight row) and the M <= 16
//    activation rows its N = 16 (rows past M arrive as zeros from TMA);
//  * expansion: a nibble q becomes the bf16 value q - 8, exactly. Two nibbles OR-ed into the
//    mantissas of the pattern 0x4300 (128.0) give 128 + q for two k at once, and one packed
//    bf16 subtraction of 136 leaves q - 8. The expanded weights go from registers straight
//    into TMEM (tcgen05.st), where the MMA reads its A operand;
//  * per group j, kind::f16 MMAs (K = 16 each) accumulate P_j into one of several 16-column
//    TMEM buffers; promotion warps read it back and add s (P - (z - 8) X) to fp32 registers.
//    For asymmetric weights a group-sum warp forms X_j from the activation tile in shared
//    memory (each half-warp sums half of a stage's k for 16 rows, the halves meet by a
//    shuffle) and hands it over next to the accumulator (its barrier counts the MMA commit and
//    this warp). The product of an expanded weight and a bf16 activation is exact in fp32;
//    rounding enters in the accumulation;
//  * stream-K: the (tile, k-block) units of the problem, in order, are split evenly over the
//    CTAs; when several CTAs share a tile, each warp of the last one to finish adds the
//    others' partial sums for its 32 rows in CTA order, so results do not depend on timing;
//  * weights (W4_LAYOUT_TC) are stored unit by unit, each unit one contiguous record, so a
//    CTA's share is one contiguous byte range streamed by bulk copies;
//  * warp roles: warps 0-3 and 11-14 expansion (each set half of a stage's k), 4-7 promotion
//    (a warp touches the TMEM lane quarter warp % 4), warp 8 the producer (one bulk copy per
//    record, TMA of activation tiles), warp 9 TMEM owner and single-thread MMA issuer, warp 10
//    group sums;
//  * every mbarrier wait is bounded by wall-clock time; on expiry the kernel records
//    W4_ERR_TIMEOUT, every role sees the abort flag, TMEM is freed and the CTA returns.
#include "w4_common.cuh"
#include "w4_layout.cuh"

#include <cuda.h>

namespace w4 {
namespace tc16 {

constexpr int THREADS = 480;
constexpr int TM = 128;                       // weight rows per tile (MMA M)
constexpr int TN = 16;                        // activation rows per tile (MMA N)
constexpr uint64_t kWaitNs = 2000000000ull;   // 2 s per wait
constexpr uint32_t SMEM_RING = 200 * 1024;    // shared memory for the stage ring

// Geometry for group size G.
template <int G> struct Geo {
    static constexpr int KS = TcLayoutGeo::ks(G);          // k per unit (one pipeline stage)
    static constexpr int GPS = KS / G;                     // groups per stage
    static constexpr int SPG = G / 16;                     // MMAs (K = 16) per group
    static constexpr int CHUNKS = KS / 32;                 // 16-byte code chunks per row and stage
    static constexpr uint32_t CODE_BYTES = TcLayoutGeo::code_bytes(G);
    static constexpr uint32_t REC = TcLayoutGeo::record_bytes(G);
    static constexpr uint32_t XB = KS * TN * 2;            // activation tile: 16 rows x KS bf16
    static constexpr uint32_t STAGE = (XB + REC + 1023) / 1024 * 1024;
    static constexpr int NS = (int)(SMEM_RING / STAGE) < 16 ? (int)(SMEM_RING / STAGE) : 16;
    static constexpr int ACOLS = KS / 2;                   // TMEM columns of one expanded stage
    static constexpr int NA = KS == 256 ? 2 : 4;           // expanded stages in TMEM
    static constexpr int NACC = 8;                         // accumulator buffers
    static constexpr int COL_ACC = NA * ACOLS;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t SMEM_BYTES = NS * STAGE + 1024 /*control*/ + 1024 /*alignment*/;
    static constexpr int HALF = KS / 2;                    // k of a stage per half-warp (group sums)
    static constexpr int XPL = G <= HALF ? HALF / G : 1;   // group sums a lane holds per stage
    static_assert(COL_ACC + NACC * TN <= (int)TMEM_COLS, "TMEM budget");
    static_assert(XB % 1024 == 0 && STAGE % 1024 == 0, "swizzle atoms stay aligned");
    static_assert(NS >= 4, "ring depth");
};

struct Smem {
    uint64_t full[16];      // record and activation tile landed (TMA / bulk-copy bytes)
    uint64_t empty[16];     // the stage is free: MMA commit + 8 expansion + 4 promotion warps
                            // + the group-sum warp
    uint64_t afull[4];      // an expanded stage is in TMEM (one arrival per expansion warp)
    uint64_t afree[4];      // the MMAs that read an expanded stage completed (commit)
    uint64_t accf[8];       // a group's accumulator (commit) and its sums X_j (group-sum warp)
    uint64_t acce[8];       // the promotion warps read them (one arrival per warp)
    float xs[8][16];        // X_j per accumulator buffer and activation row
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Smem) <= 1024, "control block");

struct Args {
    const uint8_t *w;       // W4_LAYOUT_TC records
    void *y;                // [M][N] bf16 or fp32
    float *part;            // [grid][2][128][16] partial sums of shared tiles
    uint32_t *cnt;          // [T][4] arrival counters (zero between calls)
    int *status;
    int64_t N;
    int64_t L;              // units = T * NKB
    int NKB;                // k-blocks (units) per tile
    int M;
    int mw;                 // float4 per row of a partial sum: ceil(M / 4)
    int x3d;                // activation tiles by one 3-D TMA (K % 64 == 0), else 2-D per 64 k
    int out_fp32;
    int asym;
    int pdl;
};

// instruction descriptor: D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9, 10-12 = 1), both
// K-major, N = 16 (bits 17-22 = N / 8), M = 128 (bits 24-28 = M / 16)
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TN >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);

// B (activation) descriptor, K-major with the 128-byte swizzle: low word = start address in
// 16-byte units | leading byte offset 1 (unused for swizzled K-major); high word = stride byte
// offset between 8-row atoms (1024 bytes = 64 units), descriptor version 1 (bit 46), swizzle
// mode 2 (bits 61-63). One K step of 16 bf16 (32 bytes) adds 2 to the low word.
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr) { return ((saddr & 0x3FFFFu) >> 4) | (1u << 16); }
constexpr uint32_t kDescHi = 64u | (1u << 14) | (2u << 29);

// D[tmem_d] (+)= A[tmem_a] * B[desc] for one K step of 16, A read from TMEM
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint32_t b_lo, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n .reg .b64 db;\n setp.ne.b32 p, %3, 0;\n mov.b64 db, {%2, %4};\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %5, p;\n}\n" ::"r"(tmem_d),
        "r"(tmem_a), "r"(b_lo), "r"(accumulate), "r"(kDescHi), "r"(kIdesc));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 16 columns of 32-bit values from registers into TMEM (one column per register)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 columns of 32-bit accumulator (one column per register)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// Wait for this thread's tcgen05.ld; the loaded registers are in/out operands so that no use
// of them moves above the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_addr(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
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

__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Eight codes of one W4_LAYOUT_TC word (nibble p holds k = 2p for p < 4 and k = 2(p-4)+1
// otherwise) as four bf16 pairs (k = 2s, 2s+1), each value q - 8.
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t *o) {
#pragma unroll
    for (int s = 0; s < 4; ++s) o[s] = sub_bf16x2(((w >> (4 * s)) & 0x000F000Fu) | 0x43004300u, 0x43084308u);
}

// A wait by lane 0 for the warp; the warp barrier orders the other lanes after its acquire.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    bool r = true;
    if ((threadIdx.x & 31) == 0) r = mbar_wait_abortable(bar, parity, &sm->abort, status, kWaitNs);
    r = __shfl_sync(FULL, r ? 1 : 0, 0) != 0;
    __syncwarp();
    return r;
}
__device__ __forceinline__ bool wait1(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    return mbar_wait_abortable<true>(bar, parity, &sm->abort, status, kWaitNs);
}

// First unit of CTA c and the CTA that holds unit u, for L units over P CTAs (64-bit
// divisions: used once per CTA and once per shared tile, never per stage).
__device__ __forceinline__ int64_t unit_begin(int64_t c, int64_t L, int64_t P) { return c * L / P; }
__device__ __forceinline__ int64_t unit_owner(int64_t u, int64_t L, int64_t P) {
    const int64_t c = ((u + 1) * P - 1) / L;
    return c < P - 1 ? c : P - 1;
}

// position in a ring of N slots and the phase parity of the current lap
template <int N> struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next() {
        if (++slot == N) { slot = 0; phase ^= 1u; }
    }
};

__device__ __forceinline__ void store_row(const Args &a, int64_t n, const float (&acc)[TN]) {
    if (n >= a.N) return;
    if (a.out_fp32) {
        float *y = static_cast<float *>(a.y);
#pragma unroll
        for (int m = 0; m < TN; ++m)
            if (m < a.M) y[(int64_t)m * a.N + n] = acc[m];
    } else {
        __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(a.y);
#pragma unroll
        for (int m = 0; m < TN; ++m)
            if (m < a.M) y[(int64_t)m * a.N + n] = __float2bfloat16_rn(acc[m]);
    }
}

// Sum of the partial sums of weight row r (within its tile) over the CTAs cf..cl, in CTA order:
// MW float4 (activation rows 4q .. 4q+3) per CTA, 16 loads in flight at a time. CTA cf's part
// is in its slot w_first, every later CTA's in its slot 0.
template <int MW>
__device__ __forceinline__ void reduce_parts(const Args &a, int r, int64_t cf, int64_t cl, int w_first,
                                             float (&sum)[TN]) {
    constexpr int CPR = 16 / MW;  // CTAs per round
    for (int64_t c0 = cf; c0 <= cl; c0 += CPR) {
        float4 pv[CPR][MW];
#pragma unroll
        for (int j = 0; j < CPR; ++j) {
            const int64_t c = c0 + j <= cl ? c0 + j : cl;
            const int wc = c == cf ? w_first : 0;
            const float4 *src = reinterpret_cast<const float4 *>(a.part + (((size_t)c * 2 + wc) * TM + r) * TN);
#pragma unroll
            for (int q = 0; q < MW; ++q) pv[j][q] = __ldcg(src + q);
        }
#pragma unroll
        for (int j = 0; j < CPR; ++j) {
            if (c0 + j > cl) break;
#pragma unroll
            for (int q = 0; q < MW; ++q) {
                sum[4 * q] += pv[j][q].x;
                sum[4 * q + 1] += pv[j][q].y;
                sum[4 * q + 2] += pv[j][q].z;
                sum[4 * q + 3] += pv[j][q].w;
            }
        }
    }
}

template <int G>
__global__ void __launch_bounds__(THREADS, 1) w4a16_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const Args a) {
    using GE = Geo<G>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *sm = reinterpret_cast<Smem *>(base + GE::NS * GE::STAGE);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t P = gridDim.x;
    const int64_t u0 = unit_begin(blockIdx.x, a.L, P), u1 = unit_begin((int64_t)blockIdx.x + 1, a.L, P);
    const int n_units = (int)(u1 - u0);
    const int64_t t0 = u0 / a.NKB;          // tile of the first unit
    const int kb0 = (int)(u0 - t0 * a.NKB);  // its k-block

    if (threadIdx.x == 0) {
        for (int s = 0; s < GE::NS; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 14);
        }
        for (int s = 0; s < GE::NA; ++s) {
            mbar_init(&sm->afull[s], 8);
            mbar_init(&sm->afree[s], 1);
        }
        for (int b = 0; b < GE::NACC; ++b) {
            mbar_init(&sm->accf[b], 2);
            mbar_init(&sm->acce[b], 4);
        }
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sm->tmem_base)),
                     "r"(GE::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;

    if (warp == 8) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            // activations (and, for the next kernel, this one's outputs) are ordered after the
            // previous kernel on the stream
            if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
            Ring<GE::NS> rs;
            int issued = 0, kb = kb0;
            const uint8_t *src = a.w + (size_t)u0 * GE::REC;
            for (int i = 0; i < n_units; ++i, rs.next(), src += GE::REC) {
                if (!wait1(&sm->empty[rs.slot], rs.phase ^ 1u, sm, a.status)) break;
                uint8_t *st = base + (size_t)rs.slot * GE::STAGE;
                mbar_arrive_expect_tx(&sm->full[rs.slot], GE::XB + GE::REC);
                bulk_g2s_stream(st + GE::XB, src, GE::REC, &sm->full[rs.slot]);
                if (a.x3d) {
                    tma_load_3d(st, &tm_x, 0, 0, kb * (GE::KS / 64), &sm->full[rs.slot]);
                } else {
#pragma unroll
                    for (int h = 0; h < GE::KS / 64; ++h)
                        tma_load_2d(st + h * (TN * 128), &tm_x, kb * GE::KS + 64 * h, 0, &sm->full[rs.slot]);
                }
                kb = kb + 1 == a.NKB ? 0 : kb + 1;
                ++issued;
            }
            if (a.pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
            // no copy may land after the CTA exits
            for (int i = issued > GE::NS ? issued - GE::NS : 0; i < issued; ++i)
                (void)mbar_wait_bounded(&sm->full[i % GE::NS], (uint32_t)(i / GE::NS) & 1u, a.status);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            Ring<GE::NS> rs;
            Ring<GE::NA> ra;
            Ring<GE::NACC> rb;
            int done = 0;
            bool ok = true;
            for (int i = 0; i < n_units && ok; ++i, rs.next(), ra.next()) {
                if (!wait1(&sm->full[rs.slot], rs.phase, sm, a.status)) break;
                if (!wait1(&sm->afull[ra.slot], ra.phase, sm, a.status)) break;
                tc_fence_after();
                const uint32_t xlo = desc_lo(smem_addr(base + (size_t)rs.slot * GE::STAGE));
                const uint32_t at = tmem + (uint32_t)(ra.slot * GE::ACOLS);
#pragma unroll 1
                for (int gg = 0; gg < GE::GPS; ++gg, rb.next()) {
                    if (!wait1(&sm->acce[rb.slot], rb.phase ^ 1u, sm, a.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t dacc = tmem + (uint32_t)(GE::COL_ACC + rb.slot * TN);
#pragma unroll
                    for (int kk = 0; kk < GE::SPG; ++kk) {
                        const int ks = gg * GE::SPG + kk;                                // K step in the stage
                        const uint32_t blo = xlo + (uint32_t)((ks >> 2) * (TN * 128 / 16) + (ks & 3) * 2);
                        mma_ts(dacc, at + (uint32_t)(ks * 8), blo, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sm->accf[rb.slot]);
                }
                if (!ok) break;
                mma_commit(&sm->afree[ra.slot]);
                mma_commit(&sm->empty[rs.slot]);
                ++done;
            }
            // no commit may arrive after the CTA exits: wait for the last stages' MMAs
            for (int i = done > GE::NA ? done - GE::NA : 0; i < done; ++i)
                (void)mbar_wait_bounded(&sm->afree[i % GE::NA], (uint32_t)(i / GE::NA) & 1u, a.status);
        }
        __syncwarp();
    } else if (warp < 4 || warp >= 11) {
        // ------------------------------------------------ expansion (row 32 (warp % 4) + lane;
        // warps 0-3 take the first half of a stage's code chunks, warps 11-14 the second)
        const int q4 = warp & 3, r = q4 * 32 + lane;
        const int c0 = warp < 4 ? 0 : GE::CHUNKS / 2;
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        Ring<GE::NS> rs;
        Ring<GE::NA> ra;
        for (int i = 0; i < n_units; ++i, rs.next(), ra.next()) {
            if (!warp_wait(&sm->full[rs.slot], rs.phase, sm, a.status)) break;
            if (!warp_wait(&sm->afree[ra.slot], ra.phase ^ 1u, sm, a.status)) break;
            tc_fence_after();
            const uint32_t rec = smem_addr(base + (size_t)rs.slot * GE::STAGE + GE::XB);
            uint4 cw[GE::CHUNKS / 2];
#pragma unroll
            for (int c = 0; c < GE::CHUNKS / 2; ++c) cw[c] = lds128(rec + (uint32_t)((c0 + c) * TM + r) * 16u);
#pragma unroll
            for (int c = 0; c < GE::CHUNKS / 2; ++c) {
                uint32_t o[16];
                expand_word(cw[c].x, o);
                expand_word(cw[c].y, o + 4);
                expand_word(cw[c].z, o + 8);
                expand_word(cw[c].w, o + 12);
                tmem_st16(tl + (uint32_t)(ra.slot * GE::ACOLS + (c0 + c) * 16), o);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm->afull[ra.slot]);
                mbar_arrive(&sm->empty[rs.slot]);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------ promotion (row 32 (warp - 4) + lane)
        const int q4 = warp & 3, r = q4 * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        // outputs and partial sums may still be read by the previous kernel on the stream
        if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
        float acc[TN];
#pragma unroll
        for (int m = 0; m < TN; ++m) acc[m] = 0.0f;
        Ring<GE::NS> rs;
        Ring<GE::NACC> rb;
        int64_t t = t0;          // tile of the current unit
        int kb = kb0, seg_kb = kb0;  // its k-block, and the first k-block of the current segment
        bool ok = true;
        for (int i = 0; i < n_units && ok; ++i, rs.next()) {
            if (!warp_wait(&sm->full[rs.slot], rs.phase, sm, a.status)) break;
            const uint32_t scb = smem_addr(base + (size_t)rs.slot * GE::STAGE + GE::XB + GE::CODE_BYTES);
            uint32_t sc[GE::GPS];
#pragma unroll
            for (int gg = 0; gg < GE::GPS; ++gg) sc[gg] = lds32(scb + (uint32_t)(gg * TM + r) * 4u);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->empty[rs.slot]);
#pragma unroll
            for (int gg = 0; gg < GE::GPS; ++gg, rb.next()) {
                if (!warp_wait(&sm->accf[rb.slot], rb.phase, sm, a.status)) { ok = false; break; }
                tc_fence_after();
                uint32_t v[16];
                tmem_ld16(tl + (uint32_t)(GE::COL_ACC + rb.slot * TN), v);
                float X[TN];
                const float4 *xq = reinterpret_cast<const float4 *>(sm->xs[rb.slot]);
#pragma unroll
                for (int q = 0; q < TN / 4; ++q) {
                    const float4 f = xq[q];
                    X[4 * q] = f.x;
                    X[4 * q + 1] = f.y;
                    X[4 * q + 2] = f.z;
                    X[4 * q + 3] = f.w;
                }
                tmem_wait_ld(v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->acce[rb.slot]);
                const float s = __half2float(__ushort_as_half((unsigned short)(sc[gg] & 0xFFFFu)));
                const float zf = (float)((int)(int16_t)(sc[gg] >> 16) - 8);
#pragma unroll
                for (int m = 0; m < TN; ++m) acc[m] = fmaf(s, fmaf(-zf, X[m], __uint_as_float(v[m])), acc[m]);
            }
            if (!ok) break;
            if (i + 1 < n_units && kb + 1 < a.NKB) {
                ++kb;
                continue;
            }
            // ---- end of a segment (this CTA's run of units of one tile)
            const int64_t n = t * TM + r;
            if (seg_kb == 0 && kb + 1 == a.NKB) {
                store_row(a, n, acc);  // the whole tile's K range
            } else {
                const int which = t == t0 ? 0 : 1;  // a CTA's first segment, or its last
                float4 *dst = reinterpret_cast<float4 *>(a.part + (((size_t)blockIdx.x * 2 + which) * TM + r) * TN);
#pragma unroll
                for (int q = 0; q < TN / 4; ++q)
                    if (q < a.mw) dst[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
                __threadfence();
                __syncwarp();
                const int64_t cf = unit_owner(t * a.NKB, a.L, P), cl = unit_owner(t * a.NKB + a.NKB - 1, a.L, P);
                uint32_t old = 0;
                if (lane == 0) old = atomicAdd(a.cnt + t * 4 + q4, 1u);
                old = __shfl_sync(FULL, old, 0);
                if (old == (uint32_t)(cl - cf)) {
                    // last of the tile's CTAs for these 32 rows: add the parts in CTA order. CTA
                    // cf holds the tile's first unit: the tile is its first segment only if it
                    // starts there; every later CTA of the tile starts inside it (first segment).
                    __threadfence();
                    const int w_first = unit_begin(cf, a.L, P) == t * a.NKB ? 0 : 1;
                    float sum[TN];
#pragma unroll
                    for (int m = 0; m < TN; ++m) sum[m] = 0.0f;
                    switch (a.mw) {
                        case 1: reduce_parts<1>(a, r, cf, cl, w_first, sum); break;
                        case 2: reduce_parts<2>(a, r, cf, cl, w_first, sum); break;
                        case 3: reduce_parts<3>(a, r, cf, cl, w_first, sum); break;
                        default: reduce_parts<4>(a, r, cf, cl, w_first, sum); break;
                    }
                    store_row(a, n, sum);
                    if (lane == 0) a.cnt[t * 4 + q4] = 0u;  // ready for the next call
                }
            }
#pragma unroll
            for (int m = 0; m < TN; ++m) acc[m] = 0.0f;
            ++t;
            kb = 0;
            seg_kb = 0;
        }
    } else if (warp == 10) {
        // ------------------------------------------------ group sums X_j of the activation rows
        Ring<GE::NS> rs;
        Ring<GE::NACC> rb;
        const int tr = lane & 15, h = lane >> 4;
        for (int i = 0; i < n_units; ++i, rs.next()) {
            if (!warp_wait(&sm->full[rs.slot], rs.phase, sm, a.status)) break;
            // row tr: this half-warp's half of the stage's k, read from the 128-byte-swizzled
            // tile (16-byte chunk c of row t of a 64-k atom sits at chunk c ^ (t & 7)), summed
            // in k order per group; a group wider than half a stage is completed with the other
            // half's sum
            float xsum[GE::XPL];
#pragma unroll
            for (int j = 0; j < GE::XPL; ++j) xsum[j] = 0.0f;
            if (a.asym) {
                const uint32_t xb = smem_addr(base + (size_t)rs.slot * GE::STAGE);
#pragma unroll
                for (int c = 0; c < GE::HALF / 8; ++c) {   // 8 k per chunk
                    const int kin = h * GE::HALF + 8 * c;   // k of the chunk within the stage
                    const uint4 v = lds128(xb + (uint32_t)((kin >> 6) * (TN * 128) + tr * 128 + ((((kin >> 3) & 7) ^ (tr & 7)) << 4)));
                    const int j = GE::XPL > 1 ? (8 * c) / G : 0;
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) xsum[j] += __uint_as_float(w[q] << 16) + __uint_as_float(w[q] & 0xFFFF0000u);
                }
                if (G > GE::HALF) xsum[0] += __shfl_xor_sync(FULL, xsum[0], 16);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->empty[rs.slot]);
            bool ok = true;
#pragma unroll
            for (int gg = 0; gg < GE::GPS; ++gg, rb.next()) {
                if (!warp_wait(&sm->acce[rb.slot], rb.phase ^ 1u, sm, a.status)) { ok = false; break; }
                // group gg lies in half gg / XPL (register gg % XPL) when a group fits in a half
                const int hg = G <= GE::HALF ? gg / GE::XPL : 0;
                if (h == hg) sm->xs[rb.slot][tr] = xsum[G <= GE::HALF ? gg % GE::XPL : 0];
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->accf[rb.slot]);
            }
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(GE::TMEM_COLS) : "memory");
}

}  // namespace tc16
}  // namespace w4

// ------------------------------------------------------------------ host side

using namespace w4;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool tc_shape_ok(int64_t M, int64_t N, int64_t K) {
    return M >= 1 && M <= tc16::TN && N >= 1 && N <= (int64_t)1 << 31 && K >= 32 && K <= (int64_t)1 << 24 && K % 32 == 0;
}

int64_t tc_tiles(int64_t N) { return (N + tc16::TM - 1) / tc16::TM; }

// CTAs per 128-row tile at most: a tile shared by more CTAs finishes with a longer ordered
// reduction of their partial sums than the extra units per CTA cost.
constexpr int64_t kMaxPerTile = 8;

template <int G>
w4_status tc_start(const CUtensorMap &tm, const tc16::Args &a, int grid, cudaStream_t stream) {
    using GE = tc16::Geo<G>;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(tc16::w4a16_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)GE::SMEM_BYTES) != cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(tc16::THREADS);
    cfg.dynamicSmemBytes = GE::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = a.pdl;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, tc16::w4a16_tc_kernel<G>, tm, a) != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}

}  // namespace

W4_API size_t w4a16_gemm_tc_workspace_bytes(int64_t N, int64_t K, int group) {
    if (!tc_shape_ok(1, N, K) || !valid_group(group) || K % group != 0) return 0;
    const size_t parts = (size_t)num_sms() * 2 * tc16::TM * tc16::TN * 4;
    const size_t cnt = ((size_t)tc_tiles(N) * 4 * 4 + 15) / 16 * 16;
    return parts + cnt;
}

W4_API w4_status w4a16_gemm_tc_schedule(int64_t M, int64_t N, int64_t K, int group, int sms, int64_t *out) {
    if (!out) return W4_ERR_NULL;
    if (!tc_shape_ok(M, N, K) || sms < 1 || sms > 4096) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    const int ks = TcLayoutGeo::ks(group);
    const int64_t nkb = (K + ks - 1) / ks, T = tc_tiles(N), L = T * nkb;
    const int64_t gmax = T * kMaxPerTile < (int64_t)sms ? T * kMaxPerTile : (int64_t)sms;
    const int64_t grid = L < gmax ? L : gmax;
    out[0] = T;
    out[1] = nkb;
    out[2] = L;
    out[3] = grid;
    out[4] = ks;
    out[5] = (int64_t)TcLayoutGeo::record_bytes(group);
    return W4_OK;
}

W4_API w4_status w4a16_gemm_tc(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K, int group,
                               int mode, void *y, int flags, void *workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
    if (!x_bf16 || !packed || !y) return W4_ERR_NULL;
    if (!tc_shape_ok(M, N, K)) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!valid_mode(mode) || (flags & ~(W4_OUT_FP32 | W4_OVERLAP_PREVIOUS)) != 0) return W4_ERR_ARG;
    if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(y) || (workspace && !aligned16(workspace)))
        return W4_ERR_ALIGN;
    const size_t need = w4a16_gemm_tc_workspace_bytes(N, K, group);
    if (!workspace || workspace_bytes < need) return W4_ERR_WORKSPACE;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return W4_ERR_CUDA;

    const int ks = TcLayoutGeo::ks(group);
    const int64_t nkb = (K + ks - 1) / ks, T = tc_tiles(N), L = T * nkb;
    const int sms = num_sms();
    const int64_t gmax = T * kMaxPerTile < (int64_t)sms ? T * kMaxPerTile : (int64_t)sms;
    const int grid = (int)(L < gmax ? L : gmax);

    // bf16 [M][K]: boxes of 64 k (128 bytes) x 16 rows with the 128-byte swizzle (the MMA's
    // K-major layout); rows past M and k past K read as zero
    CUtensorMap tm;
    const bool x3d = K % 64 == 0;
    if (x3d) {
        // [K/64 atoms][M rows][64 k]: one box holds a whole stage (KS/64 atoms of 16 rows)
        const cuuint64_t dims[3] = {64, (cuuint64_t)M, (cuuint64_t)(K / 64)};
        const cuuint64_t strides[2] = {(cuuint64_t)K * 2, 128};
        const cuuint32_t box[3] = {64, (cuuint32_t)tc16::TN, (cuuint32_t)(ks / 64)};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(x_bf16), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    } else {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {64, (cuuint32_t)tc16::TN};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x_bf16), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }

    tc16::Args a;
    a.w = static_cast<const uint8_t *>(packed);
    a.y = y;
    a.part = static_cast<float *>(workspace);
    a.cnt = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) +
                                         (size_t)sms * 2 * tc16::TM * tc16::TN * 4);
    a.status = device_status_ptr();
    a.N = N;
    a.L = L;
    a.NKB = (int)nkb;
    a.M = (int)M;
    a.mw = (int)((M + 3) / 4);
    a.x3d = x3d ? 1 : 0;
    a.out_fp32 = (flags & W4_OUT_FP32) ? 1 : 0;
    a.asym = mode == W4_ASYM ? 1 : 0;
    a.pdl = (flags & W4_OVERLAP_PREVIOUS) ? 1 : 0;
    switch (group) {
        case 32: return tc_start<32>(tm, a, grid, stream);
        case 64: return tc_start<64>(tm, a, grid, stream);
        case 128: return tc_start<128>(tm, a, grid, stream);
        default: return tc_start<256>(tm, a, grid, stream);
    }
}
