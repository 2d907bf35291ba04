// w4a8_gemm / w4a8_grouped_gemm: INT4 weights x FP8 E4M3 activations on the sm_100a
// tensor cores (tcgen05.mma, TMEM accumulators, TMA operand loads).
//
// "Four-bit inference ... Tahoma", Achievement 2 (the W4A8 dataflow: packed 4-bit weights
// read from HBM, expanded to E4M3 inside the GEMM, FP8 tensor-core MMA with FP32
// accumulation, per-token activation scale in the epilogue, BF16 result) and
// "4-bit by default" (mixture-of-experts weights are the 4-bit target).
//
//   Y[m, n] = s_a[m] * ( sum_j 512 s[n,j] P_j[m,n]  -  Z[m,n] ),
//   P_j[m,n] = sum_{k in j} a8[m,k] * (q[n,k] * 2^-9),   Z[m,n] = sum_j s[n,j] z[n,j] G[m,j],
//   G[m,j] = sum_{k in j} a8[m,k]
//
// Design (one persistent CTA per SM, tiles of 128 weight rows x 256 tokens):
//  * swap-AB: the weight tile is the MMA's A operand (M = 128 weight rows, one TMEM lane per
//    weight row), 256 tokens are its N; each promotion thread owns one weight row, so the
//    group scale is a per-thread scalar;
//  * expansion: a nibble q in [0, 15] zero-extended to a byte IS the E4M3 pattern of q*2^-9
//    (exponent field 0/1 spans the integer grid m*2^-9, m = 0..15), so the expanded weights
//    are exact and the expansion is one AND (and one shift) per 4 weights, written straight
//    into the 128-byte-swizzled K-major layout the MMA reads;
//  * per group j, kind::f8f6f4 MMAs (K = 32 each) accumulate P_j into one of two TMEM
//    buffers (2 x 256 columns); 8 promotion warps read it back (tcgen05.ld) and add
//    512 s[n,j] P_j into fp32 registers (packed f32x2 FMAs) while the MMA fills the other;
//  * the zero-point term Z is a rank-J product computed on the tensor cores as well: after a
//    tile's last group, pseudo-stages bring bf16 hi/lo splits of s*z (from the prepacked
//    weight) and of G (from the row quantizer) by TMA -- [hi|hi|lo] x [hi|lo|hi] along K,
//    error ~2^-16 relative -- and kind::f16 MMAs accumulate Z into a TMEM buffer that the
//    promotion warps subtract as one more "group";
//  * warp roles: warp 0 TMA producer, warp 1 TMEM owner + single-thread MMA issuer, warps
//    4-11 promotion/epilogue (register budget raised with setmaxnreg), warps 12-15
//    expansion; one ring of 4 stages, each with raw operands (codes + activations, or the
//    two zero-point operands) and an expanded-weight buffer: TMA -> full -> expansion ->
//    exp_full -> MMA -> empty -> TMA. Every stage passes the expansion warps, so each wait
//    on the ring sees its phases in order, and the MMA thread has one wait and one commit
//    per stage (plus one of each per accumulator group);
//  * every mbarrier wait is bounded by wall-clock time; on expiry the kernel records
//    W4_ERR_TIMEOUT, every role sees the abort flag, TMEM is freed and the CTA returns;
//  * w4a8_gemm_rowquant runs the same kernel from bf16 activations (FUSE): its blocks
//    quantize the rows into the workspace first (staged through the ring) and, for short
//    rows, partly while the tiles run (warps 2-3); the producer and the epilogue read a
//    token tile's rows only after its row count is complete.
#include "w4_common.cuh"
#include "w4_layout.cuh"
#include "w4_rowquant.cuh"

#include <cuda.h>

namespace w4 {
namespace gemm {

constexpr int BM = 128;       // weight rows per tile (MMA M)
constexpr int BN = 256;       // tokens per tile (MMA N)
constexpr int BK = 128;       // k per pipeline stage (one 128-byte swizzle row of E4M3)
constexpr int STAGES = 4;     // pipeline stages (raw operands + one expanded-weight buffer each)
constexpr int NBUF = 2;       // TMEM accumulator buffers
constexpr int TMEM_COLS = NBUF * BN;
constexpr int THREADS = 512;
constexpr int ZKC = 32;       // bf16 columns of the zero-point operands per pseudo-stage (64-byte rows)
constexpr uint32_t C_BYTES = BM * BK / 2;   // packed codes of a stage
constexpr uint32_t B_BYTES = BN * BK;       // activations of a stage
constexpr uint32_t RAW_BYTES = C_BYTES + B_BYTES;
constexpr uint32_t ZA_BYTES = BM * ZKC * 2;  // s*z operand of a pseudo-stage (in place of the codes)
constexpr uint32_t ZB_BYTES = BN * ZKC * 2;  // group-sum operand of a pseudo-stage
constexpr uint32_t A_BYTES = BM * BK;       // expanded weights
constexpr uint32_t SMEM_BYTES = STAGES * (RAW_BYTES + A_BYTES) + 1024 /*control*/ + 1024 /*alignment*/;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait
static_assert(ZA_BYTES <= C_BYTES && C_BYTES + ZB_BYTES <= RAW_BYTES, "pseudo-stage operands fit a raw stage");
static_assert(RAW_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle atoms stay aligned");

struct Smem {
    uint64_t full[STAGES];     // raw operands landed (TMA bytes); waited by the expansion warps
    uint64_t exp_full[STAGES]; // expansion warps passed the stage (one arrival per warp); waited by the MMA
    uint64_t empty[STAGES];    // stage consumed by the MMA: raw and expanded buffers free again
    uint64_t acc_full[NBUF];   // a group's accumulator is complete in TMEM
    uint64_t acc_empty[NBUF];  // promotion finished reading it (one arrival per warp)
    uint32_t tmem_base;
    int abort;
    // the row quant of the kernel variant that quantizes its own activation rows, before the
    // ring is in use: two halves of row slots in the ring, each completed by one barrier, and
    // the row maxima (magnitude bits, by atomicMax) of the batches of each parity
    uint64_t rq_full[2];
    uint32_t rq_mb[2][16];
};
static_assert(sizeof(Smem) <= 1024, "control block");
constexpr uint32_t RING_BYTES = STAGES * (RAW_BYTES + A_BYTES);  // ring data bytes (row slots before the GEMM)
constexpr int RQ_MAX_SLOTS = 32;

struct Args {
    const uint8_t *packed;         // slab 0
    size_t slab_bytes;             // bytes per expert slab
    size_t codes_bytes;            // codes part of a slab (scales follow)
    const float *row_scale;        // [M_total]
    const int32_t *offsets;        // [E+1] device, or null: one problem of M rows
    void *Y;                       // [M_total, N]
    int *status;
    int64_t M, N, Npad, K, Kpad;
    int E, g, out_fp32;
    int NT;                        // weight tiles (Npad / BM)
    int MTU;                       // token tiles (upper bound for grouped problems)
    int KT;                        // raw stages per tile
    int ZT;                        // zero-point pseudo-stages per tile
    int64_t DPT;                   // tiles [0, DPT) are whole-tile work, strided over the grid
    int64_t R;                     // tiles [DPT, DPT + R) are split along K over PS CTAs
    int64_t PS;
    float *part;                   // split tiles: 2 PS partial-result slots (PART_FLOATS each)
    uint32_t *cnt;                 // split tiles: R x 8 arrival counters (zero between calls)
    // kernels that quantize their own activation rows (FUSE):
    const uint16_t *xq;            // bf16 activations [M, K]
    uint8_t *q8;                   // their E4M3 codes [M, K] (row_scale points at their scales)
    float *qscale;                 // row scales [M]
    uint16_t *qgop;                // group-sum operand [M, KZ]
    uint32_t *qcnt;                // per token tile: rows quantized so far (zero at launch)
    int64_t KZ;                    // columns of the group-sum operand
    int64_t qa1, qa2;              // rows [0, qa1) and [qa2, M) first, by every warp; the rest by warps 2-3
    int qstaged;                   // rows staged through the ring by bulk copies (rows of <= half the ring)
};

// ------------------------------------------------------------------ split-K schedule
// The last, partial wave of tiles is spread over the CTAs along K: its R tiles form R*KT
// k-blocks in tile-major order, and CTA c takes the contiguous range
// [c*Q/PS, (c+1)*Q/PS) of them (Q = R*KT). With R <= PS a range covers at most two tiles, so
// a CTA has at most two segments. The plan keeps PS <= Q/8, so no range is empty and the
// contributors of a tile are exactly the CTAs from the one holding its first k-block to the
// one holding its last. Each segment's fp32 partial sum goes to the CTA's slot
// 2c + (0 for the first segment, 1 for the second); the last contributor to arrive (per
// promotion warp, counted in the workspace) adds the partials of the tile in CTA order and
// stores the result, so the result does not depend on arrival order.
constexpr int PART_FLOATS = BM * BN;  // one slot: the 128 x 256 fp32 tile

__host__ __device__ __forceinline__ int64_t split_begin(int64_t Q, int64_t PS, int64_t c) { return c * Q / PS; }

// the CTA whose range holds k-block q: the largest c with split_begin(c) <= q
__host__ __device__ __forceinline__ int64_t split_cta_of(int64_t Q, int64_t PS, int64_t q) {
    return ((q + 1) * PS + Q - 1) / Q - 1;
}

// partial-result slot of contributor c to split tile i
__host__ __device__ __forceinline__ int64_t split_slot(int64_t Q, int64_t PS, int KT, int64_t c, int64_t i) {
    return 2 * c + (split_begin(Q, PS, c) / KT == i ? 0 : 1);
}

// the segment that starts at k-block q of a range ending at q1: split tile i, k-blocks
// [kb0, kb1) of it; returns the start of the next segment
__host__ __device__ __forceinline__ int64_t split_segment(int64_t q, int64_t q1, int KT, int64_t &i, int &kb0,
                                                          int &kb1) {
    i = q / KT;
    const int64_t e = (i + 1) * KT < q1 ? (i + 1) * KT : q1;
    kb0 = (int)(q - i * KT);
    kb1 = (int)(e - i * KT);
    return e;
}

__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    return mbar_wait_abortable(bar, parity, &sm->abort, status, kWaitNs);
}

// The wait of a single latency-critical thread (MMA issuer, TMA producer): polls without a
// suspend hint so that it resumes as soon as the phase completes.
__device__ __forceinline__ bool wait_phase_short(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    return mbar_wait_abortable<true>(bar, parity, &sm->abort, status, kWaitNs);
}

// Position in a ring of STAGES slots: slot and the parity of the current use of that slot.
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next() {
        if (++slot == STAGES) { slot = 0; phase ^= 1u; }
    }
};

// The same wait taken by a whole warp, with one outcome for all its lanes (the warp then runs
// warp-collective instructions, which need every lane). Only lane 0 polls, so that twelve
// waiting warps do not flood the barrier unit that the MMA thread also uses; once lane 0 has
// seen the phase complete, every lane takes one try_wait of its own for the acquire. That try
// cannot fail: the barrier's next phase needs this warp's own later arrival (or work that
// waits for it).
__device__ __forceinline__ bool warp_wait_phase(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    bool r = true;
    if ((threadIdx.x & 31) == 0) r = wait_phase(bar, parity, sm, status);
    r = __shfl_sync(FULL, r ? 1 : 0, 0) != 0;
    if (r) r = __all_sync(FULL, mbar_try_wait_short(bar, parity));
    return r;
}

// The same with lane 0 polling without a suspend hint, for the promotion warps' wait on a
// finished accumulator: it resumes as soon as the MMA's commit lands, which matters most
// when every MMA ends a group (group size 32).
__device__ __forceinline__ bool warp_wait_phase_short(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    bool r = true;
    if ((threadIdx.x & 31) == 0) r = wait_phase_short(bar, parity, sm, status);
    r = __shfl_sync(FULL, r ? 1 : 0, 0) != 0;
    if (r) r = __all_sync(FULL, mbar_try_wait_short(bar, parity));
    return r;
}

// Shared-memory operand descriptors (K-major), kept as two 32-bit words so that the MMA
// thread only does 32-bit adds: the low word holds the start address in 16-byte units
// (bits 0-13) and the leading byte offset 16 bytes (bits 16-29, unused by swizzled K-major
// operands whose K extent fits one swizzle row); the high word holds the stride byte offset
// between 8-row atoms (bits 32-45), descriptor version 1 (bit 46) and the swizzle mode
// (bits 61-63: 2 = 128-byte, 4 = 64-byte). Advancing K by 32 bytes adds 2 to the low word.
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr) { return ((saddr & 0x3FFFFu) >> 4) | (1u << 16); }
constexpr uint32_t kDescHiSW128 = 64u | (1u << 14) | (2u << 29);  // rows of 128 bytes, atoms 1024 bytes apart
constexpr uint32_t kDescHiSW64 = 32u | (1u << 14) | (4u << 29);   // rows of 64 bytes, atoms 512 bytes apart

// instruction descriptors: D fp32, both operands K-major, N = BN, M = BM;
// A/B E4M3 (kind::f8f6f4) or BF16 (kind::f16)
constexpr uint32_t kIdescF8 = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescBF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// D[tmem_d] (+)= A * B for one K step; the descriptors are given as (low word, shared high word)
__device__ __forceinline__ void mma_f8(uint32_t tmem_d, uint32_t a_lo, uint32_t b_lo, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n .reg .b64 da, db;\n setp.ne.b32 p, %4, 0;\n"
        " mov.b64 da, {%1, %5};\n mov.b64 db, {%2, %5};\n"
        " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %3, p;\n}\n" ::"r"(tmem_d),
        "r"(a_lo), "r"(b_lo), "r"(kIdescF8), "r"(accumulate), "r"(kDescHiSW128));
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint32_t a_lo, uint32_t b_lo, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n .reg .b64 da, db;\n setp.ne.b32 p, %4, 0;\n"
        " mov.b64 da, {%1, %5};\n mov.b64 db, {%2, %5};\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n}\n" ::"r"(tmem_d),
        "r"(a_lo), "r"(b_lo), "r"(kIdescBF16), "r"(accumulate), "r"(kDescHiSW64));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 16 columns of 32-bit accumulator (one column per register)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Wait for this thread's tcgen05.ld. The registers of the load are in/out operands, so the
// compiler cannot move a use of them above the wait.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

// 32 lanes x 16 columns of 32-bit values from registers into TMEM (one column per register)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float2 *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "f"(v[0].x), "f"(v[0].y), "f"(v[1].x), "f"(v[1].y), "f"(v[2].x), "f"(v[2].y), "f"(v[3].x), "f"(v[3].y),
        "f"(v[4].x), "f"(v[4].y), "f"(v[5].x), "f"(v[5].y), "f"(v[6].x), "f"(v[6].y), "f"(v[7].x), "f"(v[7].y)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Transpose 8x8 blocks of 16-bit values held by each aligned group of 8 lanes: lane l holds
// row l as R[k] = (col 2k, col 2k+1); afterwards it holds column l as R[k] = (row 2k, row 2k+1).
// Butterfly stages over lane distance 4 and 2 swap 32-bit pairs; distance 1 swaps halves.
__device__ __forceinline__ void transpose8x8_b16(uint32_t (&R)[4], int lane) {
    const int l = lane & 7;
#pragma unroll
    for (int p = 0; p < 2; ++p) {  // distance 4: registers (0, 2) and (1, 3)
        const bool up = (l & 4) != 0;
        const uint32_t recv = __shfl_xor_sync(FULL, up ? R[p] : R[p + 2], 4);
        if (up) R[p] = recv;
        else R[p + 2] = recv;
    }
#pragma unroll
    for (int p = 0; p < 4; p += 2) {  // distance 2: registers (0, 1) and (2, 3)
        const bool up = (l & 2) != 0;
        const uint32_t recv = __shfl_xor_sync(FULL, up ? R[p] : R[p + 1], 2);
        if (up) R[p] = recv;
        else R[p + 1] = recv;
    }
    const bool odd = (l & 1) != 0;
#pragma unroll
    for (int p = 0; p < 4; p += 2) {  // distance 1: 16-bit halves of registers (p, p + 1)
        const uint32_t recv = __shfl_xor_sync(FULL, __byte_perm(R[p], R[p + 1], odd ? 0x5410 : 0x7632), 1);
        const uint32_t a = __byte_perm(odd ? recv : R[p], odd ? R[p] : recv, odd ? 0x7610 : 0x5410);
        const uint32_t b = __byte_perm(odd ? recv : R[p + 1], odd ? R[p + 1] : recv, odd ? 0x7632 : 0x7610);
        R[p] = a;
        R[p + 1] = b;
    }
}

// acc[i] += s * (p[2i], p[2i+1]) with the packed fp32 FMA of sm_100 (two lanes per instruction)
__device__ __forceinline__ void promote16(float2 *acc, float2 s, const uint32_t (&p)[16]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
        acc[i] = __ffma2_rn(s, make_float2(__uint_as_float(p[2 * i]), __uint_as_float(p[2 * i + 1])), acc[i]);
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

struct Tile {
    int e;          // expert
    int64_t row0;   // first token row
    int64_t rows;   // token rows that belong to this tile's problem (may exceed BN)
    int64_t n0;     // first weight row
};

// Tile t -> (token tile, weight tile) with the weight tile fastest, so that CTAs running at
// the same time share a token tile and walk one expert's weight; false if t names no tile.
__device__ __forceinline__ bool locate_tile(const Args &a, int64_t t, Tile &T) {
    const int64_t mt = t / a.NT;
    const int64_t nt = t - mt * a.NT;
    T.n0 = nt * BM;
    if (!a.offsets) {
        T.e = 0;
        T.row0 = mt * BN;
        T.rows = a.M - T.row0;
        return T.row0 < a.M;
    }
    int64_t cum = 0;
    for (int x = 0; x < a.E; ++x) {
        const int64_t lo = a.offsets[x], hi = a.offsets[x + 1];
        const int64_t tiles = (hi - lo + BN - 1) / BN;
        if (mt < cum + tiles) {
            T.e = x;
            T.row0 = lo + (mt - cum) * BN;
            T.rows = hi - T.row0;
            return true;
        }
        cum += tiles;
    }
    return false;
}

// One unit of a CTA's work: k-blocks [kb0, kb1) of tile t, followed by the zero-point
// pseudo-stages when z. seg < 0: a whole tile, stored directly; otherwise the ordinal (0 or 1)
// of a split-tile segment in this CTA's range.
struct Item {
    int64_t t;
    int kb0, kb1;
    int seg;
    bool z;
};

// The sequence of items of this CTA, identical for every role: its split-tile segments first
// (so that the combine step of a split tile, which only the last contributor runs, overlaps
// the next whole tile's first stages), then its whole tiles.
struct Work {
    int64_t t, q, q1;
    int seg = 0;
    __device__ __forceinline__ explicit Work(const Args &a) {
        t = blockIdx.x;
        const int64_t Q = a.R * a.KT;
        q = blockIdx.x < a.PS ? split_begin(Q, a.PS, blockIdx.x) : 0;
        q1 = blockIdx.x < a.PS ? split_begin(Q, a.PS, blockIdx.x + 1) : 0;
    }
    __device__ __forceinline__ bool next(const Args &a, Item &it) {
        if (q < q1) {
            int64_t i;
            q = split_segment(q, q1, a.KT, i, it.kb0, it.kb1);
            it.t = a.DPT + i;
            it.seg = seg++;
            it.z = it.kb1 == a.KT;  // the segment that ends the tile also adds its zero-point term
            return true;
        }
        if (t < a.DPT) {
            it.t = t;
            it.kb0 = 0;
            it.kb1 = a.KT;
            it.seg = -1;
            it.z = true;
            t += gridDim.x;
            return true;
        }
        return false;
    }
};

// Split tile, promotion warp wq (weight rows 32*(wq&3).., token columns 128*(wq>>2)..), whose
// partial sum is in TMEM at taddr (32 lanes x 128 columns): store it in the CTA's slot and
// count it. The warp whose arrival completes the count adds every contributor's partial of its
// part, in CTA order, into TMEM at taddr, resets the counter for the next call and returns
// true; the others return false. Kept out of line and working through TMEM so that the
// promotion loop's code and registers are those of a kernel without split tiles.
// Slot layout: [8 warps][32 column quads][32 lanes] float4, so that each store or load of a
// warp covers 512 contiguous bytes.
// Arguments are passed as scalars (no reference to the kernel's parameter block, which would
// need a local copy of it).
__device__ __noinline__ bool split_combine(float *part_base, uint32_t *cnt, int *status, int64_t R, int KT,
                                           int64_t PS, int64_t i, int seg, int wq, uint32_t taddr) {
    const int lane = threadIdx.x & 31;
    const int64_t Q = R * KT, me = blockIdx.x;
    const int64_t c0 = split_cta_of(Q, PS, i * KT), c1 = split_cta_of(Q, PS, i * KT + KT - 1);
    const int64_t slot = 2 * me + seg;
    if (i < 0 || i >= R || c0 < 0 || me < c0 || me > c1 || c1 >= PS || split_slot(Q, PS, KT, me, i) != slot) {
        if (lane == 0) record_status(status, W4_ERR_DEVICE_CHECK);
        return false;
    }
    float4 *part = reinterpret_cast<float4 *>(part_base) + wq * 1024 + lane;  // + slot * 8192
    {
        float4 *mine = part + slot * 8192;
        uint32_t v[16];
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {  // 16 columns: float4 quads 4c .. 4c+3
            tmem_ld16(taddr + c * 16, v);
            tmem_wait_ld16(v);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                __stcg(mine + (4 * c + q) * 32, make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
        }
    }
    __threadfence();
    __syncwarp();
    uint32_t *ctr = cnt + i * 8 + wq;
    uint32_t old = 0;
    if (lane == 0) old = atomicAdd(ctr, 1u);
    old = __shfl_sync(FULL, old, 0);
    if (old != (uint32_t)(c1 - c0)) return false;
    __threadfence();
    // 64 columns (16 quads) at a time: the first contributor's quads, then each later one's
    // added in CTA order, then the sums into TMEM
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
        float4 sum[16];
        const float4 *src = part + split_slot(Q, PS, KT, c0, i) * 8192 + h * 16 * 32;
#pragma unroll
        for (int k = 0; k < 16; ++k) sum[k] = __ldcg(src + k * 32);
#pragma unroll 1
        for (int64_t c = c0 + 1; c <= c1; ++c) {
            src = part + split_slot(Q, PS, KT, c, i) * 8192 + h * 16 * 32;
            float4 v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = __ldcg(src + k * 32);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                sum[k].x += v[k].x;
                sum[k].y += v[k].y;
                sum[k].z += v[k].z;
                sum[k].w += v[k].w;
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st16(taddr + (4 * h + c) * 16, reinterpret_cast<const float2 *>(sum + 4 * c));
    }
    tmem_wait_st();
    if (lane == 0) atomicExch(ctr, 0u);
    return true;
}

// ------------------------------------------------------------------ row quant inside the GEMM
// The kernel variant that takes bf16 activations quantizes every activation row itself
// ("Four-bit inference ... Tahoma", Achievement 2: the per-token scale is recomputed on every
// forward pass) into the workspace -- E4M3 codes, row scale, group-sum operand, the same
// values as fp8_row_quant bit for bit -- and the tiles then read those rows like the
// operands of the two-launch path. Rows are either staged through the still-empty ring by
// bulk copies (quant_rows_staged, before the GEMM's roles start) or streamed by one warp per
// row (quant_row_warp: the max over the row's magnitude bits, the row scale and its
// reciprocal, then a second pass over the row from L2 that converts, stores the codes and
// adds each group's codes exactly as integers in units of 2^-9; used while the GEMM runs and
// for rows too long for the ring). A finished row is counted in its token tile's counter by a release add
// after a proxy fence, so that the TMA (async proxy) loads issued after an acquire load of a
// full count see it. The readers use acquire loads, not fences: a gpu-scope fence would wait
// for the reader's own earlier stores (the previous tile's outputs) to drain.
__device__ __forceinline__ void red_release_add(uint32_t *p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait until the counter at p reaches n (acquire); on expiry records W4_ERR_TIMEOUT
// and raises the CTA's abort flag.
__device__ __forceinline__ bool count_reached(const uint32_t *p, uint32_t n, Smem *sm, int *status) {
    if (ld_acquire(p) >= n) return true;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(p) < n) {
        if (*(volatile int *)&sm->abort) return false;
        if (globaltimer_ns() - t0 > kWaitNs) {
            *(volatile int *)&sm->abort = 1;
            record_status(status, W4_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(128);
    }
    return true;
}

template <int G>
__device__ __forceinline__ void quant_row_warp(const uint16_t *__restrict__ xq, int64_t K, int64_t KZ, int64_t m,
                                               int64_t next, int64_t next2, uint8_t *q8, float *qscale,
                                               uint16_t *qgop, uint32_t *qcnt) {
    const int lane = threadIdx.x & 31;
    const int64_t nchunk = K / 8, J = K / G;
    const uint4 *src = reinterpret_cast<const uint4 *>(xq + m * K);
    // the warp's next rows into L2 while this one is worked on (a warp holds few loads in flight)
    if (lane == 0 && next >= 0) bulk_prefetch_l2(xq + next * K, (uint32_t)(K * 2));
    if (lane == 0 && next2 >= 0) bulk_prefetch_l2(xq + next2 * K, (uint32_t)(K * 2));
    // pass 1: max over the magnitude bits, eight 16-byte loads per lane in flight
    // (every loop below runs the same trip count on every lane: the group sums are warp
    // shuffles over all 32 lanes)
    uint32_t mb = 0;
    for (int64_t b = 0; b < nchunk; b += 32 * 8) {
        const int64_t c0 = b + lane;
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = c0 + 32 * u < nchunk ? __ldg(src + c0 + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 8; ++u) mb = absmax_bits(mb, v[u]);
    }
    mb = __reduce_max_sync(FULL, __vmaxu2(mb, mb >> 16) & 0xFFFFu);
    const bool special = mb >= 0x7F80u;  // an infinity or a NaN in the row
    float amax = __uint_as_float(mb << 16);
    if (mb > 0x7F80u) {  // NaN: the maximum of the other values (non-negative floats order as bits)
        float x = 0.0f;
        for (int64_t c = lane; c < nchunk; c += 32) x = absmax_float(x, __ldg(src + c));
        amax = __uint_as_float(__reduce_max_sync(FULL, __float_as_uint(x)));
    }
    const float s = scale_of(amax);
    const float r = __frcp_rn(s);
    if (lane == 0) qscale[m] = s;
    uint2 *dst = reinterpret_cast<uint2 *>(q8 + m * K);
    uint16_t *gop = qgop + m * KZ;
    // pass 2 (from L2), four rounds of 32 chunks per iteration with their loads issued first;
    // a group's G / 8 chunks sit on consecutive lanes of one round (32 * 8 is a multiple of G),
    // so its sum is a butterfly over those lanes
    for (int64_t b = 0; b < nchunk; b += 32 * 4) {
        const int64_t c0 = b + lane;
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = c0 + 32 * u < nchunk ? __ldg(src + c0 + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t c = c0 + 32 * u;
            const bool live = c < nchunk;
            int isum = 0;
            if (live) {
                const uint2 o = special ? quantize8<true>(v[u], s, r) : quantize8<false>(v[u], s, r);
                dst[c] = o;
                isum = e4m3x8_sum_times512(o.x, o.y);
            }
#pragma unroll
            for (int off = 1; off < G / 8; off <<= 1) isum += __shfl_xor_sync(FULL, isum, off);
            if (live && (lane & (G / 8 - 1)) == 0) {
                const float gs = __fmul_rn(__int2float_rn(isum), 0.001953125f);
                const uint16_t hi = bf16_rn_bits(gs);
                const int64_t j = (c * 8) / G;
                gop[j] = hi;
                gop[J + j] = bf16_rn_bits(__fsub_rn(gs, __uint_as_float((uint32_t)hi << 16)));
                gop[2 * J + j] = hi;
            }
        }
    }
    for (int64_t t = 3 * J + lane; t < KZ; t += 32) gop[t] = 0;
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __threadfence();
    __syncwarp();
    if (lane == 0) red_release_add(qcnt + m / BN, 1u);
}

// The rows [0, qa1) and [qa2, M) quantized by the CTAs before the GEMM's roles start, staged
// through the (still unused) ring: the CTA's rows (index i = blockIdx.x + k * gridDim.x of that
// row set) go by batches of h rows into one half of the ring's row slots by bulk copies, while
// the other half's batch is worked on, so HBM streams the rows at full rate instead of one
// warp's loads in flight at a time. Two block barriers per batch:
//  1. after the batch's rows landed -- it also ends the previous batch: that batch's rows are
//     counted in their token tiles (one gpu-scope fence, cumulative over the block's stores,
//     then release adds), its half of the slots is refilled with the next batch, and the row
//     maxima of the next parity are cleared;
//  2. after all 16 warps took the rows' maxima by rounds of 32 chunks (combined per row in
//     shared memory).
// Then every warp forms each row's scale from its maximum and converts rounds of 32 chunks
// (a round holds whole groups, whose sums are warp butterflies), storing codes and group-sum
// operand, and fences its stores for the async proxy. Returns false (every thread alike) if a
// bulk copy did not land in time.
template <int G>
__device__ __forceinline__ bool quant_rows_staged(const Args &a, uint8_t *ring, Smem *sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t K = a.K, nchunk = K / 8, J = K / G;
    const uint32_t row_bytes = (uint32_t)(K * 2);
    int nslots = (int)(RING_BYTES / row_bytes);
    if (nslots > RQ_MAX_SLOTS) nslots = RQ_MAX_SLOTS;
    const int h = nslots / 2;  // rows per batch (>= 1: the host stages only rows of <= half the ring)
    const int64_t nA1 = a.qa1, nA = a.qa1 + (a.M - a.qa2);  // the row set: [0, qa1) then [qa2, M)
    const int64_t nr = blockIdx.x < nA ? (nA - 1 - blockIdx.x) / gridDim.x + 1 : 0;  // rows of this CTA
    const int64_t nb = (nr + h - 1) / h;
    auto row_of = [&](int64_t k) {  // the CTA's k-th row
        const int64_t i = blockIdx.x + k * (int64_t)gridDim.x;
        return i < nA1 ? i : a.qa2 + (i - nA1);
    };
    auto batch_rows = [&](int64_t b) { return (int)(nr - b * h < h ? nr - b * h : h); };
    auto issue = [&](int64_t b) {  // thread 0: batch b into half b & 1
        const int half = (int)(b & 1), n = batch_rows(b);
        mbar_arrive_expect_tx(&sm->rq_full[half], (uint32_t)n * row_bytes);
        for (int i = 0; i < n; ++i) {
            const int64_t m = row_of(b * h + i);
            bulk_g2s(ring + (size_t)(half * h + i) * row_bytes, a.xq + m * K, row_bytes, &sm->rq_full[half]);
        }
    };
    if (threadIdx.x == 0) {
        mbar_init(&sm->rq_full[0], 1);
        mbar_init(&sm->rq_full[1], 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) sm->rq_mb[threadIdx.x >> 4][threadIdx.x & 15] = 0u;
    __syncthreads();
    if (threadIdx.x == 0) {
        if (nb > 0) issue(0);
        if (nb > 1) issue(1);
    }
    bool ok = true;
    for (int64_t b = 0; b <= nb; ++b) {  // the pass with b == nb only ends batch nb - 1
        const int half = (int)(b & 1);
        bool got = true;
        if (b < nb) {
            if (lane == 0) got = wait_phase(&sm->rq_full[half], (uint32_t)(b >> 1) & 1u, sm, a.status);
            got = __shfl_sync(FULL, got ? 1 : 0, 0) != 0;
            if (got) got = __all_sync(FULL, mbar_try_wait_short(&sm->rq_full[half], (uint32_t)(b >> 1) & 1u));
        }
        ok = __syncthreads_and(got ? 1 : 0) != 0;  // barrier 1
        if (!ok) break;
        if (b > 0) {
            // batch b - 1 is done by every warp: count its rows, refill its half
            const int np = batch_rows(b - 1);
            if (warp == 0) {
                if (lane == 0) __threadfence();
                __syncwarp();
                if (lane < np) red_release_add(a.qcnt + row_of((b - 1) * h + lane) / BN, 1u);
            }
            if (threadIdx.x == 0 && b + 1 < nb) issue(b + 1);
        }
        if (b == nb) break;
        // the maxima of the next batch (last read by batch b - 1, before barrier 1)
        if (threadIdx.x < 16) sm->rq_mb[half ^ 1][threadIdx.x] = 0u;
        const int n = batch_rows(b);
        const uint8_t *slots = ring + (size_t)half * h * row_bytes;
        uint32_t *mbs = sm->rq_mb[half];
        // max over each row's magnitude bits: each row's rounds of 32 chunks spread over the 16
        // warps (row outer, round inner: warp-uniform trip counts, no division)
        for (int i = 0; i < n; ++i) {
            const uint4 *src = reinterpret_cast<const uint4 *>(slots + (size_t)i * row_bytes);
            uint32_t mb = 0;
            for (int64_t c0 = (int64_t)warp * 32; c0 < nchunk; c0 += THREADS)
                if (c0 + lane < nchunk) mb = absmax_bits(mb, src[c0 + lane]);
            mb = __reduce_max_sync(FULL, __vmaxu2(mb, mb >> 16) & 0xFFFFu);
            if (lane == 0 && mb) atomicMax(&mbs[i], mb);
        }
        __syncthreads();  // barrier 2
        // scale, codes and group sums: each warp forms every row's scale from its maximum,
        // then converts its share of the row's rounds (a round holds whole groups)
        for (int i = 0; i < n; ++i) {
            const uint4 *src = reinterpret_cast<const uint4 *>(slots + (size_t)i * row_bytes);
            const int64_t m = row_of(b * h + i);
            const uint32_t mb = mbs[i];
            float amax = __uint_as_float(mb << 16);
            if (mb > 0x7F80u) {  // NaN: the maximum of the other values
                float x = 0.0f;
                for (int64_t c = lane; c < nchunk; c += 32) x = absmax_float(x, src[c]);
                amax = __uint_as_float(__reduce_max_sync(FULL, __float_as_uint(x)));
            }
            const float sc = scale_of(amax), rc = __frcp_rn(sc);
            const bool sp = mb >= 0x7F80u;  // an infinity or a NaN in the row
            uint16_t *gop = a.qgop + m * a.KZ;
            if (warp == (i & 15)) {  // the row's scale and the group-sum operand's zero padding
                if (lane == 0) a.qscale[m] = sc;
                for (int64_t t = 3 * J + lane; t < a.KZ; t += 32) gop[t] = 0;
            }
            uint2 *dst = reinterpret_cast<uint2 *>(a.q8 + m * K);
            for (int64_t c0 = (int64_t)warp * 32; c0 < nchunk; c0 += THREADS) {
                const int64_t c = c0 + lane;
                const bool live = c < nchunk;
                int isum = 0;
                if (live) {
                    const uint2 o = sp ? quantize8<true>(src[c], sc, rc) : quantize8<false>(src[c], sc, rc);
                    dst[c] = o;
                    isum = e4m3x8_sum_times512(o.x, o.y);
                }
#pragma unroll
                for (int off = 1; off < G / 8; off <<= 1) isum += __shfl_xor_sync(FULL, isum, off);
                if (live && (lane & (G / 8 - 1)) == 0) {
                    const float gs = __fmul_rn(__int2float_rn(isum), 0.001953125f);
                    const uint16_t hi = bf16_rn_bits(gs);
                    const int64_t j = (c * 8) / G;
                    gop[j] = hi;
                    gop[J + j] = bf16_rn_bits(__fsub_rn(gs, __uint_as_float((uint32_t)hi << 16)));
                    gop[2 * J + j] = hi;
                }
            }
        }
        // the batch's stores visible to the async proxy; this thread's reads of the slots
        // ordered before the bulk copies (async proxy) that refill them after barrier 1
        asm volatile("fence.proxy.async.global;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    return ok;
}

// The producer's wait for the rows of the token tile at row0 (n rows): then the async proxy's
// loads of them are ordered after the acquire.
__device__ __forceinline__ bool rows_ready(const uint32_t *qcnt, int64_t row0, int64_t n, Smem *sm, int *status) {
    if (!count_reached(qcnt + row0 / BN, (uint32_t)n, sm, status)) return false;
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
}

// A promotion lane's four row scales (token columns half * 128 + 32 c + lane of the tile at
// row0), written by this kernel: the tile's count acquired first (one acquire load per lane),
// the scales read through L2; columns past the tile's rows give 0. NaN in x when the wait ran
// out (kept out of line so that the promotion loop's registers are those of the two-launch
// kernel).
__device__ __noinline__ float4 fused_row_scales(const uint32_t *qcnt, const float *row_scale, int64_t row0,
                                                int64_t rows, int64_t M, int half, Smem *sm, int *status) {
    const int lane = threadIdx.x & 31;
    const int64_t n = M - row0 < (int64_t)BN ? M - row0 : (int64_t)BN;
    if (!count_reached(qcnt + row0 / BN, (uint32_t)n, sm, status))
        return make_float4(__int_as_float(0x7fffffff), 0.0f, 0.0f, 0.0f);
    float v[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int col = half * 128 + c * 32 + lane;
        const int64_t m = row0 + col;
        v[c] = (col < rows && m < M) ? __ldcg(row_scale + m) : 0.0f;
    }
    return make_float4(v[0], v[1], v[2], v[3]);
}

// group size: 32, 64 or 128; FUSE: the activation rows are quantized by this kernel
template <int G, bool FUSE>
__global__ void __launch_bounds__(THREADS, 1) w4a8_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                          const __grid_constant__ CUtensorMap tm_act,
                                                          const __grid_constant__ CUtensorMap tm_zop,
                                                          const __grid_constant__ CUtensorMap tm_gop, const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *raw = base;                                   // STAGES x (codes | activations)
    uint8_t *sA = base + STAGES * RAW_BYTES;               // STAGES x expanded weights
    Smem *sm = reinterpret_cast<Smem *>(base + STAGES * (RAW_BYTES + A_BYTES));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int GPS = BK / G;    // groups per raw stage
    constexpr int KPG = G / 32;    // f8 MMAs (K = 32 each) per group

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->exp_full[s], 4);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], 8);
        }
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sm->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;

    if (FUSE && a.qstaged) {
        // the first tiles' rows (or every row), staged through the ring before it holds any stage
        quant_rows_staged<G>(a, base, sm);
        __syncthreads();
    } else if (FUSE) {
        // the rows the first tiles of every CTA read, by every warp of the grid: [0, qa1)
        // (token tiles of the first wave of whole tiles) and [qa2, M) (token tiles of the
        // split tiles, which CTAs take first)
        // (CTA index fastest, so that the rows spread over every SM)
        const int64_t nA1 = a.qa1, nA = a.qa1 + (a.M - a.qa2), step = (int64_t)gridDim.x * (THREADS / 32);
        for (int64_t i = (int64_t)warp * gridDim.x + blockIdx.x; i < nA; i += step) {
            const int64_t in = i + step;
            quant_row_warp<G>(a.xq, a.K, a.KZ, i < nA1 ? i : a.qa2 + (i - nA1),
                              in < nA ? (in < nA1 ? in : a.qa2 + (in - nA1)) : -1, -1, a.q8, a.qscale, a.qgop,
                              a.qcnt);
        }
    }

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 64;\n" ::: "memory");
        if (FUSE && warp >= 2) {
            // ------------------------------------------------ row quant of the later token tiles
            // (warps 2 and 3 of every CTA, in row order, while the tiles of the first rows run;
            // these warps wait on nothing, so the rows always come out)
            const int64_t step = (int64_t)gridDim.x * 2;
            const int64_t m0 = a.qa1 + (int64_t)(warp - 2) * gridDim.x + blockIdx.x;
            if (lane == 0 && m0 < a.qa2) bulk_prefetch_l2(a.xq + m0 * a.K, (uint32_t)(a.K * 2));
            for (int64_t m = m0; m < a.qa2; m += step)
                quant_row_warp<G>(a.xq, a.K, a.KZ, m, m + step < a.qa2 ? m + step : -1,
                                  m + 2 * step < a.qa2 ? m + 2 * step : -1, a.q8, a.qscale, a.qgop, a.qcnt);
        } else if (warp == 0 && lane == 0) {
            // ------------------------------------------------ TMA producer
            Ring r;
            int64_t uses = 0;
            bool ok = true;
            int64_t ready_row0 = -1;  // FUSE: the token tile whose rows are known to be out
            Work w(a);
            Item it;
            while (ok && w.next(a, it)) {
                Tile T;
                if (!locate_tile(a, it.t, T)) continue;
                if (FUSE && T.row0 != ready_row0) {
                    const int64_t n = a.M - T.row0 < (int64_t)BN ? a.M - T.row0 : (int64_t)BN;
                    if (!rows_ready(a.qcnt, T.row0, n, sm, a.status)) { ok = false; continue; }
                    ready_row0 = T.row0;
                }
                const int send = it.kb1 + (it.z ? a.ZT : 0);
                for (int s = it.kb0; s < send; ++s, r.next(), ++uses) {
                    const int slot = r.slot;
                    if (!wait_phase_short(&sm->empty[slot], r.phase ^ 1u, sm, a.status)) { ok = false; break; }
                    uint8_t *dst = raw + slot * RAW_BYTES;
                    if (s < it.kb1) {
                        mbar_arrive_expect_tx(&sm->full[slot], C_BYTES + B_BYTES);
                        tma_load_3d(dst, &tm_codes, s * (BK / 2), (int)T.n0, T.e, &sm->full[slot]);
                        tma_load_2d(dst + C_BYTES, &tm_act, s * BK, (int)T.row0, &sm->full[slot]);
                    } else {
                        const int z = s - it.kb1;
                        mbar_arrive_expect_tx(&sm->full[slot], ZA_BYTES + ZB_BYTES);
                        tma_load_3d(dst, &tm_zop, z * ZKC, (int)T.n0, T.e, &sm->full[slot]);
                        tma_load_2d(dst + C_BYTES, &tm_gop, z * ZKC, (int)T.row0, &sm->full[slot]);
                    }
                }
            }
            // tail: wait for the completion of the last STAGES uses (use u: slot u % STAGES,
            // parity (u / STAGES) & 1), so no commit-arrive lands after this CTA exits
            for (int64_t u = uses > STAGES ? uses - STAGES : 0; u < uses && ok; ++u)
                if (!wait_phase(&sm->empty[u % STAGES], (uint32_t)(u / STAGES) & 1, sm, a.status)) break;
        } else if (warp == 1 && lane == 0) {
            // ------------------------------------------------ MMA issuer
            // One wait per stage (exp_full: the expansion warps have seen the TMA bytes land and
            // written the expanded weights) and one per accumulator group; one commit per stage
            // (empty: raw and expanded buffers free) and one per group (acc_full). This thread's
            // instruction stream sets the pace of the tensor core, so everything between MMAs is
            // kept to 32-bit arithmetic on precomputed descriptor words.
            Ring r;
            uint32_t jg = 0;
            bool ok = true;
            const uint32_t aLo0 = desc_lo(smem_addr(sA)), rLo0 = desc_lo(smem_addr(raw));
            Work w(a);
            Item it;
            while (ok && w.next(a, it)) {
                Tile T;
                if (!locate_tile(a, it.t, T)) continue;
                const int send = it.kb1 + (it.z ? a.ZT : 0);
                for (int s = it.kb0; s < send && ok; ++s, r.next()) {
                    const int slot = r.slot;
                    if (!wait_phase_short(&sm->exp_full[slot], r.phase, sm, a.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t rLo = rLo0 + (uint32_t)slot * (RAW_BYTES >> 4);
                    if (s < it.kb1) {
                        const uint32_t aLo = aLo0 + (uint32_t)slot * (A_BYTES >> 4), bLo = rLo + (C_BYTES >> 4);
#pragma unroll
                        for (int gi = 0; gi < GPS; ++gi, ++jg) {
                            const uint32_t b = jg & 1u;
                            if (!wait_phase_short(&sm->acc_empty[b], ((jg >> 1) & 1u) ^ 1u, sm, a.status)) { ok = false; break; }
                            tc_fence_after();
                            const uint32_t d = tmem + b * BN;
#pragma unroll
                            for (int kk = 0; kk < KPG; ++kk)
                                mma_f8(d, aLo + (gi * KPG + kk) * 2, bLo + (gi * KPG + kk) * 2, kk > 0 ? 1u : 0u);
                            mma_commit(&sm->acc_full[b]);
                        }
                    } else {
                        // zero-point term: all pseudo-stages of the tile accumulate into one buffer
                        const int z = s - it.kb1;
                        const uint32_t b = jg & 1u;
                        if (z == 0 && !wait_phase_short(&sm->acc_empty[b], ((jg >> 1) & 1u) ^ 1u, sm, a.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem + b * BN, zbLo = rLo + (C_BYTES >> 4);
                        mma_bf16(d, rLo, zbLo, z > 0 ? 1u : 0u);
                        mma_bf16(d, rLo + 2, zbLo + 2, 1u);
                        if (z == a.ZT - 1) {
                            mma_commit(&sm->acc_full[b]);
                            ++jg;
                        }
                    }
                    if (!ok) break;
                    mma_commit(&sm->empty[slot]);
                }
            }
        }
        __syncwarp();
    } else if (warp < 12) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
        // ------------------------------------------------ promotion / epilogue (8 warps)
        const int quarter = warp & 3;            // TMEM lanes 32*quarter ...
        const int half = (warp - 4) >> 2;        // token columns 128*half ...
        const int row = quarter * 32 + lane;
        int64_t jg = 0;
        bool ok = true;
        Work w(a);
        Item it;
        while (ok && w.next(a, it)) {
            Tile T;
            if (!locate_tile(a, it.t, T)) continue;
            const int64_t n = T.n0 + row;
            const uint32_t *scales =
                reinterpret_cast<const uint32_t *>(a.packed + (size_t)T.e * a.slab_bytes + a.codes_bytes);
            // token scales of this warp's 128 columns, column 32c + l held by lane l; read
            // now, used (through shuffles) only in the epilogue
            float rsv[4];
            if (FUSE) {
                const float4 v = fused_row_scales(a.qcnt, a.row_scale, T.row0, T.rows, a.M, half, sm, a.status);
                if (!__all_sync(FULL, v.x == v.x)) {  // NaN: a wait ran out or the CTA aborts
                    ok = false;
                    break;
                }
                rsv[0] = v.x; rsv[1] = v.y; rsv[2] = v.z; rsv[3] = v.w;
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int col = half * 128 + c * 32 + lane;
                    const int64_t m = T.row0 + col;
                    rsv[c] = (col < T.rows && m < a.M) ? __ldg(a.row_scale + m) : 0.0f;
                }
            }
            float2 acc[64];  // columns (2i, 2i+1) of this thread's weight row
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
            // groups [jb, je) of the item, then (when it.z) the zero-point term as group je
            const int jb = it.kb0 * GPS, je = it.kb1 * GPS, jn = je + (it.z ? 1 : 0);
            uint32_t ent0 = scales[(int64_t)jb * a.Npad + n];
            uint32_t ent1 = (jb + 1 < je) ? scales[(int64_t)(jb + 1) * a.Npad + n] : 0u;
            int bl = 0;           // TMEM buffer of the item's last group
            uint32_t tl_addr = 0;  // this warp's columns in it
            for (int j = jb; j < jn && ok; ++j, ++jg) {
                const int b = (int)(jg % NBUF);
                float s512 = -1.0f;  // the zero-point term is subtracted
                if (j < je) {
                    s512 = __half2float(__ushort_as_half((unsigned short)(ent0 & 0xFFFF))) * 512.0f;
                    ent0 = ent1;
                    ent1 = (j + 2 < je) ? scales[(int64_t)(j + 2) * a.Npad + n] : 0u;
                }
                if (!warp_wait_phase_short(&sm->acc_full[b], (uint32_t)(jg / NBUF) & 1, sm, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN + half * 128);
                // 8 chunks of 16 columns, double-buffered: the load of chunk c+1 is in flight
                // while chunk c is promoted
                const float2 s2 = make_float2(s512, s512);
                uint32_t pa[16], pb[16];
                tmem_ld16(taddr, pa);
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    tmem_wait_ld16(pa);
                    tmem_ld16(taddr + (c + 1) * 16, pb);
                    promote16(acc + c * 8, s2, pa);
                    tmem_wait_ld16(pb);
                    if (c + 2 < 8) tmem_ld16(taddr + (c + 2) * 16, pa);
                    promote16(acc + (c + 1) * 8, s2, pb);
                }
                if (j == jn - 1) {
                    // the item's last group: its buffer holds the result for the epilogue below
                    // and is released after it
                    bl = b;
                    tl_addr = taddr;
                    continue;  // ends the loop with jg counted
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->acc_empty[b]);
            }
            if (!ok) break;
            // Epilogue. The result goes through the last group's TMEM buffer so that the store
            // loop can stay rolled (an unrolled 128-column loop runs once per tile and its code
            // is fetched cold every time): 8 stores of 16 columns, then per 16-column chunk one
            // load, the row scale (lane-held, broadcast by shuffle) and the global stores.
#pragma unroll
            for (int c = 0; c < 8; ++c) tmem_st16(tl_addr + c * 16, acc + c * 8);
            tmem_wait_st();
            if (it.seg >= 0 &&
                !split_combine(a.part, a.cnt, a.status, a.R, a.KT, a.PS, it.t - a.DPT, it.seg, warp - 4, tl_addr)) {
                // a split tile's partial sum, stored for the contributor that finishes the tile
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->acc_empty[bl]);
                continue;
            }
            const bool row_ok = n < a.N;
            const int64_t lim = (T.rows < (int64_t)BN ? T.rows : (int64_t)BN);  // valid columns of the tile
            const int64_t lim_m = a.M - T.row0;
            const int64_t ncol = (lim < lim_m ? lim : lim_m) - half * 128;      // valid columns of this half
            // bf16 output with N a multiple of 8: 8x8 transposes across lanes, so that each lane
            // stores 8 consecutive outputs of one token row (16-byte stores); otherwise one value
            // per lane and store
            const bool vec = !a.out_fp32 && (a.N & 7) == 0;
            const int64_t nbase = T.n0 + quarter * 32 + 8 * (lane >> 3);  // first row of the lane's group
            const int li = lane & 7;
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
                uint32_t v[16];
                tmem_ld16(tl_addr + c * 16, v);
                tmem_wait_ld16(v);
                const float rsc = (c >> 1) == 0 ? rsv[0] : (c >> 1) == 1 ? rsv[1] : (c >> 1) == 2 ? rsv[2] : rsv[3];
                const int64_t m0 = T.row0 + half * 128 + c * 16;
                const int l0 = (c & 1) * 16;
                if (vec) {
                    uint32_t h0[4], h1[4];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float r0 = __shfl_sync(FULL, rsc, l0 + 2 * q), r1 = __shfl_sync(FULL, rsc, l0 + 2 * q + 1);
                        const __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(__uint_as_float(v[2 * q]) * r0, __uint_as_float(v[2 * q + 1]) * r1);
                        const uint32_t w = *reinterpret_cast<const uint32_t *>(&b2);
                        if (q < 4) h0[q] = w;
                        else h1[q - 4] = w;
                    }
                    transpose8x8_b16(h0, lane);
                    transpose8x8_b16(h1, lane);
                    if (nbase < a.N) {
                        __nv_bfloat16 *yb = static_cast<__nv_bfloat16 *>(a.Y);
                        if (c * 16 + li < ncol)
                            *reinterpret_cast<uint4 *>(yb + (m0 + li) * a.N + nbase) = make_uint4(h0[0], h0[1], h0[2], h0[3]);
                        if (c * 16 + 8 + li < ncol)
                            *reinterpret_cast<uint4 *>(yb + (m0 + 8 + li) * a.N + nbase) =
                                make_uint4(h1[0], h1[1], h1[2], h1[3]);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float rs = __shfl_sync(FULL, rsc, l0 + k);
                        if (row_ok && c * 16 + k < ncol) {
                            const float val = __uint_as_float(v[k]) * rs;
                            if (a.out_fp32) static_cast<float *>(a.Y)[(m0 + k) * a.N + n] = val;
                            else static_cast<__nv_bfloat16 *>(a.Y)[(m0 + k) * a.N + n] = __float2bfloat16_rn(val);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->acc_empty[bl]);
        }
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 64;\n" ::: "memory");
        // ------------------------------------------------ expansion warps
        const int et = threadIdx.x - 384;  // 0..127
        Ring r;
        bool ok = true;
        Work w(a);
        Item it;
        while (ok && w.next(a, it)) {
            Tile T;
            if (!locate_tile(a, it.t, T)) continue;
            const int send = it.kb1 + (it.z ? a.ZT : 0);
            for (int s = it.kb0; s < send; ++s, r.next()) {
                const int slot = r.slot;
                // the TMA bytes of this use have landed; the producer issued them only after the
                // MMA released the slot's previous use, so the expanded buffer is free as well.
                // Every stage is waited for, pseudo-stages included, so that this role sees each
                // phase of the ring in order.
                if (!warp_wait_phase(&sm->full[slot], r.phase, sm, a.status)) { ok = false; break; }
                if (s < it.kb1) {
                    const uint8_t *src = raw + slot * RAW_BYTES;
                    uint8_t *dstA = sA + slot * A_BYTES;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int idx = et + 128 * i;  // 0..511: (row r, 32-wide part p)
                        const int rr = idx >> 2, p = idx & 3;
                        const uint4 w = *reinterpret_cast<const uint4 *>(src + rr * 64 + p * 16);
                        uint4 o0, o1;
                        o0.x = w.x & 0x0F0F0F0Fu; o0.y = (w.x >> 4) & 0x0F0F0F0Fu;
                        o0.z = w.y & 0x0F0F0F0Fu; o0.w = (w.y >> 4) & 0x0F0F0F0Fu;
                        o1.x = w.z & 0x0F0F0F0Fu; o1.y = (w.z >> 4) & 0x0F0F0F0Fu;
                        o1.z = w.w & 0x0F0F0F0Fu; o1.w = (w.w >> 4) & 0x0F0F0F0Fu;
                        const int c0 = (2 * p) ^ (rr & 7), c1 = (2 * p + 1) ^ (rr & 7);
                        *reinterpret_cast<uint4 *>(dstA + rr * 128 + c0 * 16) = o0;
                        *reinterpret_cast<uint4 *>(dstA + rr * 128 + c1 * 16) = o1;
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                if ((threadIdx.x & 31) == 0) mbar_arrive(&sm->exp_full[slot]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ------------------------------------------------------------------ split-weight FP16 path
//
// With groups of 32 every FP8 MMA (K = 32) ends a group, and the exact per-group promotion
// (a TMEM readback and 128 x 256 fp32 FMAs on the CUDA cores per MMA) costs several times
// the MMA itself. For such groups this kernel keeps the whole K in one TMEM accumulator
// instead: every weight is dequantized exactly and split into two fp16 parts,
//   w = (q - z) s,  hi = fp16(w),  lo = fp16(w - hi),  w = hi + lo,
// and the E4M3 activations arrive as fp16 (exact: every E4M3 value is an fp16 value; the row
// quant writes that copy, so no tile of activations is converted again for every weight
// tile). kind::f16 MMAs accumulate A_hi B + A_lo B in fp32, so the tensor core sees the
// dequantized operands of the method, as in the promoted path, and nothing is read back
// until the tile is done.
// Exactness: q - z is an fp16 integer (1024 + q minus 1024 + z) for |z| < 1024, s is the
// stored fp16 scale, so w has at most 11 + 11 significant bits; hi keeps the leading 11 and
// the fp16 FMA forms lo = w - hi exactly (it is a multiple of 2^-24, the smallest fp16
// subnormal, so it never underflows). A group with |z| >= 1024 forms q - z in fp32 and
// rounds it to fp16, and one with |(q - z) s| >= 65504 overflows fp16; the first is exact
// while |q - z| <= 2048, and both lie far outside any trained weight's range. The cost is
// two fp16 MMAs per K step, a quarter of the FP8 rate, with no per-group readback.
//
// Warp roles (512 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps 4-7
// epilogue (one TMEM lane quarter each, all 256 columns), warps 8-15 expansion. One ring of
// stages, each holding the packed codes and the fp16 activations (B, 128-byte swizzle,
// K-major) loaded by TMA, and the expanded A_hi and A_lo the expansion warps write in the
// layout the MMA reads: TMA -> full -> expansion -> exp_full -> MMA -> empty -> TMA. Two
// TMEM accumulators alternate between tiles, so the epilogue of one tile overlaps the MMAs
// of the next.
namespace f16p {

constexpr int BK = 64;                        // k per stage (one 128-byte swizzle row of fp16)
constexpr int STAGES = 3;
constexpr int EXW = 8;                        // expansion warps
constexpr uint32_t RC_BYTES = BM * BK / 2;    // packed codes of a stage (4 KB)
constexpr uint32_t B_BYTES = BN * BK * 2;     // fp16 activations (32 KB)
constexpr uint32_t AH_BYTES = BM * BK * 2;    // one fp16 weight part (16 KB)
constexpr uint32_t OFF_B = RC_BYTES, OFF_AH = OFF_B + B_BYTES, OFF_AL = OFF_AH + AH_BYTES;
constexpr uint32_t STAGE_BYTES = OFF_AL + AH_BYTES;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 1024;
static_assert(RC_BYTES % 1024 == 0 && B_BYTES % 1024 == 0 && AH_BYTES % 1024 == 0, "swizzle atoms stay aligned");

struct Smem {
    uint64_t full[STAGES];       // TMA bytes (codes + activations) landed
    uint64_t exp_full[STAGES];   // expansion wrote A_hi, A_lo (one arrival per expansion warp)
    uint64_t empty[STAGES];      // the MMAs reading the stage completed (tcgen05.commit)
    uint64_t acc_full[NBUF];     // a tile's accumulator is complete
    uint64_t acc_empty[NBUF];    // the epilogue has read it (one arrival per epilogue warp)
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Smem) <= 1024, "control block");

// instruction descriptor: D fp32, A and B fp16, both K-major, M = BM, N = n (a multiple of 16
// up to BN: a tile's last token columns past its rows are not computed)
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t n) {
    return (1u << 4) | ((n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n .reg .b64 da, db;\n setp.ne.b32 p, %4, 0;\n"
        " mov.b64 da, {%1, %5};\n mov.b64 db, {%2, %5};\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n}\n" ::"r"(tmem_d),
        "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(kDescHiSW128));
}

// token columns of tile T that hold rows of its problem, rounded up to the MMA's N granule
__device__ __forceinline__ uint32_t tile_cols16(const Args &a, const Tile &T) {
    int64_t c = T.rows < (int64_t)BN ? T.rows : (int64_t)BN;
    const int64_t lim_m = a.M - T.row0;
    if (c > lim_m) c = lim_m;
    return (uint32_t)((c + 15) / 16 * 16);
}

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }
__device__ __forceinline__ __half2 bits_h2(uint32_t v) { return *reinterpret_cast<__half2 *>(&v); }

__device__ __forceinline__ bool wait_f(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    return mbar_wait_abortable<true>(bar, parity, &sm->abort, status, kWaitNs);
}
__device__ __forceinline__ bool warp_wait_f(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    bool r = true;
    if ((threadIdx.x & 31) == 0) r = mbar_wait_abortable(bar, parity, &sm->abort, status, kWaitNs);
    r = __shfl_sync(FULL, r ? 1 : 0, 0) != 0;
    if (r) r = __all_sync(FULL, mbar_try_wait_short(bar, parity));
    return r;
}

// position in a ring of N slots
template <int N> struct RingN {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next() {
        if (++slot == N) { slot = 0; phase ^= 1u; }
    }
};

__global__ void __launch_bounds__(THREADS, 1) w4a8_f16split_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                                   const __grid_constant__ CUtensorMap tm_act,
                                                                   const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *sm = reinterpret_cast<Smem *>(base + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = (int)(a.Kpad / BK);
    const int64_t ntiles = (int64_t)a.MTU * a.NT;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->exp_full[s], EXW);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], 4);
        }
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sm->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            RingN<STAGES> r;
            int64_t uses = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                Tile T;
                if (!locate_tile(a, t, T)) continue;
                for (int s = 0; s < KT; ++s, r.next(), ++uses) {
                    if (!wait_f(&sm->empty[r.slot], r.phase ^ 1u, sm, a.status)) { ok = false; break; }
                    uint8_t *dst = base + r.slot * STAGE_BYTES;
                    mbar_arrive_expect_tx(&sm->full[r.slot], RC_BYTES + B_BYTES);
                    tma_load_3d(dst, &tm_codes, s * (BK / 2), (int)T.n0, T.e, &sm->full[r.slot]);
                    tma_load_2d(dst + OFF_B, &tm_act, s * BK, (int)T.row0, &sm->full[r.slot]);
                }
            }
            // no copy may land after the CTA exits: wait for the last uses' bytes
            for (int64_t u = uses > STAGES ? uses - STAGES : 0; u < uses; ++u)
                (void)mbar_wait_bounded(&sm->full[u % STAGES], (uint32_t)(u / STAGES) & 1, a.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            RingN<STAGES> r;
            uint32_t tiles_done = 0;
            int64_t uses = 0;
            bool ok = true;
            const uint32_t lo0 = desc_lo(smem_addr(base));
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                Tile T;
                if (!locate_tile(a, t, T)) continue;
                const uint32_t b = tiles_done & 1u;
                if (!wait_f(&sm->acc_empty[b], ((tiles_done >> 1) & 1u) ^ 1u, sm, a.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + b * BN;
                const uint32_t idesc = idesc_f16(tile_cols16(a, T));
                for (int s = 0; s < KT; ++s, r.next()) {
                    if (!wait_f(&sm->exp_full[r.slot], r.phase, sm, a.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = lo0 + (uint32_t)r.slot * (STAGE_BYTES >> 4);
                    const uint32_t bLo = st + (OFF_B >> 4), hLo = st + (OFF_AH >> 4), lLo = st + (OFF_AL >> 4);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {  // K = 16 per fp16 MMA: 32 bytes
                        mma_f16(d, hLo + kk * 2, bLo + kk * 2, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                        mma_f16(d, lLo + kk * 2, bLo + kk * 2, idesc, 1u);
                    }
                    mma_commit(&sm->empty[r.slot]);
                    ++uses;
                }
                if (!ok) break;
                mma_commit(&sm->acc_full[b]);
                ++tiles_done;
            }
            // no commit may arrive after the CTA exits: wait for the last stages' completions
            for (int64_t u = uses > STAGES ? uses - STAGES : 0; u < uses; ++u)
                (void)mbar_wait_bounded(&sm->empty[u % STAGES], (uint32_t)(u / STAGES) & 1, a.status);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ epilogue (4 warps)
        const int quarter = warp & 3;  // TMEM lanes (weight rows) 32*quarter ...
        uint32_t tiles_done = 0;
        for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
            Tile T;
            if (!locate_tile(a, t, T)) continue;
            const uint32_t b = tiles_done & 1u;
            if (!warp_wait_f(&sm->acc_full[b], (tiles_done >> 1) & 1u, sm, a.status)) break;
            tc_fence_after();
            const uint32_t tl_addr = tmem + ((uint32_t)(quarter * 32) << 16) + b * BN;
            const int64_t n = T.n0 + quarter * 32 + lane;
            const bool row_ok = n < a.N;
            const int64_t lim = (T.rows < (int64_t)BN ? T.rows : (int64_t)BN);
            const int64_t lim_m = a.M - T.row0;
            const int64_t ncol = lim < lim_m ? lim : lim_m;  // valid token columns of the tile
            const bool vec = !a.out_fp32 && (a.N & 7) == 0;
            const int64_t nbase = T.n0 + quarter * 32 + 8 * (lane >> 3);
            const int li = lane & 7;
            const int nchunks = (int)((ncol + 15) / 16);  // TMEM columns the MMAs wrote
#pragma unroll 1
            for (int c = 0; c < nchunks; ++c) {
                uint32_t v[16];
                tmem_ld16(tl_addr + c * 16, v);
                // token scale of column 16c + (lane & 15)
                const int colr = c * 16 + (lane & 15);
                const float rsc = colr < ncol ? __ldg(a.row_scale + T.row0 + colr) : 0.0f;
                tmem_wait_ld16(v);
                const int64_t m0 = T.row0 + c * 16;
                if (vec) {
                    uint32_t h0[4], h1[4];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float r0 = __shfl_sync(FULL, rsc, 2 * q), r1 = __shfl_sync(FULL, rsc, 2 * q + 1);
                        const __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(__uint_as_float(v[2 * q]) * r0, __uint_as_float(v[2 * q + 1]) * r1);
                        const uint32_t w = *reinterpret_cast<const uint32_t *>(&b2);
                        if (q < 4) h0[q] = w;
                        else h1[q - 4] = w;
                    }
                    transpose8x8_b16(h0, lane);
                    transpose8x8_b16(h1, lane);
                    if (nbase < a.N) {
                        __nv_bfloat16 *yb = static_cast<__nv_bfloat16 *>(a.Y);
                        if (c * 16 + li < ncol)
                            *reinterpret_cast<uint4 *>(yb + (m0 + li) * a.N + nbase) = make_uint4(h0[0], h0[1], h0[2], h0[3]);
                        if (c * 16 + 8 + li < ncol)
                            *reinterpret_cast<uint4 *>(yb + (m0 + 8 + li) * a.N + nbase) =
                                make_uint4(h1[0], h1[1], h1[2], h1[3]);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float rs = __shfl_sync(FULL, rsc, k);
                        if (row_ok && c * 16 + k < ncol) {
                            const float val = __uint_as_float(v[k]) * rs;
                            if (a.out_fp32) static_cast<float *>(a.Y)[(m0 + k) * a.N + n] = val;
                            else static_cast<__nv_bfloat16 *>(a.Y)[(m0 + k) * a.N + n] = __float2bfloat16_rn(val);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->acc_empty[b]);
            ++tiles_done;
        }
    } else if (warp >= 8) {
        // ------------------------------------------------ expansion (8 warps, 256 threads)
        const int et = threadIdx.x - 256;        // 0..255
        const int wr = et >> 1, wh = et & 1;      // weight row, half of the stage's 64 k
        RingN<STAGES> r;
        bool ok = true;
        const __half2 h1024 = __float2half2_rn(1024.0f);
        const uint32_t magic = 0x64646464u;      // high bytes of fp16 1024 + q
        for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            Tile T;
            if (!locate_tile(a, t, T)) continue;
            const int64_t n = T.n0 + wr;
            const uint32_t *scales =
                reinterpret_cast<const uint32_t *>(a.packed + (size_t)T.e * a.slab_bytes + a.codes_bytes);
            // this thread's scale entry for stage s (k = 64 s + 32 wh + 0..31 lies in group
            // (64 s + 32 wh) / g) is loaded four stages ahead, in a queue of registers: it does not
            // depend on the ring, and an L2 load under the weight stream takes about a stage
            auto ent_at = [&](int st) -> uint32_t {
                return st < KT ? __ldg(scales + ((int64_t)st * BK + wh * 32) / a.g * a.Npad + n) : 0u;
            };
            uint32_t q0 = ent_at(0), q1 = ent_at(1), q2 = ent_at(2), q3 = ent_at(3);
            for (int s = 0; s < KT; ++s, r.next()) {
                const uint32_t ent = q0;
                q0 = q1;
                q1 = q2;
                q2 = q3;
                q3 = ent_at(s + 4);
                // the stage was refilled only after the MMAs that read its previous A_hi and
                // A_lo completed, so once its TMA bytes landed both buffers are free
                if (!warp_wait_f(&sm->full[r.slot], r.phase, sm, a.status)) { ok = false; break; }
                uint8_t *stg = base + r.slot * STAGE_BYTES;
                const int z = (int)(int16_t)(ent >> 16);
                const __half2 s2 = __half2half2(__ushort_as_half((unsigned short)(ent & 0xFFFFu)));
                const uint4 cw = *reinterpret_cast<const uint4 *>(stg + wr * 32 + wh * 16);
                const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
                uint32_t hi[16], lo[16];
                if (z > -1024 && z < 1024) {
                    const __half2 c0 = __hadd2(h1024, __float2half2_rn((float)z));
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t bl = wv[i] & 0x0F0F0F0Fu, bh = (wv[i] >> 4) & 0x0F0F0F0Fu;
                        const uint32_t p[4] = {__byte_perm(bl, magic, 0x4140), __byte_perm(bl, magic, 0x4342),
                                               __byte_perm(bh, magic, 0x4140), __byte_perm(bh, magic, 0x4342)};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __half2 cc = __hsub2(bits_h2(p[e]), c0);
                            const __half2 h = __hmul2(cc, s2);
                            hi[4 * i + e] = h2_bits(h);
                            lo[4 * i + e] = h2_bits(__hfma2(cc, s2, __hneg2(h)));
                        }
                    }
                } else {
                    // zero point beyond fp16's exact integers around 1024: q - z in fp32
                    const float sf = __half2float(__ushort_as_half((unsigned short)(ent & 0xFFFFu)));
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            // nibble slots: k0 + p/2 + 4 (p % 2) holds slot p
                            const int k0 = 2 * e;  // weights k0 and k0 + 1 of this word
                            const int p0 = (k0 & 3) * 2 + (k0 >> 2), p1 = ((k0 + 1) & 3) * 2 + ((k0 + 1) >> 2);
                            const float q0 = (float)((wv[i] >> (4 * p0)) & 0xFu), q1 = (float)((wv[i] >> (4 * p1)) & 0xFu);
                            const __half2 cc = __floats2half2_rn(q0 - (float)z, q1 - (float)z);
                            const __half2 h = __hmul2(cc, __float2half2_rn(sf));
                            hi[4 * i + e] = h2_bits(h);
                            lo[4 * i + e] = h2_bits(__hfma2(cc, __float2half2_rn(sf), __hneg2(h)));
                        }
                    }
                }
                // 16-byte chunks 4 wh .. 4 wh + 3 of row wr (8 k each), 128-byte swizzle
                uint8_t *ah = stg + OFF_AH + wr * 128, *al = stg + OFF_AL + wr * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int pc = (4 * wh + c) ^ (wr & 7);
                    *reinterpret_cast<uint4 *>(ah + pc * 16) = make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                    *reinterpret_cast<uint4 *>(al + pc * 16) = make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->exp_full[r.slot]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

}  // namespace f16p

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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

static int sm_count_cached() {
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return num_sms();
    if (!cache[dev]) cache[dev] = num_sms();
    return cache[dev];
}

// Launch the kernel instantiation for group size G (first call per device sets its shared
// memory limit).
template <int G, bool FUSE = false>
static w4_status start(int grid, const CUtensorMap &tm_codes, const CUtensorMap &tm_act, const CUtensorMap &tm_zop,
                       const CUtensorMap &tm_gop, const Args &a, cudaStream_t stream) {
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(w4a8_kernel<G, FUSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES) != cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev] = 1;
    }
    w4a8_kernel<G, FUSE><<<grid, THREADS, SMEM_BYTES, stream>>>(tm_codes, tm_act, tm_zop, tm_gop, a);
    return launch_status();
}

// Work split of a dense problem of `tiles` tiles of KT k-blocks over `sms` SMs. Whole tiles go
// round-robin over the grid; when the last wave would leave a useful share of the SMs idle,
// its R tiles are split along K instead, over PS CTAs with at least kMinSplitBlocks k-blocks
// each and at most about kMaxParts contributors per tile. With whole waves as well, PS is the
// whole grid (the least work per CTA; the combine steps overlap the whole tiles that follow).
// With none, PS is a multiple of R, so that every CTA works on one tile and each tile has the
// fewest contributors, since there the combine step is the kernel's last.
constexpr int64_t kMinSplitBlocks = 8;
constexpr int64_t kMaxParts = 8;

struct Plan {
    int64_t tiles, dpt, r, ps;
    int grid;
    size_t ws_bytes;
};

static Plan make_plan(int64_t tiles, int64_t KT, int sms, bool splittable) {
    Plan p;
    p.tiles = tiles;
    p.dpt = tiles;
    p.r = 0;
    p.ps = 0;
    p.grid = (int)(tiles < sms ? tiles : sms);
    p.ws_bytes = 0;
    if (!splittable || sms < 1 || tiles < 1) return p;
    const int64_t waves = tiles / sms, r = tiles % sms;
    if (r == 0 || (waves > 0 && r > sms - sms / 8)) return p;  // the last wave is (nearly) full
    int64_t ps = r * KT / kMinSplitBlocks;
    if (ps > r * kMaxParts) ps = r * kMaxParts;
    if (ps > sms) ps = sms;
    if (waves == 0 && ps / r >= 2) ps = r * (ps / r);
    if (ps < r + r / 4 + 1) return p;  // splitting would shorten the last wave by too little
    if (ps * kMinSplitBlocks > r * KT) return p;  // every CTA needs a non-empty range
    p.dpt = tiles - r;
    p.r = r;
    p.ps = ps;
    p.grid = waves > 0 ? sms : (int)ps;
    p.ws_bytes = (size_t)(2 * ps) * PART_FLOATS * sizeof(float) + (size_t)(r * 8) * sizeof(uint32_t);
    return p;
}

static int64_t dense_tiles(int64_t M, int64_t N, int64_t K, int group) {
    const GemmLayout L = gemm_layout(N, K, group);
    return ((M + BN - 1) / BN) * (L.Npad / BM);
}

// Groups of 32 and 256: the split-weight fp16 kernel (no per-group promotion, no zero-point
// operand); the activations are the fp16 copy of the E4M3 values.
static w4_status launch_f16(const uint16_t *X16, const float *row_scale, const int32_t *offsets, int E, int64_t M,
                            const void *packed, int64_t N, int64_t K, int group, void *Y, int out_fp32,
                            cudaStream_t stream) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return W4_ERR_CUDA;
    const GemmLayout L = gemm_layout(N, K, group);
    const uint8_t *pk = static_cast<const uint8_t *>(packed);
    CUtensorMap tm_codes, tm_act;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)(L.Kpad / 2), (cuuint64_t)L.Npad, (cuuint64_t)E};
        const cuuint64_t strides[2] = {(cuuint64_t)(L.Kpad / 2), (cuuint64_t)L.total};
        const cuuint32_t box[3] = {f16p::BK / 2, BM, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(pk), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    {
        // fp16 [M][K]: 64 k (128 bytes) x 256 rows per stage, 128-byte swizzle (the MMA's
        // K-major layout); rows past M and k past K read as zero
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {f16p::BK, BN};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tm_act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t *>(X16), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    Args a{};
    a.packed = pk;
    a.slab_bytes = L.total;
    a.codes_bytes = L.codes_bytes;
    a.row_scale = row_scale;
    a.offsets = offsets;
    a.Y = Y;
    a.status = device_status_ptr();
    a.M = M; a.N = N; a.Npad = L.Npad; a.K = K; a.Kpad = L.Kpad;
    a.E = E; a.g = group; a.out_fp32 = out_fp32;
    a.NT = (int)(L.Npad / BM);
    const int64_t mtu = offsets ? (M + BN - 1) / BN + E : (M + BN - 1) / BN;
    if (mtu > 0x7fffffffLL || mtu * a.NT > 0x7fffffffLL) return W4_ERR_SHAPE;
    a.MTU = (int)mtu;
    const int64_t tiles = mtu * a.NT;
    const int sms = sm_count_cached();
    const int grid = (int)(tiles < sms ? tiles : sms);
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(f16p::w4a8_f16split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)f16p::SMEM_BYTES) !=
            cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev] = 1;
    }
    f16p::w4a8_f16split_kernel<<<grid, THREADS, f16p::SMEM_BYTES, stream>>>(tm_codes, tm_act, a);
    return launch_status();
}

// The workspace of the kernel variant that quantizes its own activation rows: the split-tile
// partials and counters of the plan, one row counter per token tile (both cleared before
// every launch by one memset), then the E4M3 rows, the row scales and the group-sum operand.
struct FusedLayout {
    size_t cnt, rowcnt, q8, scale, gop, end;  // byte offsets; end = total size
};

static size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

static FusedLayout fused_layout(const Plan &P, int64_t M, int64_t K, int64_t KZ) {
    FusedLayout f;
    f.cnt = (size_t)(2 * P.ps) * PART_FLOATS * sizeof(float);
    f.rowcnt = round256(f.cnt + (size_t)(P.r * 8) * sizeof(uint32_t));
    f.q8 = round256(f.rowcnt + (size_t)((M + BN - 1) / BN) * sizeof(uint32_t));
    f.scale = round256(f.q8 + (size_t)M * (size_t)K);
    f.gop = round256(f.scale + (size_t)M * sizeof(float));
    f.end = round256(f.gop + (size_t)M * (size_t)KZ * 2);
    return f;
}

// Row ranges quantized before the roles start: the token tiles of the first `waves` waves of
// whole tiles, [0, a1), and those of the split tiles, [a2, M), which the CTAs holding split
// segments take first. Warps 2-3 quantize [a1, a2) while the GEMM runs.
static void fused_first_rows(const Plan &P, int64_t M, int64_t NT, int waves, int64_t &a1, int64_t &a2) {
    const int64_t w = (int64_t)P.grid * waves;
    const int64_t first_whole = P.dpt < w ? P.dpt : w;
    a1 = first_whole > 0 ? ((first_whole - 1) / NT + 1) * BN : 0;
    a2 = P.r > 0 ? (P.dpt / NT) * BN : M;
    if (a2 > M) a2 = M;
    if (a1 > a2) a1 = a2;
}

constexpr int64_t kBackgroundMaxK = 16384;

struct FusedIn {
    const uint16_t *X;  // bf16 activations [M, K]
};

static w4_status launch(const uint8_t *X8, const uint16_t *X16, const float *row_scale, const uint16_t *gop,
                        const int32_t *offsets, int E, int64_t M, const void *packed, int64_t N, int64_t K, int group,
                        void *Y, int out_fp32, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                        const FusedIn *fz = nullptr) {
    if (fz && (group != 64 && group != 128)) return W4_ERR_UNSUPPORTED;
    if (group == 32 || group == 256)
        return launch_f16(X16, row_scale, offsets, E, M, packed, N, K, group, Y, out_fp32, stream);
    EncodeTiledFn enc = encode_fn();
    if (!enc) return W4_ERR_CUDA;
    const GemmLayout L = gemm_layout(N, K, group);
    const uint8_t *pk = static_cast<const uint8_t *>(packed);
    const int64_t NT = L.Npad / BM;
    const int64_t mtu = offsets ? (M + BN - 1) / BN + E : (M + BN - 1) / BN;
    if (mtu > 0x7fffffffLL) return W4_ERR_SHAPE;
    const Plan P = make_plan(mtu * NT, L.Kpad / BK, sm_count_cached(), !offsets && workspace != nullptr);
    FusedLayout FL{};
    if (fz) {
        FL = fused_layout(P, M, K, L.KZ);
        if (!workspace || FL.end > workspace_bytes) return W4_ERR_WORKSPACE;
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        X8 = ws + FL.q8;
        row_scale = reinterpret_cast<const float *>(ws + FL.scale);
        gop = reinterpret_cast<const uint16_t *>(ws + FL.gop);
    }
    CUtensorMap tm_codes, tm_act, tm_zop, tm_gop;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)(L.Kpad / 2), (cuuint64_t)L.Npad, (cuuint64_t)E};
        const cuuint64_t strides[2] = {(cuuint64_t)(L.Kpad / 2), (cuuint64_t)L.total};
        const cuuint32_t box[3] = {BK / 2, BM, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(pk), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K};
        const cuuint32_t box[2] = {BK, BN};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tm_act, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(X8), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    {
        const cuuint64_t dims[3] = {(cuuint64_t)L.KZ, (cuuint64_t)L.Npad, (cuuint64_t)E};
        const cuuint64_t strides[2] = {(cuuint64_t)(L.KZ * 2), (cuuint64_t)L.total};
        const cuuint32_t box[3] = {ZKC, BM, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tm_zop, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                const_cast<uint8_t *>(pk + L.codes_bytes + L.scales_bytes), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)L.KZ, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)(L.KZ * 2)};
        const cuuint32_t box[2] = {ZKC, BN};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tm_gop, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(gop), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    Args a{};
    a.packed = pk;
    a.slab_bytes = L.total;
    a.codes_bytes = L.codes_bytes;
    a.row_scale = row_scale;
    a.offsets = offsets;
    a.Y = Y;
    a.status = device_status_ptr();
    a.M = M; a.N = N; a.Npad = L.Npad; a.K = K; a.Kpad = L.Kpad;
    a.E = E; a.g = group; a.out_fp32 = out_fp32;
    a.NT = (int)NT;
    a.MTU = (int)mtu;
    a.KT = (int)(L.Kpad / BK);
    a.ZT = (int)(L.KZ / ZKC);
    if (P.ws_bytes > workspace_bytes) return W4_ERR_WORKSPACE;
    a.DPT = P.dpt;
    a.R = P.r;
    a.PS = P.ps;
    a.part = P.r ? static_cast<float *>(workspace) : nullptr;
    a.cnt = P.r ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) +
                                               (size_t)(2 * P.ps) * PART_FLOATS * sizeof(float))
                : nullptr;
    const int grid = P.grid;
    if (fz) {
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        a.xq = fz->X;
        a.q8 = ws + FL.q8;
        a.qscale = reinterpret_cast<float *>(ws + FL.scale);
        a.qgop = reinterpret_cast<uint16_t *>(ws + FL.gop);
        a.qcnt = reinterpret_cast<uint32_t *>(ws + FL.rowcnt);
        a.KZ = L.KZ;
        a.qstaged = (size_t)K * 2 * 2 <= RING_BYTES ? 1 : 0;
        // staged: the token tiles of the first two waves of whole tiles before the GEMM starts
        // (room for the background warps to get ahead); streamed: those of the first wave
        fused_first_rows(P, M, NT, a.qstaged ? 2 : 1, a.qa1, a.qa2);
        // Rows of at most half the ring are staged through it before the GEMM starts: those of
        // the token tiles the first two waves and the split tiles read; the rest are quantized
        // while the GEMM runs, by two warps per block, whose loads in flight keep up with the
        // third wave's demand up to rows of kBackgroundMaxK elements; longer staged rows all go
        // before the GEMM. Rows too long for the ring are streamed by warps.
        if (a.qstaged && K > kBackgroundMaxK) a.qa1 = a.qa2 = M;
        // split-tile counters and token-tile row counters start at zero on every call
        if (cudaMemsetAsync(ws + FL.cnt, 0, FL.q8 - FL.cnt, stream) != cudaSuccess) return W4_ERR_CUDA;
        return group == 64 ? start<64, true>(grid, tm_codes, tm_act, tm_zop, tm_gop, a, stream)
                           : start<128, true>(grid, tm_codes, tm_act, tm_zop, tm_gop, a, stream);
    }
    switch (group) {
        case 32: return start<32>(grid, tm_codes, tm_act, tm_zop, tm_gop, a, stream);
        case 64: return start<64>(grid, tm_codes, tm_act, tm_zop, tm_gop, a, stream);
        default: return start<128>(grid, tm_codes, tm_act, tm_zop, tm_gop, a, stream);
    }
}

}  // namespace gemm
}  // namespace w4

using namespace w4;

static bool gemm_shape_ok(int64_t M, int64_t N, int64_t K) {
    return M >= 1 && M <= 0x7fffffffLL && N >= 1 && N <= 0x7fffffffLL && K >= 128 && K % 32 == 0 && K <= (1LL << 24);
}

W4_API size_t w4a8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int group) {
    if (!gemm_shape_ok(M, N, K) || !valid_group(group) || K % group != 0) return 0;
    const int sms = gemm::sm_count_cached();
    if (sms < 1) return 0;
    return gemm::make_plan(gemm::dense_tiles(M, N, K, group), gemm_layout(N, K, group).Kpad / gemm::BK, sms,
                           group == 64 || group == 128)
        .ws_bytes;
}

W4_API w4_status w4a8_gemm_schedule(int64_t M, int64_t N, int64_t K, int group, int sms, int64_t *out) {
    if (!out) return W4_ERR_NULL;
    if (!gemm_shape_ok(M, N, K) || sms < 1 || sms > 4096) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    const int64_t KT = gemm_layout(N, K, group).Kpad / gemm::BK;
    const gemm::Plan p = gemm::make_plan(gemm::dense_tiles(M, N, K, group), KT, sms, group == 64 || group == 128);
    out[0] = p.tiles;
    out[1] = p.dpt;
    out[2] = p.r;
    out[3] = p.ps;
    out[4] = p.grid;
    out[5] = (int64_t)p.ws_bytes;
    out[6] = KT;
    return W4_OK;
}

W4_API w4_status w4a8_gemm_split_segment(int64_t R, int64_t KT, int64_t PS, int64_t c, int s, int64_t *out) {
    if (!out) return W4_ERR_NULL;
    if (R < 1 || KT < 1 || KT > (1LL << 20) || PS < R || PS > 4096 || PS > R * KT || c < 0 || c >= PS || s < 0)
        return W4_ERR_ARG;
    const int64_t Q = R * KT;
    int64_t q = gemm::split_begin(Q, PS, c);
    const int64_t q1 = gemm::split_begin(Q, PS, c + 1);
    for (int k = 0; k < 7; ++k) out[k] = -1;
    out[0] = 0;
    for (int k = 0; q < q1; ++k) {
        int64_t i;
        int kb0, kb1;
        q = gemm::split_segment(q, q1, (int)KT, i, kb0, kb1);
        if (k == s) {
            out[0] = 1;
            out[1] = i;
            out[2] = kb0;
            out[3] = kb1;
            out[4] = gemm::split_cta_of(Q, PS, i * KT);
            out[5] = gemm::split_cta_of(Q, PS, i * KT + KT - 1);
            out[6] = gemm::split_slot(Q, PS, (int)KT, c, i);
            break;
        }
    }
    return W4_OK;
}

// The activation operands a group size needs: E4M3 codes and the group-sum operand for the
// promoted path (64, 128), the binary16 copy for the split-weight path (32, 256).
static bool operands_given(int group, const uint8_t *X8, const uint16_t *X16, const uint16_t *gop) {
    if (group == 32 || group == 256) return X16 != nullptr;
    return X8 && gop;
}

W4_API w4_status w4a8_gemm(const uint8_t *X_e4m3, const uint16_t *X_f16, const float *row_scale,
                           const uint16_t *gsum_op, int64_t M, const void *packed, int64_t N, int64_t K, int group,
                           int mode, void *Y, int out_fp32, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    if (!row_scale || !packed || !Y || !operands_given(group, X_e4m3, X_f16, gsum_op)) return W4_ERR_NULL;
    if (!valid_mode(mode) || (out_fp32 != 0 && out_fp32 != 1)) return W4_ERR_ARG;
    if (!gemm_shape_ok(M, N, K)) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(X_e4m3) || !aligned16(X_f16) || !aligned16(row_scale) || !aligned16(gsum_op) ||
        !aligned16(packed) || !aligned16(Y) || !aligned16(workspace))
        return W4_ERR_ALIGN;
    return gemm::launch(X_e4m3, X_f16, row_scale, gsum_op, nullptr, 1, M, packed, N, K, group, Y, out_fp32,
                        workspace, workspace_bytes, stream);
}

W4_API w4_status w4a8_grouped_gemm(const uint8_t *X_e4m3, const uint16_t *X_f16, const float *row_scale,
                                   const uint16_t *gsum_op, const int32_t *expert_row_offsets, int E,
                                   int64_t M_total, const void *packed, int64_t N, int64_t K, int group, int mode,
                                   void *Y, cudaStream_t stream) {
    if (!row_scale || !expert_row_offsets || !packed || !Y || !operands_given(group, X_e4m3, X_f16, gsum_op))
        return W4_ERR_NULL;
    if (!valid_mode(mode)) return W4_ERR_ARG;
    if (E < 1 || E > 1024 || M_total < 1 || M_total > 0x7fffffffLL || N < 1 || N > 0x7fffffffLL || K < 128 ||
        K % 32 != 0 || K > (1LL << 24))
        return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(X_e4m3) || !aligned16(X_f16) || !aligned16(row_scale) || !aligned16(gsum_op) ||
        !aligned16(packed) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(expert_row_offsets) & 3))
        return W4_ERR_ALIGN;
    return gemm::launch(X_e4m3, X_f16, row_scale, gsum_op, expert_row_offsets, E, M_total, packed, N, K, group, Y, 0,
                        nullptr, 0, stream);
}

// ------------------------------------------------------------------ row quant + GEMM in one launch

static bool rowquant_layout(int64_t M, int64_t N, int64_t K, int group, gemm::FusedLayout &F) {
    if (!gemm_shape_ok(M, N, K) || (group != 64 && group != 128) || K % group != 0) return false;
    const int sms = gemm::sm_count_cached();
    if (sms < 1) return false;
    const GemmLayout L = gemm_layout(N, K, group);
    const gemm::Plan P = gemm::make_plan(gemm::dense_tiles(M, N, K, group), L.Kpad / gemm::BK, sms, true);
    F = gemm::fused_layout(P, M, K, L.KZ);
    return true;
}

W4_API size_t w4a8_gemm_rowquant_workspace_bytes(int64_t M, int64_t N, int64_t K, int group) {
    gemm::FusedLayout F;
    return rowquant_layout(M, N, K, group, F) ? F.end : 0;
}

W4_API w4_status w4a8_gemm_rowquant_layout(int64_t M, int64_t N, int64_t K, int group, int64_t *out) {
    if (!out) return W4_ERR_NULL;
    if (!gemm_shape_ok(M, N, K)) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    gemm::FusedLayout F;
    if (!rowquant_layout(M, N, K, group, F)) return W4_ERR_UNSUPPORTED;
    out[0] = (int64_t)F.q8;
    out[1] = (int64_t)F.scale;
    out[2] = (int64_t)F.gop;
    out[3] = (int64_t)F.end;
    return W4_OK;
}

W4_API w4_status w4a8_gemm_rowquant(const void *X_bf16, int64_t M, const void *packed, int64_t N, int64_t K,
                                    int group, int mode, void *Y, int out_fp32, void *workspace,
                                    size_t workspace_bytes, cudaStream_t stream) {
    if (!X_bf16 || !packed || !Y || !workspace) return W4_ERR_NULL;
    if (!valid_mode(mode) || (out_fp32 != 0 && out_fp32 != 1)) return W4_ERR_ARG;
    if (!gemm_shape_ok(M, N, K)) return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (group != 64 && group != 128) return W4_ERR_UNSUPPORTED;
    if (!aligned16(X_bf16) || !aligned16(packed) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return W4_ERR_ALIGN;
    const gemm::FusedIn fz{static_cast<const uint16_t *>(X_bf16)};
    return gemm::launch(nullptr, nullptr, nullptr, nullptr, nullptr, 1, M, packed, N, K, group, Y, out_fp32, workspace,
                        workspace_bytes, stream, &fz);
}
