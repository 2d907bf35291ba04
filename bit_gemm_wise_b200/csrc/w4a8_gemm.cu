// w4a8_gemm / w4a8_grouped_gemm: INT4 weights x FP8 E4M3 activations on the sm_100a
// tensor cores (tcgen05.mma, TMEM accumulators, TMA operand loads).
//
// "Four-bit inference ... Tahoma", Achievement 2 (the W4A8 dataflow: packed 4-bit weights
// read from HBM, expanded to E4M3 inside the GEMM, FP8 tensor-core MMA with FP32
// accumulation, per-token activation scale in the epilogue, BF16 result) and
// "4-bit by default" (mixture-of-experts weights are the 4-bit target).
//
//   Y[m, n] = s_a[m] * ( sum_j 512 s[n,j] P_j[m,n]  -  sum_j s[n,j] z[n,j] G[m,j] ),
//   P_j[m,n] = sum_{k in j} a8[m,k] * (q[n,k] * 2^-9),   G[m,j] = sum_{k in j} a8[m,k]
//
// Design (one persistent CTA per SM, tiles of 128 weight rows x 256 tokens):
//  * swap-AB: the weight tile is the MMA's A operand (M = 128 weight rows, one TMEM lane per
//    weight row), 256 tokens are its N; each promotion thread owns one weight row, so the
//    group scale is a per-thread scalar;
//  * expansion: a nibble q in [0, 15] zero-extended to a byte IS the E4M3 pattern of q*2^-9
//    (exponent field 0/1 spans the integer grid m*2^-9, m = 0..15), so the expanded weights
//    are exact and the expansion is two AND/shift ops per 8 weights, written straight into
//    the 128-byte-swizzled K-major layout the MMA reads;
//  * per group j, kind::f8f6f4 MMAs (K = 32 each) accumulate P_j into one of two TMEM
//    buffers (2 x 256 columns); 8 promotion warps read it back (tcgen05.ld) and add
//    512 s[n,j] P_j into fp32 registers while the MMA fills the other buffer;
//  * the zero-point term is a rank-J product Z = (s z) G^T computed on the tensor cores too:
//    after a tile's last group the expansion warps write bf16 hi/lo splits of s*z (A) and of
//    G (B) -- [hi|hi|lo] x [hi|lo|hi] along K, error ~2^-16 relative -- into the same
//    pipeline buffers, the MMA thread accumulates them with kind::f16 into a TMEM buffer,
//    and the promotion warps subtract it as one more "group";
//  * warp roles: warp 0 TMA producer, warp 1 TMEM owner + single-thread MMA issuer, warps
//    4-11 promotion/epilogue (register budget raised with setmaxnreg), warps 12-15
//    expansion; rings: 4 raw stages (codes + activations) and 2 expanded-weight buffers;
//  * every mbarrier wait is bounded by wall-clock time; on expiry the kernel records
//    W4_ERR_TIMEOUT, every role sees the abort flag, TMEM is freed and the CTA returns.
#include "w4_common.cuh"
#include "w4_layout.cuh"

#include <cuda.h>

namespace w4 {
namespace gemm {

constexpr int BM = 128;       // weight rows per tile (MMA M)
constexpr int BN = 256;       // tokens per tile (MMA N)
constexpr int BK = 128;       // k per pipeline stage (one 128-byte swizzle row of E4M3)
constexpr int STAGES = 4;     // raw stages: packed codes + activations
constexpr int EXP = 2;        // expanded-weight buffers
constexpr int NBUF = 2;       // TMEM accumulator buffers
constexpr int TMEM_COLS = NBUF * BN;
constexpr int THREADS = 512;
constexpr int ZK = 64;        // bf16 elements of the zero-point product per pseudo-stage
constexpr uint32_t C_BYTES = BM * BK / 2;   // packed codes of a stage
constexpr uint32_t B_BYTES = BN * BK;       // activations of a stage
constexpr uint32_t S_BYTES = BM * 4 * 4;    // scale/zero entries of a stage (up to 4 groups)
constexpr uint32_t RAW_BYTES = C_BYTES + B_BYTES + S_BYTES;
constexpr uint32_t A_BYTES = BM * BK;       // expanded weights
constexpr uint32_t SMEM_BYTES = STAGES * RAW_BYTES + EXP * A_BYTES + 4096 /*control*/ + 1024 /*alignment*/;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait

struct Smem {
    uint64_t full[STAGES];     // raw stage ready (TMA bytes, or a pseudo-stage written by threads)
    uint64_t empty[STAGES];    // raw stage consumed by the MMA
    uint64_t exp_full[EXP];    // expanded weights / zero-point A operand ready
    uint64_t exp_empty[EXP];   // expanded buffer consumed by the MMA
    uint64_t acc_full[NBUF];   // a group's accumulator is complete in TMEM
    uint64_t acc_empty[NBUF];  // promotion finished reading it
    uint32_t tmem_base;
    int abort;
};

struct Args {
    const uint8_t *packed;         // slab 0
    size_t slab_bytes;             // bytes per expert slab
    size_t codes_bytes;            // codes part of a slab (scales follow)
    const float *row_scale;        // [M_total]
    const float *gsum;             // [M_total, Jr]
    const int32_t *offsets;        // [E+1] device, or null: one problem of M rows
    void *Y;                       // [M_total, N]
    int *status;
    int64_t M, N, Npad, K, Kpad;
    int E, g, Jr, out_fp32;
    size_t flags_off;              // per-tile zero-point flags, from the start of a slab
    int NT;                        // weight tiles (Npad / BM)
    int MTU;                       // token tiles (upper bound for grouped problems)
    int KT;                        // raw stages per tile
    int ZT;                        // zero-point pseudo-stages per tile
};

__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    return mbar_wait_abortable(bar, parity, &sm->abort, status, kWaitNs);
}

// K-major operand descriptor, 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes
// apart (stride byte offset), leading byte offset 16 bytes, descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// instruction descriptors: D fp32, both operands K-major, N = BN, M = BM;
// A/B E4M3 (kind::f8f6f4) or BF16 (kind::f16)
constexpr uint32_t kIdescF8 = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescBF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdescF8), "r"(accumulate));
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdescBF16), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

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

// bf16 round-to-nearest-even of an fp32 value, as the 16-bit pattern (finite inputs)
__device__ __forceinline__ uint32_t bf16_bits_rn(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

struct Tile {
    int zflag;      // the weight tile has zero points outside [0, 15]
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
        T.zflag = a.packed[a.flags_off + nt];
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
            T.zflag = a.packed[(size_t)x * a.slab_bytes + a.flags_off + nt];
            return true;
        }
        cum += tiles;
    }
    return false;
}

// The nibble bytes Q (four codes 0..15, one per byte) minus the zero point zc (0..15) as
// sign-magnitude E4M3 subnormal bytes, value (q - zc) * 2^-9, exact for every pair.
// C1 = 0x80808080 - zc * 0x01010101 makes each byte 0x80 + q - zc without inter-byte
// borrows; bit 7 of that byte says q >= zc, where the magnitude is its low 7 bits, otherwise
// the byte is 0x100 - it = 0x80 | (zc - q). prmt with the sign-replicate selector turns bit 7
// of every byte into a byte mask.
__device__ __forceinline__ uint32_t minus_zero_e4m3(uint32_t Q, uint32_t C1) {
    const uint32_t D1 = Q + C1;
    uint32_t P;
    asm("prmt.b32 %0, %1, %1, 0xBA98;" : "=r"(P) : "r"(D1));
    P &= 0x7F7F7F7Fu;
    const uint32_t X = 0x01010100u - D1;
    return (D1 & P) | (X & ~P);
}

__global__ void __launch_bounds__(THREADS, 1) w4a8_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                          const __grid_constant__ CUtensorMap tm_act,
                                                          const __grid_constant__ CUtensorMap tm_sc, const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *raw = base;                                   // STAGES x (codes | activations)
    uint8_t *sA = base + STAGES * RAW_BYTES;               // EXP x expanded weights
    Smem *sm = reinterpret_cast<Smem *>(base + STAGES * RAW_BYTES + EXP * A_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t total_tiles = (int64_t)a.MTU * a.NT;
    const int GPS = BK / a.g;      // groups per raw stage
    const int KPG = a.g / 32;      // f8 MMAs (K = 32 each) per group
    const int J = (int)(a.Kpad / a.g);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 1);
        }
        for (int e = 0; e < EXP; ++e) {
            mbar_init(&sm->exp_full[e], 128);
            mbar_init(&sm->exp_empty[e], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], 256);
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

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 64;\n" ::: "memory");
        if (warp == 0 && lane == 0) {
            // ------------------------------------------------ TMA producer
            int64_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                Tile T;
                if (!locate_tile(a, t, T)) continue;
                const int SPT = a.KT + (T.zflag ? a.ZT : 0);  // pipeline stages of this tile
                for (int s = 0; s < SPT; ++s, ++it) {
                    const int slot = (int)(it % STAGES);
                    // wait for the slot's previous use on every use, including the zero-point
                    // pseudo-stages the expansion warps fill: a parity wait can only tell phases
                    // apart one ring cycle back, so skipping uses would let this thread lap the ring
                    if (!wait_phase(&sm->empty[slot], ((uint32_t)(it / STAGES) & 1) ^ 1, sm, a.status)) { ok = false; break; }
                    if (s >= a.KT) continue;
                    uint8_t *dst = raw + slot * RAW_BYTES;
                    mbar_arrive_expect_tx(&sm->full[slot], C_BYTES + B_BYTES + (uint32_t)GPS * BM * 4);
                    tma_load_3d(dst, &tm_codes, s * (BK / 2), (int)T.n0, T.e, &sm->full[slot]);
                    tma_load_2d(dst + C_BYTES, &tm_act, s * BK, (int)T.row0, &sm->full[slot]);
                    tma_load_3d(dst + C_BYTES + B_BYTES, &tm_sc, (int)T.n0, s * GPS, T.e, &sm->full[slot]);
                }
            }
            // tail: every stage released, so no commit-arrive lands after this CTA exits
            for (int64_t u = it > STAGES ? it - STAGES : 0; u < it && ok; ++u)
                if (!wait_phase(&sm->empty[u % STAGES], (uint32_t)(u / STAGES) & 1, sm, a.status)) break;
        } else if (warp == 1 && lane == 0) {
            // ------------------------------------------------ MMA issuer
            int64_t it = 0, jg = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                Tile T;
                if (!locate_tile(a, t, T)) continue;
                const int SPT = a.KT + (T.zflag ? a.ZT : 0);
                for (int s = 0; s < SPT && ok; ++s, ++it) {
                    const int slot = (int)(it % STAGES), eb = (int)(it % EXP);
                    if (s < a.KT) {
                        if (!wait_phase(&sm->full[slot], (uint32_t)(it / STAGES) & 1, sm, a.status)) { ok = false; break; }
                    } else {
                        // a pseudo-stage is written by the expansion warps (their exp_full arrival
                        // covers both operands); complete this use of the raw slot's "full" phase
                        // here so that its phase count stays one per use
                        mbar_arrive(&sm->full[slot]);
                    }
                    if (!wait_phase(&sm->exp_full[eb], (uint32_t)(it / EXP) & 1, sm, a.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_addr(sA + eb * A_BYTES);
                    const uint32_t b_addr = smem_addr(raw + slot * RAW_BYTES + C_BYTES);
                    if (s < a.KT) {
                        for (int gi = 0; gi < GPS; ++gi, ++jg) {
                            const int b = (int)(jg % NBUF);
                            if (!wait_phase(&sm->acc_empty[b], ((uint32_t)(jg / NBUF) & 1) ^ 1, sm, a.status)) { ok = false; break; }
                            tc_fence_after();
                            for (int kk = 0; kk < KPG; ++kk) {
                                const uint32_t koff = (uint32_t)(gi * KPG + kk) * 32;
                                mma_f8(tmem + (uint32_t)(b * BN), sw128_desc(a_addr + koff), sw128_desc(b_addr + koff),
                                       kk > 0 ? 1u : 0u);
                            }
                            mma_commit(&sm->acc_full[b]);
                        }
                    } else {
                        // zero-point term: all pseudo-stages of the tile accumulate into one buffer
                        const int z = s - a.KT;
                        const int b = (int)(jg % NBUF);
                        if (z == 0 && !wait_phase(&sm->acc_empty[b], ((uint32_t)(jg / NBUF) & 1) ^ 1, sm, a.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        for (int kk = 0; kk < ZK / 16; ++kk)
                            mma_bf16(tmem + (uint32_t)(b * BN), sw128_desc(a_addr + kk * 32), sw128_desc(b_addr + kk * 32),
                                     (z > 0 || kk > 0) ? 1u : 0u);
                        if (z == a.ZT - 1) {
                            mma_commit(&sm->acc_full[b]);
                            ++jg;
                        }
                    }
                    if (!ok) break;
                    mma_commit(&sm->empty[slot]);
                    mma_commit(&sm->exp_empty[eb]);
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
        for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
            Tile T;
            if (!locate_tile(a, t, T)) continue;
            const int64_t n = T.n0 + row;
            const uint32_t *scales =
                reinterpret_cast<const uint32_t *>(a.packed + (size_t)T.e * a.slab_bytes + a.codes_bytes);
            float acc[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            const int JG = J + (T.zflag ? 1 : 0);  // groups, plus the zero-point term if any
            uint32_t ent0 = scales[n], ent1 = (J > 1) ? scales[a.Npad + n] : 0u;
            for (int j = 0; j < JG && ok; ++j, ++jg) {
                const int b = (int)(jg % NBUF);
                float s512 = -1.0f;  // the zero-point term is subtracted
                if (j < J) {
                    s512 = __half2float(__ushort_as_half((unsigned short)(ent0 & 0xFFFF))) * 512.0f;
                    ent0 = ent1;
                    ent1 = (j + 2 < J) ? scales[(int64_t)(j + 2) * a.Npad + n] : 0u;
                }
                if (!wait_phase(&sm->acc_full[b], (uint32_t)(jg / NBUF) & 1, sm, a.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN + half * 128);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t p[32];
                    tmem_ld32(taddr + c * 32, p);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[c * 32 + i] = fmaf(s512, __uint_as_float(p[i]), acc[c * 32 + i]);
                }
                tc_fence_before();
                mbar_arrive(&sm->acc_empty[b]);
            }
            if (!ok) break;
            if (n < a.N) {
#pragma unroll
                for (int i = 0; i < 128; ++i) {
                    const int col = half * 128 + i;
                    if (col < T.rows) {
                        const int64_t m = T.row0 + col;
                        if (m < a.M) {
                            const float v = acc[i] * __ldg(a.row_scale + m);
                            if (a.out_fp32) static_cast<float *>(a.Y)[m * a.N + n] = v;
                            else static_cast<__nv_bfloat16 *>(a.Y)[m * a.N + n] = __float2bfloat16_rn(v);
                        }
                    }
                }
            }
        }
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 64;\n" ::: "memory");
        // ------------------------------------------------ expansion warps
        const int et = threadIdx.x - 384;  // 0..127
        int64_t it = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
            Tile T;
            if (!locate_tile(a, t, T)) continue;
            const uint32_t *scales =
                reinterpret_cast<const uint32_t *>(a.packed + (size_t)T.e * a.slab_bytes + a.codes_bytes);
            const int SPT = a.KT + (T.zflag ? a.ZT : 0);
            for (int s = 0; s < SPT; ++s, ++it) {
                const int slot = (int)(it % STAGES), eb = (int)(it % EXP);
                if (!wait_phase(&sm->exp_empty[eb], ((uint32_t)(it / EXP) & 1) ^ 1, sm, a.status)) { ok = false; break; }
                uint8_t *dstA = sA + eb * A_BYTES;
                if (s < a.KT) {
                    if (!wait_phase(&sm->full[slot], (uint32_t)(it / STAGES) & 1, sm, a.status)) { ok = false; break; }
                    const uint8_t *src = raw + slot * RAW_BYTES;
                    const uint32_t *ssc = reinterpret_cast<const uint32_t *>(src + C_BYTES + B_BYTES);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int idx = et + 128 * i;  // 0..511
                        const int r = idx >> 2, p = idx & 3;
                        const uint4 w = *reinterpret_cast<const uint4 *>(src + r * 64 + p * 16);
                        // zero point of (row r, the group of this 32-wide part), clamped to [0, 15];
                        // the remainder z - zc of flagged tiles goes through the correction term
                        const int z = (int)(int16_t)(ssc[((p * 32) / a.g) * BM + r] >> 16);
                        const uint32_t zc = (uint32_t)min(max(z, 0), 15);
                        const uint32_t C1 = 0x80808080u - zc * 0x01010101u;
                        uint4 o0, o1;
                        o0.x = minus_zero_e4m3(w.x & 0x0F0F0F0Fu, C1); o0.y = minus_zero_e4m3((w.x >> 4) & 0x0F0F0F0Fu, C1);
                        o0.z = minus_zero_e4m3(w.y & 0x0F0F0F0Fu, C1); o0.w = minus_zero_e4m3((w.y >> 4) & 0x0F0F0F0Fu, C1);
                        o1.x = minus_zero_e4m3(w.z & 0x0F0F0F0Fu, C1); o1.y = minus_zero_e4m3((w.z >> 4) & 0x0F0F0F0Fu, C1);
                        o1.z = minus_zero_e4m3(w.w & 0x0F0F0F0Fu, C1); o1.w = minus_zero_e4m3((w.w >> 4) & 0x0F0F0F0Fu, C1);
                        const int c0 = (2 * p) ^ (r & 7), c1 = (2 * p + 1) ^ (r & 7);
                        *reinterpret_cast<uint4 *>(dstA + r * 128 + c0 * 16) = o0;
                        *reinterpret_cast<uint4 *>(dstA + r * 128 + c1 * 16) = o1;
                    }
                } else {
                    // zero-point pseudo-stage z: columns kk = 64z .. 64z+63 of [hi|hi|lo](s z) x [hi|lo|hi](G)
                    // the MMA released this raw slot's previous use
                    const bool got = wait_phase(&sm->empty[slot], ((uint32_t)(it / STAGES) & 1) ^ 1, sm, a.status);
                    if (got) {
                        const int z = s - a.KT;
                        uint8_t *dstB = raw + slot * RAW_BYTES + C_BYTES;
                        const int Jr = a.Jr;
                        // A': weight row n = n0 + et, 64 bf16, written 8 at a time
                        const int64_t n = T.n0 + et;
#pragma unroll 1
                        for (int c = 0; c < 8; ++c) {
                            uint32_t wv[4];
#pragma unroll
                            for (int q2 = 0; q2 < 4; ++q2) {
                                uint32_t v2[2];
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const int kk = z * ZK + c * 8 + q2 * 2 + h;
                                    const int part = kk / Jr, j = kk - part * Jr;
                                    uint32_t v = 0;
                                    if (part < 3) {
                                        const uint32_t en = scales[(int64_t)j * a.Npad + n];
                                        const float sc = __half2float(__ushort_as_half((unsigned short)(en & 0xFFFF)));
                                        const int zz = (int)(int16_t)(en >> 16);
                                        const float sz = sc * (float)(zz - min(max(zz, 0), 15));
                                        const uint32_t hi = bf16_bits_rn(sz);
                                        v = (part < 2) ? hi : bf16_bits_rn(sz - __uint_as_float(hi << 16));
                                    }
                                    v2[h] = v;
                                }
                                wv[q2] = v2[0] | (v2[1] << 16);
                            }
                            *reinterpret_cast<uint4 *>(dstA + et * 128 + ((c ^ (et & 7)) * 16)) =
                                make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        }
                        // B': tokens row0 + et and row0 + et + 128, 64 bf16 each
#pragma unroll 1
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const int r = et + 128 * h2;
                            const int64_t m = T.row0 + r;
                            const bool live = r < T.rows && m < a.M;
#pragma unroll 1
                            for (int c = 0; c < 8; ++c) {
                                uint32_t wv[4];
#pragma unroll
                                for (int q2 = 0; q2 < 4; ++q2) {
                                    uint32_t v2[2];
#pragma unroll
                                    for (int h = 0; h < 2; ++h) {
                                        const int kk = z * ZK + c * 8 + q2 * 2 + h;
                                        const int part = kk / Jr, j = kk - part * Jr;
                                        uint32_t v = 0;
                                        if (live && part < 3) {
                                            const float gv = __ldg(a.gsum + m * Jr + j);
                                            const uint32_t hi = bf16_bits_rn(gv);
                                            v = (part == 1) ? bf16_bits_rn(gv - __uint_as_float(hi << 16)) : hi;
                                        }
                                        v2[h] = v;
                                    }
                                    wv[q2] = v2[0] | (v2[1] << 16);
                                }
                                *reinterpret_cast<uint4 *>(dstB + r * 128 + ((c ^ (r & 7)) * 16)) =
                                    make_uint4(wv[0], wv[1], wv[2], wv[3]);
                            }
                        }
                    }
                    if (!got) { ok = false; break; }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(&sm->exp_full[eb]);
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

static w4_status launch(const uint8_t *X8, const float *row_scale, const float *gsum, const int32_t *offsets, int E,
                        int64_t M, const void *packed, int64_t N, int64_t K, int group, void *Y, int out_fp32,
                        cudaStream_t stream) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return W4_ERR_CUDA;
    const GemmLayout L = gemm_layout(N, K, group);
    CUtensorMap tm_codes, tm_act;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)(L.Kpad / 2), (cuuint64_t)L.Npad, (cuuint64_t)E};
        const cuuint64_t strides[2] = {(cuuint64_t)(L.Kpad / 2), (cuuint64_t)L.total};
        const cuuint32_t box[3] = {BK / 2, BM, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(packed), dims, strides, box, es,
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
    CUtensorMap tm_sc;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)L.Npad, (cuuint64_t)L.J, (cuuint64_t)E};
        const cuuint64_t strides[2] = {(cuuint64_t)(L.Npad * 4), (cuuint64_t)L.total};
        const cuuint32_t box[3] = {BM, (cuuint32_t)(BK / group), 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tm_sc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3,
                const_cast<uint8_t *>(static_cast<const uint8_t *>(packed) + L.codes_bytes), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return W4_ERR_CUDA;
    }
    Args a;
    a.packed = static_cast<const uint8_t *>(packed);
    a.slab_bytes = L.total;
    a.flags_off = L.codes_bytes + L.scales_bytes;
    a.codes_bytes = L.codes_bytes;
    a.row_scale = row_scale;
    a.gsum = gsum;
    a.offsets = offsets;
    a.Y = Y;
    a.status = device_status_ptr();
    a.M = M; a.N = N; a.Npad = L.Npad; a.K = K; a.Kpad = L.Kpad;
    a.E = E; a.g = group; a.Jr = (int)(K / group); a.out_fp32 = out_fp32;
    a.NT = (int)(L.Npad / BM);
    const int64_t mtu = offsets ? (M + BN - 1) / BN + E : (M + BN - 1) / BN;
    if (mtu > 0x7fffffffLL) return W4_ERR_SHAPE;
    a.MTU = (int)mtu;
    a.KT = (int)(L.Kpad / BK);
    a.ZT = (int)((3 * a.Jr + ZK - 1) / ZK);
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(w4a8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
            cudaSuccess)
            return W4_ERR_CUDA;
        attr_done[dev] = 1;
    }
    const int64_t tiles = mtu * a.NT;
    const int grid = (int)(tiles < sm_count_cached() ? tiles : sm_count_cached());
    w4a8_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(tm_codes, tm_act, tm_sc, a);
    return launch_status();
}

}  // namespace gemm
}  // namespace w4

using namespace w4;

W4_API w4_status w4a8_gemm(const uint8_t *X_e4m3, const float *row_scale, const float *group_sums, int64_t M,
                           const void *packed, int64_t N, int64_t K, int group, int mode, void *Y, int out_fp32,
                           cudaStream_t stream) {
    if (!X_e4m3 || !row_scale || !group_sums || !packed || !Y) return W4_ERR_NULL;
    if (!valid_mode(mode) || (out_fp32 != 0 && out_fp32 != 1)) return W4_ERR_ARG;
    if (M < 1 || M > 0x7fffffffLL || N < 1 || N > 0x7fffffffLL || K < 128 || K % 32 != 0 || K > (1LL << 24))
        return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(X_e4m3) || !aligned16(row_scale) || !aligned16(group_sums) || !aligned16(packed) || !aligned16(Y))
        return W4_ERR_ALIGN;
    return gemm::launch(X_e4m3, row_scale, group_sums, nullptr, 1, M, packed, N, K, group, Y, out_fp32, stream);
}

W4_API w4_status w4a8_grouped_gemm(const uint8_t *X_e4m3, const float *row_scale, const float *group_sums,
                                   const int32_t *expert_row_offsets, int E, int64_t M_total, const void *packed,
                                   int64_t N, int64_t K, int group, int mode, void *Y, cudaStream_t stream) {
    if (!X_e4m3 || !row_scale || !group_sums || !expert_row_offsets || !packed || !Y) return W4_ERR_NULL;
    if (!valid_mode(mode)) return W4_ERR_ARG;
    if (E < 1 || E > 1024 || M_total < 1 || M_total > 0x7fffffffLL || N < 1 || N > 0x7fffffffLL || K < 128 ||
        K % 32 != 0 || K > (1LL << 24))
        return W4_ERR_SHAPE;
    if (!valid_group(group) || K % group != 0) return W4_ERR_GROUP;
    if (!aligned16(X_e4m3) || !aligned16(row_scale) || !aligned16(group_sums) || !aligned16(packed) ||
        !aligned16(Y) || (reinterpret_cast<uintptr_t>(expert_row_offsets) & 3))
        return W4_ERR_ALIGN;
    return gemm::launch(X_e4m3, row_scale, group_sums, expert_row_offsets, E, M_total, packed, N, K, group, Y, 0,
                        stream);
}
