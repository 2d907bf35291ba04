// w4a8_gemm / w4a8_grouped_gemm: INT4 weights x FP8 E4M3 activations on the sm_100a
// tensor cores (tcgen05.mma kind::f8f6f4, TMEM accumulators, TMA operand loads).
//
// "Four-bit inference ... Tahoma", Achievement 2 (the W4A8 dataflow: packed 4-bit weights
// read from HBM, expanded to E4M3 inside the GEMM, FP8 tensor-core MMA with FP32
// accumulation, per-token activation scale in the epilogue, BF16 result) and
// "4-bit by default" (mixture-of-experts weights are the 4-bit target).
//
//   Y[m, n] = s_a[m] * sum_j s[n,j] * ( sum_{k in j} a8[m,k] * q[n,k]  -  z[n,j] * G[m,j] )
//
// with G[m,j] = sum_{k in j} a8[m,k] from fp8_row_quant. Design:
//  * swap-AB: the weight tile is the MMA's A operand (M = 128 weight rows, one TMEM lane
//    per weight row) and 128 tokens are its N; so each epilogue thread owns one weight row
//    and its group scale is a per-thread scalar;
//  * expansion: a nibble q in [0, 15] zero-extended to a byte IS the E4M3 pattern of
//    q * 2^-9 (exponent field 0/1 gives the integer grid m * 2^-9, m = 0..15), so the
//    weights enter the MMA exactly and the expansion is two AND/shift ops per 8 weights;
//    the 2^9 goes into the group scale (512 * s is exact);
//  * per group j the MMA accumulates sum a8 * q * 2^-9 over the group into one of two TMEM
//    buffers; the epilogue warps read it (tcgen05.ld) and promote it into fp32 registers
//    with the group scale while the MMA fills the other buffer;
//  * the zero point is applied once per group through G (a rank-J correction done at the
//    end of the tile on the CUDA cores);
//  * warp roles: warp 0 TMA producer, warp 1 TMEM owner + single-thread MMA issuer,
//    warps 2-5 epilogue (TMEM lane quarters 2,3,0,1), warps 6-9 expansion;
//  * every mbarrier wait is bounded (wall clock); on expiry the kernel records
//    W4_ERR_TIMEOUT, the other roles see the abort flag, TMEM is freed and the CTA returns.
#include "w4_common.cuh"
#include "w4_layout.cuh"

#include <cuda.h>

namespace w4 {
namespace gemm {

constexpr int BM = 128;       // weight rows per tile (MMA M)
constexpr int BN = 128;       // tokens per tile (MMA N)
constexpr int BK = 128;       // k per pipeline stage (one 128-byte swizzle row of E4M3)
constexpr int STAGES = 4;
constexpr int NBUF = 2;       // TMEM accumulator buffers
constexpr int TMEM_COLS = 256;
constexpr int THREADS = 320;
constexpr uint32_t A_BYTES = BM * BK;       // expanded weights, E4M3
constexpr uint32_t B_BYTES = BN * BK;       // activations, E4M3
constexpr uint32_t C_BYTES = BM * BK / 2;   // packed codes
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*barriers*/ + 1024 /*alignment*/;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait

struct Smem {
    uint64_t full_tma[STAGES];
    uint64_t full_exp[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[NBUF];
    uint64_t acc_empty[NBUF];
    uint32_t tmem_base;
    int abort;
    int epi_go;
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
    int n_tiles_n;                 // Npad / BM
};

__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, Smem *sm, int *status) {
    return mbar_wait_abortable(bar, parity, &sm->abort, status, kWaitNs);
}

// K-major operand descriptor, 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes
// apart (stride byte offset), leading byte offset 16 bytes, descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// instruction descriptor: D fp32, A and B E4M3, both K-major, N = BN, M = BM
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
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

// Find the (expert, first row, rows) of this CTA's token tile; false if past the last tile.
__device__ __forceinline__ bool locate_tile(const Args &a, int t, int &e, int64_t &row0, int64_t &rows) {
    if (!a.offsets) {
        e = 0;
        row0 = (int64_t)t * BN;
        rows = a.M - row0;
        return row0 < a.M;
    }
    int cum = 0;
    for (int x = 0; x < a.E; ++x) {
        const int64_t lo = a.offsets[x], hi = a.offsets[x + 1];
        const int tiles = (int)((hi - lo + BN - 1) / BN);
        if (t < cum + tiles) {
            e = x;
            row0 = lo + (int64_t)(t - cum) * BN;
            rows = hi - row0;
            return true;
        }
        cum += tiles;
    }
    return false;
}

__global__ void __launch_bounds__(THREADS, 1) w4a8_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                          const __grid_constant__ CUtensorMap tm_act, const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = base + STAGES * A_BYTES;
    uint8_t *sC = base + STAGES * (A_BYTES + B_BYTES);
    Smem *sm = reinterpret_cast<Smem *>(base + STAGES * STAGE_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int e;
    int64_t row0, rows;
    if (!locate_tile(a, blockIdx.y, e, row0, rows)) return;  // uniform across the CTA
    const int64_t n0 = (int64_t)blockIdx.x * BM;
    const int KT = (int)(a.Kpad / BK);
    const int J = (int)(a.Kpad / a.g);
    const int GPS = BK / a.g;       // groups per stage
    const int KPG = a.g / 32;       // MMAs (K = 32 each) per group

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm->full_tma[s], 1);
            mbar_init(&sm->full_exp[s], 128);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], 128);
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
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (kt / STAGES) & 1;
                if (!wait_phase(&sm->empty[s], ph ^ 1, sm, a.status)) break;
                mbar_arrive_expect_tx(&sm->full_tma[s], C_BYTES + B_BYTES);
                tma_load_3d(sC + s * C_BYTES, &tm_codes, kt * (BK / 2), (int)n0, e, &sm->full_tma[s]);
                tma_load_2d(sB + s * B_BYTES, &tm_act, kt * BK, (int)row0, &sm->full_tma[s]);
            }
            // tail: wait until the MMA released the last stages, so that no commit-arrive can
            // land in this CTA's shared memory after it exits
            for (int kt = KT > STAGES ? KT - STAGES : 0; kt < KT; ++kt)
                if (!wait_phase(&sm->empty[kt % STAGES], (kt / STAGES) & 1, sm, a.status)) break;
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int jg = 0;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (kt / STAGES) & 1;
                if (!wait_phase(&sm->full_exp[s], ph, sm, a.status)) break;
                if (!wait_phase(&sm->full_tma[s], ph, sm, a.status)) break;
                tc_fence_after();
                const uint32_t a_addr = smem_addr(sA + s * A_BYTES);
                const uint32_t b_addr = smem_addr(sB + s * B_BYTES);
                bool ok = true;
                for (int gi = 0; gi < GPS; ++gi, ++jg) {
                    const int b = jg % NBUF;
                    if (!wait_phase(&sm->acc_empty[b], ((jg / NBUF) & 1) ^ 1, sm, a.status)) { ok = false; break; }
                    tc_fence_after();
                    for (int kk = 0; kk < KPG; ++kk) {
                        const uint32_t koff = (uint32_t)(gi * KPG + kk) * 32;
                        mma_f8(tmem + (uint32_t)(b * BN), sw128_desc(a_addr + koff), sw128_desc(b_addr + koff),
                               kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sm->acc_full[b]);
                }
                if (!ok) break;
                mma_commit(&sm->empty[s]);
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------ epilogue (promotion) warps
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int64_t n = n0 + row;
        const uint32_t *scales = reinterpret_cast<const uint32_t *>(a.packed + (size_t)e * a.slab_bytes + a.codes_bytes);
        float acc[BN];
#pragma unroll
        for (int i = 0; i < BN; ++i) acc[i] = 0.0f;
        uint32_t ent = scales[n];  // group 0
        bool ok = true;
        for (int j = 0; j < J; ++j) {
            const int b = j % NBUF;
            const uint32_t ent_next = (j + 1 < J) ? scales[(int64_t)(j + 1) * a.Npad + n] : 0u;
            const float s512 = __half2float(__ushort_as_half((unsigned short)(ent & 0xFFFF))) * 512.0f;
            if (!wait_phase(&sm->acc_full[b], (j / NBUF) & 1, sm, a.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN);
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                float p[32];
                tmem_ld32(taddr + c * 32, p);
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[c * 32 + i] = fmaf(s512, p[i], acc[c * 32 + i]);
            }
            tc_fence_before();
            mbar_arrive(&sm->acc_empty[b]);
            ent = ent_next;
        }
        // zero-point term: acc[i] -= sum_j s[n,j] z[n,j] G[m_i, j], G staged transposed in sB.
        // A failed wait sets the abort flag before its thread reaches this barrier, so one
        // thread's read after it decides for all 128 (named barriers need all of them).
        (void)ok;
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) sm->epi_go = !*(volatile int *)&sm->abort;
        named_bar_sync(1, 128);
        if (*(volatile int *)&sm->epi_go) {
            float *gt = reinterpret_cast<float *>(sB);
            const int JC = (int)((STAGES * B_BYTES) / (BN * 4));  // groups per staging round
            const int et = threadIdx.x - 64;                      // 0..127
            for (int j0 = 0; j0 < a.Jr; j0 += JC) {
                const int jn = min(JC, a.Jr - j0);
                for (int idx = et; idx < jn * BN; idx += 128) {
                    const int jj = idx / BN, i = idx - jj * BN;
                    gt[idx] = (i < rows && row0 + i < a.M) ? a.gsum[(row0 + i) * a.Jr + j0 + jj] : 0.0f;
                }
                named_bar_sync(1, 128);
                for (int jj = 0; jj < jn; ++jj) {
                    const uint32_t en = scales[(int64_t)(j0 + jj) * a.Npad + n];
                    const float s = __half2float(__ushort_as_half((unsigned short)(en & 0xFFFF)));
                    const float nsz = -(s * (float)(int)(int16_t)(en >> 16));
                    const float4 *gr = reinterpret_cast<const float4 *>(gt + jj * BN);
#pragma unroll
                    for (int i4 = 0; i4 < BN / 4; ++i4) {
                        const float4 gv = gr[i4];
                        acc[4 * i4 + 0] = fmaf(nsz, gv.x, acc[4 * i4 + 0]);
                        acc[4 * i4 + 1] = fmaf(nsz, gv.y, acc[4 * i4 + 1]);
                        acc[4 * i4 + 2] = fmaf(nsz, gv.z, acc[4 * i4 + 2]);
                        acc[4 * i4 + 3] = fmaf(nsz, gv.w, acc[4 * i4 + 3]);
                    }
                }
                named_bar_sync(1, 128);
            }
            // per-token scale and store
            if (n < a.N) {
#pragma unroll
                for (int i = 0; i < BN; ++i) {
                    if (i < rows) {
                        const int64_t m = row0 + i;
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
        // ------------------------------------------------ expansion warps: nibbles -> E4M3 bytes
        const int et = threadIdx.x - 192;  // 0..127
        for (int kt = 0; kt < KT; ++kt) {
            const int s = kt % STAGES;
            const uint32_t ph = (kt / STAGES) & 1;
            if (!wait_phase(&sm->full_tma[s], ph, sm, a.status)) break;
            const uint8_t *src = sC + s * C_BYTES;
            uint8_t *dst = sA + s * A_BYTES;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int idx = et + 128 * i;  // 0..511
                const int r = idx >> 2, p = idx & 3;
                const uint4 w = *reinterpret_cast<const uint4 *>(src + r * 64 + p * 16);
                uint4 o0, o1;
                o0.x = w.x & 0x0F0F0F0Fu; o0.y = (w.x >> 4) & 0x0F0F0F0Fu;
                o0.z = w.y & 0x0F0F0F0Fu; o0.w = (w.y >> 4) & 0x0F0F0F0Fu;
                o1.x = w.z & 0x0F0F0F0Fu; o1.y = (w.z >> 4) & 0x0F0F0F0Fu;
                o1.z = w.w & 0x0F0F0F0Fu; o1.w = (w.w >> 4) & 0x0F0F0F0Fu;
                const int c0 = (2 * p) ^ (r & 7), c1 = (2 * p + 1) ^ (r & 7);
                *reinterpret_cast<uint4 *>(dst + r * 128 + c0 * 16) = o0;
                *reinterpret_cast<uint4 *>(dst + r * 128 + c1 * 16) = o1;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&sm->full_exp[s]);
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
    Args a;
    a.packed = static_cast<const uint8_t *>(packed);
    a.slab_bytes = L.total;
    a.codes_bytes = L.codes_bytes;
    a.row_scale = row_scale;
    a.gsum = gsum;
    a.offsets = offsets;
    a.Y = Y;
    a.status = device_status_ptr();
    a.M = M; a.N = N; a.Npad = L.Npad; a.K = K; a.Kpad = L.Kpad;
    a.E = E; a.g = group; a.Jr = (int)(K / group); a.out_fp32 = out_fp32;
    a.n_tiles_n = (int)(L.Npad / BM);
    const int64_t m_tiles = offsets ? (M + BN - 1) / BN + E : (M + BN - 1) / BN;
    if (m_tiles > 65535) return W4_ERR_SHAPE;
    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(w4a8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
            cudaSuccess)
            return W4_ERR_CUDA;
        attr_set = true;
    }
    dim3 grid((unsigned)(L.Npad / BM), (unsigned)m_tiles);
    w4a8_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(tm_codes, tm_act, a);
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
