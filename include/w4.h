/*
 * w4.h -- C ABI of libw4: blockwise 4-bit weight quantization and the matmuls that consume
 * it, for NVIDIA B200 (sm_100a).
 *
 * Conventions for every entry point
 *   - All tensors are dense, row-major and contiguous. Device pointers unless the name says
 *     _host. Every device base pointer must be 16-byte aligned (W4_ERR_ALIGN otherwise).
 *   - The caller allocates and owns every buffer. No entry point allocates, frees or
 *     synchronizes device memory, except w4_device_status(), which synchronizes `stream`.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default stream) and
 *     runs asynchronously. A return of W4_OK means the launch was enqueued.
 *   - Arguments are validated on the host before anything is launched; on any error the
 *     call returns a non-zero w4_status and has no side effect. There is no fallback: an
 *     unsupported shape is an error, never a silently different computation.
 *   - Device-side anomalies (a bounded wait that expired) are recorded in a device status
 *     word that w4_device_status() reads; kernels never trap.
 *
 * Formats
 *   bf16 inputs are raw 16-bit bfloat16 patterns; scales are IEEE binary16 patterns;
 *   zeros are int16; FP8 values are E4M3 ("fn": no infinities, max 448) bytes.
 *
 * Canonical ("portable") quantized weight for W[N, K] and group g (the parity surface):
 *   codes  uint8 [N, K/2]  byte j of row n = q[n, 2j] | q[n, 2j+1] << 4
 *   scales uint16 [N, K/g] fp16 bits, one per group of g consecutive weights along K
 *   zeros  int16 [N, K/g]  integer zero point (asymmetric only)
 *   Symmetric codes are offset-binary: nibble = c + 8 with c in [-7, 7] (nibble 0 unused);
 *   dequantized weight = (nibble - 8) * s. Asymmetric: (q - z) * s with q in [0, 15].
 *
 * Sources: "Quantizing LLMs Without Guesswork: What 4 Bits Really Cost" (QLWG) and
 * "Four-bit inference ... Tahoma" (TAHOMA), sections named per entry point.
 */
#ifndef W4_H_
#define W4_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4_OK = 0,
    W4_ERR_NULL = 1,         /* a required pointer is NULL                              */
    W4_ERR_SHAPE = 2,        /* a size is out of the supported range                   */
    W4_ERR_GROUP = 3,        /* group not in {32,64,128,256} or K not a multiple of it */
    W4_ERR_ALIGN = 4,        /* a device pointer is not 16-byte aligned                */
    W4_ERR_ARG = 5,          /* any other bad argument (mode, clip grid, layout, ...)  */
    W4_ERR_UNSUPPORTED = 6,  /* valid request this library does not implement          */
    W4_ERR_CUDA = 7,         /* a CUDA runtime call failed (launch error)              */
    W4_ERR_TIMEOUT = 8,      /* device status: a bounded wait in a kernel expired      */
    W4_ERR_DEVICE_CHECK = 9, /* device status: a kernel's own consistency check failed */
    W4_ERR_WORKSPACE = 10,   /* workspace missing or smaller than the query says       */
    W4_ERR_SCRATCH_LIMIT = 11 /* request needs more scratch than the allocation-free
                                entry point holds (w4a16_gemv_noalloc_scratch_limit)  */
} w4_status;

typedef enum { W4_SYM = 0, W4_ASYM = 1 } w4_mode;

/* Flags of w4a16_gemv. */
enum {
    W4_OUT_FP32 = 1,        /* write y as fp32 instead of bf16                              */
    W4_OVERLAP_PREVIOUS = 2 /* programmatic dependent launch: the kernel may start while the
                               previous kernel on the stream is finishing; it streams its
                               weights at once and reads x only after that kernel completed */
};

/* Kernel layouts produced by w4_prepack. */
typedef enum { W4_LAYOUT_GEMV = 0, W4_LAYOUT_GEMM = 1, W4_LAYOUT_TC = 2 } w4_layout;

/* Human-readable name of a status code (static storage). */
const char *w4_status_str(int status);

/* Library ABI version (major * 100 + minor). */
int w4_version(void);

/*
 * w4_quantize -- group-wise INT4 quantizer with the data-free MSE clip search.
 *   QLWG "Scale and zero point" (symmetric max|x|/7; asymmetric (max-min)/15 with integer
 *   zero round(-min/s)), "Granularity" (one FP16 scale per g consecutive weights of a row),
 *   "Quantize, then dequantize" (zero-range guard s = 1, round half to even);
 *   TAHOMA "The naive symmetric baseline", "Achievement 1: asymmetric W4", "MSE clipping"
 *   (for each block: every ratio of the grid contracts the range about its midpoint, the
 *   block is quantized and reconstructed, and a ratio replaces the incumbent only with a
 *   strictly smaller block error that includes the clipped weights).
 *
 *   W_bf16         device, bf16 [N, K]
 *   group          32, 64 or 128; K % group == 0; K % 32 == 0
 *   mode           W4_SYM (amax/7, offset-binary codes) or W4_ASYM (scale + zero point)
 *   clip_grid_host HOST, n_clip fp32 ratios in (0, 1], finite; clip_grid_host[0] == 1.0f
 *                  (the incumbent is the full range); 1 <= n_clip <= 64. For W4_SYM the
 *                  ratio scales max|w|; for W4_ASYM it contracts [min, max] about its
 *                  midpoint.
 *   codes          device, uint8 [N, K/2], canonical packing (see above)
 *   scales_fp16    device, uint16 [N, K/group]
 *   zeros          device, int16 [N, K/group]; required for W4_ASYM, must be NULL for W4_SYM
 *   chosen_idx     device, uint8 [N, K/group], index of the winning ratio; may be NULL
 *   Arithmetic: fp32, IEEE division, no FMA contraction, scale rounded to fp16 before the
 *   codes, zero point and block error are formed; block error = sum of squares reduced in a
 *   fixed tree (32 contiguous chunks of group/32 weights summed in order, then pairwise at
 *   distances 16, 8, 4, 2, 1). Results are bit-identical run to run.
 *   Errors: NULL / SHAPE (N < 1, K < 32) / GROUP / ALIGN / ARG (mode, grid, zeros vs mode).
 */
w4_status w4_quantize(const void *W_bf16, int64_t N, int64_t K, int group, int mode,
                      const float *clip_grid_host, int n_clip, uint8_t *codes,
                      uint16_t *scales_fp16, int16_t *zeros, uint8_t *chosen_idx,
                      cudaStream_t stream);

/*
 * w4_prepack_bytes / w4_prepack -- re-layout of a canonical quantized weight into a kernel
 *   layout; no code, scale or zero is dequantized or requantized (TAHOMA "MSE clipping":
 *   portable codes, scales and zero terms are rearranged once into a GPU-specific layout).
 *   W4_LAYOUT_GEMM also stores, after the moved codes and scales, the GEMM's zero-point
 *   operand: bf16 hi/lo parts of s[n,j] * z[n,j] (a function of the scales and zeros, so
 *   the canonical weight stays the only source of truth).
 *   layout W4_LAYOUT_GEMV feeds w4a16_gemv, W4_LAYOUT_GEMM feeds w4a8_gemm and (one slab per
 *   expert) w4a8_grouped_gemm, W4_LAYOUT_TC feeds w4a16_gemm_tc. The packed buffer is opaque; its size is
 *   w4_prepack_bytes(N, K, group, layout) (0 for invalid arguments) and includes padding of
 *   N and K to the kernel tiles. For W4_SYM, zeros must be NULL (z = 8 is implied).
 *   Errors: NULL / SHAPE / GROUP / ALIGN / ARG.
 */
size_t w4_prepack_bytes(int64_t N, int64_t K, int group, int layout);
w4_status w4_prepack(const uint8_t *codes, const uint16_t *scales_fp16, const int16_t *zeros,
                     int64_t N, int64_t K, int group, int mode, int layout, void *packed,
                     cudaStream_t stream);

/*
 * fp8_row_quant -- dynamic per-row FP8 E4M3 activation quantization
 *   (TAHOMA "Achievement 2: 8-bit activations without a calibration set"): for every row m,
 *   amax = max_k |x[m,k]|, s[m] = max(amax, 1e-8f) / 448.0f, X8[m,k] = e4m3(x[m,k] / s[m])
 *   with IEEE fp32 division, round-to-nearest-even and saturation to +-448. An all-zero row
 *   gives all-zero codes.
 *   X_bf16      device, bf16 [M, K]; M >= 1, K >= 16, K % 16 == 0
 *   X_e4m3      device, uint8 [M, K], or NULL when X_f16 is given
 *   row_scale   device, fp32 [M]
 *   group_sums  device, fp32 [M, K/group] or NULL: G[m,j], the sum of the E4M3 VALUES (not
 *               scaled by s[m]) of group j of `group` consecutive codes, summed exactly and
 *               rounded once to fp32.
 *   gsum_op     device, bf16 [M, C] with C = w4a8_gsum_op_cols(K, group), or NULL: the
 *               group-sum operand that w4a8_gemm needs (it applies the weight zero point
 *               through it). With J = K/group, hi = bf16(G[m,j]) and lo = bf16(G[m,j] - hi),
 *               row m holds [hi(0..J-1) | lo(0..J-1) | hi(0..J-1) | 0 ...].
 *   X_f16       device, fp16 [M, K], or NULL: the same E4M3 values as binary16 (exact), the
 *               activation operand w4a8_gemm takes for groups 32 and 256. At least one of
 *               X_e4m3 and X_f16 must be given.
 *   group must be 32, 64, 128 or 256 when group_sums or gsum_op is given.
 *   Errors: NULL / SHAPE / GROUP / ALIGN.
 */
int64_t w4a8_gsum_op_cols(int64_t K, int group); /* 3 K/group rounded up to 32; 0 if invalid */
w4_status fp8_row_quant(const void *X_bf16, int64_t M, int64_t K, int group, uint8_t *X_e4m3,
                        float *row_scale, float *group_sums, uint16_t *gsum_op, uint16_t *X_f16,
                        cudaStream_t stream);

/*
 * fp8_row_quant_gather -- fp8_row_quant of gathered rows: output row m is the quantization of
 *   source row row_index[m] of X (M_src rows). Used to lay out the routed tokens of a
 *   mixture-of-experts layer by expert before the grouped GEMM (each token appears once per
 *   expert that takes it; its codes and scale are those of fp8_row_quant of that token).
 *   row_index   device, int32 [M], values in [0, M_src); an index outside that range is
 *               recorded as W4_ERR_DEVICE_CHECK in the device status and its row is
 *               quantized as zeros.
 *   Other arguments as fp8_row_quant (outputs have M rows). Errors as fp8_row_quant.
 */
w4_status fp8_row_quant_gather(const void *X_bf16, int64_t M_src, int64_t K, int group,
                               const int32_t *row_index, int64_t M, uint8_t *X_e4m3,
                               float *row_scale, float *group_sums, uint16_t *gsum_op,
                               uint16_t *X_f16, cudaStream_t stream);

/*
 * w4a16_gemv -- weight-only INT4 decode GEMV with the dequantization fused into the
 *   product (QLWG "Weight-only methods": 4-bit weights, 16-bit activations, dequantized
 *   inside the matmul; "The Problem & Context": decode reads every weight once and that
 *   read sets the pace):
 *     y[m, n] = sum_j s[n,j] * sum_{k in group j} x[m,k] * (q[n,k] - z[n,j])
 *   The products of the codes with the activations are exact integer sums: each slice of
 *   128 / MT activations (MT = 1, 2 or 4 rows per sweep) is held as 24-bit fixed point with
 *   one exponent per slice, exact for every value within 2^11 of the slice's largest
 *   magnitude and otherwise rounded to 2^-20 of it; fp32 rounding enters only where a group's
 *   integer sum is scaled and where a row is summed. The output is rounded once (to bf16, or
 *   kept fp32). One block per SM takes a contiguous run of rows; rows too long for one block
 *   are split along K and their parts are added, in a fixed order, by the last block to
 *   finish. Results are bit-identical run to run on a given GPU. A slice containing an
 *   infinity or a NaN makes its rows' outputs NaN; slices whose largest magnitude is a bf16
 *   subnormal contribute 0.
 *   x_bf16          device, bf16 [M, K]; 1 <= M <= 16
 *   packed          device, w4_prepack(..., W4_LAYOUT_GEMV) of W[N, K]
 *   y               device, bf16 [M, N], or fp32 [M, N] with W4_OUT_FP32 in flags
 *   flags           W4_OUT_FP32 | W4_OVERLAP_PREVIOUS (see the enum); other bits: W4_ERR_ARG
 *   workspace       device scratch of at least w4a16_gemv_workspace_bytes(N, K, group) bytes;
 *                   that query returns 0 for shapes whose rows fit one block (K up to about
 *                   40,000 at M = 1), and then workspace may be NULL. It must be zero-filled
 *                   before its first use; every call that completes leaves it zero-filled
 *                   again, so one workspace can serve any sequence of calls on one stream.
 *                   Calls that may run concurrently on the GPU need separate workspaces.
 *                   After a call whose kernel recorded an error in the device status,
 *                   zero-fill it again.
 *   Errors: NULL / SHAPE (M outside 1..16, N < 1 or N > 2^31, K < 32, K > 2^24, K % 32) /
 *   GROUP / ALIGN / ARG / WORKSPACE (needed and missing or too small).
 */
size_t w4a16_gemv_workspace_bytes(int64_t N, int64_t K, int group);

/*
 * w4a16_gemv_schedule -- host-only query (no GPU call): how w4a16_gemv divides the problem
 *   (M rows, N, K, group) over `sms` SMs (1 .. 4096), by the same planner the launch uses.
 *   out[8] receives: activation rows per sweep over the weights (1, 2 or 4), sweeps, K parts
 *   per row (1 = whole rows per block), row blocks, rows per block, dynamic shared memory
 *   bytes per block, shared-memory ring stages, workspace bytes this call needs.
 *   Errors: NULL / SHAPE / GROUP.
 */
w4_status w4a16_gemv_schedule(int64_t M, int64_t N, int64_t K, int group, int sms, int64_t *out);

w4_status w4a16_gemv(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K,
                     int group, int mode, void *y, int flags, void *workspace,
                     size_t workspace_bytes, cudaStream_t stream);

/*
 * w4a16_gemv_prefetch_next -- w4a16_gemv (same arguments, same results, bit for bit) that also
 *   names the weights the next GEMV on the stream will read: `next_bytes` bytes at `next`
 *   (device memory, 16-byte aligned; a trailing partial 16 bytes is not touched). Each block,
 *   once all of its own weight rows have been requested, issues L2 prefetches of its share of
 *   that range (no copy into shared memory, no wait), so that HBM reads them while this launch
 *   converts its activations, adds its row sums and exits; the next launch then streams them
 *   from L2. A decode step whose GEMVs each name their successor's weights keeps HBM busy
 *   across the launch boundaries ("The Problem & Context": decode reads every weight once per
 *   token). Every weight byte is still read from HBM once. next may be NULL with next_bytes 0
 *   (then this is w4a16_gemv). Errors: as w4a16_gemv, and NULL (next NULL with next_bytes > 0)
 *   and ALIGN (next not 16-byte aligned).
 */
w4_status w4a16_gemv_prefetch_next(const void *x_bf16, int64_t M, const void *packed, int64_t N,
                                   int64_t K, int group, int mode, void *y, int flags,
                                   void *workspace, size_t workspace_bytes, const void *next,
                                   size_t next_bytes, cudaStream_t stream);

/*
 * w4a16_gemv_grouped -- `count` independent w4a16_gemv problems in one launch (for example the
 *   q, k and v projections of a layer, or its gate and up projections, which read the same
 *   activations): problem j computes y[j] = x[j] W_j^T exactly as w4a16_gemv does, with the
 *   same M, group and mode for all. Each problem gets a share of the SMs in proportion to its
 *   weight bytes and whole weight rows per block, so the launch's fixed phases (activation
 *   conversion, first stage, row sums) are paid once for the group.
 *   x_bf16, packed, y   HOST arrays of `count` device pointers (layouts as w4a16_gemv)
 *   N, K                HOST arrays of `count` sizes
 *   1 <= count <= 8; flags as w4a16_gemv. No workspace: every problem's rows must fit one
 *   block's K range (K <= 57344 at M = 1, as for w4a16_gemv without a workspace), and all
 *   problems must take the same activation rows per sweep. Errors: NULL / SHAPE / GROUP / ARG /
 *   ALIGN / UNSUPPORTED (a group the planner cannot place) / CUDA.
 *
 * w4a16_gemv_grouped_schedule -- host-only query: blocks[j] receives the blocks of problem j in
 *   such a launch on `sms` SMs. Errors: NULL / SHAPE / GROUP / UNSUPPORTED.
 */
w4_status w4a16_gemv_grouped(int count, const void *const *x_bf16, int64_t M,
                             const void *const *packed, const int64_t *N, const int64_t *K,
                             int group, int mode, void *const *y, int flags, cudaStream_t stream);
w4_status w4a16_gemv_grouped_schedule(int count, int64_t M, const int64_t *N, const int64_t *K,
                                      int group, int sms, int64_t *blocks);

/*
 * w4a16_gemv_noalloc -- w4a16_gemv for callers that cannot allocate device memory.
 *   (No counterpart in the source pages: this is a calling convention, not part of the
 *   method.) Some callers must not call cudaMalloc on their hot path: a plug-in running
 *   inside another runtime that owns all device memory, or a latency-critical decode loop
 *   in which cudaMalloc's implicit device synchronisation is not acceptable. This entry
 *   point computes exactly what w4a16_gemv computes (same kernel, same partition, same
 *   result bits) but keeps its scratch (the partial sums of rows split along K) in a fixed
 *   array of w4a16_gemv_noalloc_scratch_limit() bytes (1 MiB) inside the library's device
 *   memory; every GPU that loads the library holds that array until the process exits. The
 *   caller still passes x, packed and y.
 *   Behaviour:
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call on a device looks up the array's device address; make that first call
 *     before any stream capture on that device.
 *   - Each call clears the arrival counters it needs (cudaMemsetAsync on `stream`) before its
 *     kernel, because the array keeps the previous call's contents.
 *   - All calls share the one array: calls on different streams that may run at the same
 *     time race on it and give wrong results. Serialise them, or use w4a16_gemv with
 *     separate workspaces. On one stream, a call that uses the array starts with its memset,
 *     which waits for the stream's previous kernel, so W4_OVERLAP_PREVIOUS never overlaps
 *     such a call with the call before it.
 *   - Only rows split along K (K beyond about 40,000 at M = 1) use the scratch: such a call
 *     needs K_parts * M * N * 4 bytes of partial sums plus 4 bytes per row block and sweep,
 *     the workspace_bytes that w4a16_gemv_schedule reports. A request above the limit returns
 *     W4_ERR_SCRATCH_LIMIT without launching anything.
 *   Arguments and other errors as w4a16_gemv.
 */
size_t w4a16_gemv_noalloc_scratch_limit(void);
w4_status w4a16_gemv_noalloc(const void *x_bf16, int64_t M, const void *packed, int64_t N,
                             int64_t K, int group, int mode, void *y, int flags,
                             cudaStream_t stream);

/*
 * w4a16_gemm_tc -- the W4A16 product of w4a16_gemv for a few activation rows, on the tensor
 *   cores (TAHOMA "Four-bit inference", the W4A16 path: 4-bit weights expanded inside the
 *   kernel against bf16 activations with fp32 accumulation; "4-bit by default": decode at small
 *   batch is bound by the weight bytes, so the per-weight work must not grow with the batch):
 *     y[m, n] = sum_j s[n,j] * sum_{k in group j} (q[n,k] - z[n,j]) * x[m,k]
 *   computed as sum_j s[n,j] (P_j - (z[n,j] - 8) X_j), P_j = sum_{k in j} (q - 8) x and
 *   X_j = sum_{k in j} x, both on the tensor cores: the weights are expanded to the exact bf16
 *   integers q - 8 (one expansion per weight serves all M rows), each product with a bf16
 *   activation is exact in fp32, P_j and X_j are fp32 sums of the tensor cores, and the
 *   group scale and zero point are applied to them in fp32. The output is rounded once (to
 *   bf16, or kept fp32). Agreement with the exact product: about 1e-6 relative in fp32.
 *   The (128-row tile, k-block) units of the problem are divided evenly over one CTA per SM;
 *   CTAs sharing a tile leave partial sums in the workspace and the last of them adds them in
 *   a fixed order, so results are bit-identical run to run on a given GPU.
 *   x_bf16          device, bf16 [M, K]; 1 <= M <= 16
 *   packed          device, w4_prepack(..., W4_LAYOUT_TC) of W[N, K]
 *   y               device, bf16 [M, N], or fp32 [M, N] with W4_OUT_FP32 in flags
 *   flags           W4_OUT_FP32 | W4_OVERLAP_PREVIOUS (as w4a16_gemv); other bits: W4_ERR_ARG
 *   workspace       device scratch of at least w4a16_gemm_tc_workspace_bytes(N, K, group) bytes
 *                   (partial sums for one CTA per SM of the current device, and arrival
 *                   counters); required. Zero-fill it before its first use; every call that
 *                   completes leaves its counters zero again. Calls that may run concurrently
 *                   need separate workspaces. After a call whose kernel recorded an error in
 *                   the device status, zero-fill it again.
 *   Errors: NULL / SHAPE (M outside 1..16, N < 1 or N > 2^31, K < 32, K > 2^24, K % 32) /
 *   GROUP / ALIGN / ARG / WORKSPACE / CUDA.
 *
 * w4a16_gemm_tc_schedule -- host-only query (no GPU call) of how w4a16_gemm_tc divides the
 *   problem over `sms` SMs: out[6] receives tiles of 128 rows, k-blocks per tile, units
 *   (tiles x k-blocks), CTAs, k per k-block (max(128, group)) and bytes per unit record.
 *   Errors: NULL / SHAPE / GROUP.
 */
size_t w4a16_gemm_tc_workspace_bytes(int64_t N, int64_t K, int group);
w4_status w4a16_gemm_tc_schedule(int64_t M, int64_t N, int64_t K, int group, int sms, int64_t *out);
w4_status w4a16_gemm_tc(const void *x_bf16, int64_t M, const void *packed, int64_t N, int64_t K,
                        int group, int mode, void *y, int flags, void *workspace,
                        size_t workspace_bytes, cudaStream_t stream);

/*
 * w4a8_gemm -- W4A8 GEMM on the FP8 tensor cores (TAHOMA "Achievement 2", the list under
 *   "the A8 in W4A8": packed 4-bit weights are read from HBM and expanded to E4M3 in the
 *   kernel, the activation and expanded weight enter an FP8 tensor-core MMA, accumulation
 *   is FP32, the per-token activation scale is applied in the epilogue, the result is BF16):
 *     Y[m, n] = s_a[m] * sum_j s[n,j] * sum_{k in group j} a8[m,k] * (q[n,k] - z[n,j])
 *   with a8 the E4M3 value of X_e4m3[m,k], computed as
 *     s_a[m] * ( sum_j s[n,j] * sum_{k in j} a8[m,k] q[n,k]  -  sum_j s[n,j] z[n,j] G[m,j] ).
 *   The expanded weights q are exact small integers in E4M3 and the FP8 MMA sums exact
 *   products; the group scale multiplies fp32 per-group partial sums; the zero-point term
 *   is a bf16 hi/lo product on the tensor cores (relative error about 2^-16 of that term).
 *   X_e4m3      device, uint8 [M, K] from fp8_row_quant (groups 64 and 128; may be NULL for
 *               groups 32 and 256)
 *   X_f16       device, fp16 [M, K] from fp8_row_quant's X_f16 output (groups 32 and 256;
 *               may be NULL for groups 64 and 128)
 *   row_scale   device, fp32 [M] from fp8_row_quant
 *   gsum_op     device, bf16 [M, w4a8_gsum_op_cols(K, group)] from fp8_row_quant with the
 *               same group (groups 64 and 128; may be NULL for groups 32 and 256)
 *   packed      device, w4_prepack(..., W4_LAYOUT_GEMM) of W[N, K]
 *   Y           device, bf16 [M, N] (out_fp32 == 0) or fp32 [M, N] (out_fp32 == 1)
 *   workspace   NULL, or device scratch of at least w4a8_gemm_workspace_bytes(M, N, K, group)
 *               bytes, zero-filled before its first use (every call that completes leaves
 *               its counters zero again; calls that may overlap on the GPU need separate
 *               workspaces; after a call whose kernel recorded an error in the device
 *               status, zero-fill it again). The output is cut into tiles of 128 weight rows x 256 tokens,
 *               one persistent block per SM. Without a workspace every tile is one block's
 *               work. With it, when the last wave of tiles would leave many SMs idle, those
 *               tiles are split along K over the SMs; each part's fp32 partial sum goes
 *               through the workspace and the last part to finish adds them in a fixed order
 *               (bit-identical results run to run; a different fp32 summation order than the
 *               unsplit schedule, within the same error bounds). A query result of 0 means
 *               the shape is never split and the workspace is not used.
 *   M >= 1; N >= 1; K >= 128, K % 32 == 0.
 *   Groups of 32 and 256: at 32 every FP8 MMA of K = 32 would end a group, and the
 *   per-group promotion (a TMEM readback and one fp32 FMA per output per group on the CUDA
 *   cores) would cost several times the MMA; at 256 the group spans two k-blocks of the
 *   promoted schedule. For these groups the kernel instead dequantizes each weight exactly
 *   into two fp16 parts, w = (q - z) s = hi + lo (exact for |z| < 1024 and |w| < 65504),
 *   and accumulates hi x a + lo x a on the fp16 tensor cores over the whole K in TMEM, a
 *   being the E4M3 activation values, which it reads as fp16 (X_f16, exact): the same
 *   dequantized operands, no zero-point operand, no split of the last wave (the workspace
 *   query returns 0).
 *   Errors: NULL / SHAPE / GROUP / ALIGN / ARG / WORKSPACE (non-NULL and smaller than the
 *   query's result).
 */
size_t w4a8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int group);
w4_status w4a8_gemm(const uint8_t *X_e4m3, const uint16_t *X_f16, const float *row_scale,
                    const uint16_t *gsum_op, int64_t M, const void *packed, int64_t N, int64_t K, int group, int mode,
                    void *Y, int out_fp32, void *workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/*
 * w4a8_gemm_rowquant -- fp8_row_quant and w4a8_gemm in ONE launch, from bf16 activations.
 *   "Four-bit inference ... Tahoma", Achievement 2: the per-token activation scale is
 *   recomputed on every forward pass, so its cost is paid on every call; here the GEMM's
 *   persistent blocks quantize the rows themselves instead of a separate launch.
 *   Computes exactly what fp8_row_quant(X, M, K, group, ...) followed by
 *   w4a8_gemm(..., workspace) computes -- the same E4M3 codes, row scales and group-sum
 *   operand bit for bit, then the same Y bit for bit:
 *     Y[m, n] = s_a[m] * sum_j s[n,j] * sum_{k in group j} e4m3(X[m,k] / s_a[m]) * (q[n,k] - z[n,j]),
 *     s_a[m] = max(max_k |X[m,k]|, 1e-8) / 448.
 *   How: one warp quantizes one row (max over the row, scale, codes, exact integer group sums)
 *   into the workspace and then counts it in its 256-row token tile's counter with a release
 *   add. Before the roles of the GEMM start, every warp of the grid quantizes the rows of the
 *   token tiles that the first tiles read; afterwards two otherwise idle warps of every block
 *   quantize the remaining rows in order. The TMA producer waits (acquire) for a token tile's
 *   full count before it loads that tile, and the epilogue warps before they read its row
 *   scales. No block waits on another block's tile work, so the rows always come out; every
 *   wait is bounded (W4_ERR_TIMEOUT in the device status).
 *   X_bf16      device, bf16 [M, K], row-major (read only)
 *   packed      device, w4_prepack(..., W4_LAYOUT_GEMM) of W[N, K] with this group
 *   Y           device, bf16 [M, N] (out_fp32 == 0) or fp32 [M, N] (out_fp32 == 1)
 *   workspace   device scratch of at least w4a8_gemm_rowquant_workspace_bytes(M, N, K, group)
 *               bytes, 256-byte aligned, owned by the caller; no initial contents are needed
 *               (each call clears its counters with one memset on `stream` before the
 *               kernel). After the call it holds the E4M3 rows, row scales and group-sum
 *               operand at the offsets w4a8_gemm_rowquant_layout reports. Calls that may
 *               overlap on the GPU need separate workspaces.
 *   group       64 or 128 (the promoted path); 32 and 256 return W4_ERR_UNSUPPORTED.
 *   M >= 1; N >= 1; K >= 128, K % 32 == 0.
 *   Errors: NULL / SHAPE / GROUP / ALIGN / ARG / UNSUPPORTED / WORKSPACE (smaller than the
 *   query's result) / CUDA.
 * w4a8_gemm_rowquant_layout -- host-only: out[0..3] = byte offsets inside the workspace of
 *   the E4M3 rows [M, K], the row scales fp32 [M], the group-sum operand bf16
 *   [M, w4a8_gsum_op_cols(K, group)], and the workspace size. Errors: NULL / SHAPE / GROUP /
 *   UNSUPPORTED.
 */
size_t w4a8_gemm_rowquant_workspace_bytes(int64_t M, int64_t N, int64_t K, int group);
w4_status w4a8_gemm_rowquant_layout(int64_t M, int64_t N, int64_t K, int group, int64_t *out);
w4_status w4a8_gemm_rowquant(const void *X_bf16, int64_t M, const void *packed, int64_t N, int64_t K,
                             int group, int mode, void *Y, int out_fp32, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/*
 * w4a8_gemm_schedule -- host-only query (no GPU call): how w4a8_gemm with a workspace divides
 *   the problem (M, N, K, group) over `sms` SMs (1 .. 4096). out[7] receives: tiles (128
 *   weight rows x 256 tokens each), whole tiles (the first ones, round-robin over the
 *   grid), split tiles (the rest), blocks sharing the split tiles, grid size, workspace
 *   bytes, k-blocks of 128 per tile. Errors: NULL / SHAPE / GROUP.
 *
 * w4a8_gemm_split_segment -- host-only query: segment s (0 or 1) of block c (0 <= c < PS) when
 *   R split tiles of KT k-blocks are shared by PS blocks, R <= PS <= R * KT (every block gets
 *   at least one k-block), computed by the same functions the kernel uses. out[7] receives: found (0/1), split tile index, first and one-past-last
 *   k-block, first and last block contributing to that tile, partial-result slot of
 *   (c, tile). Errors: NULL / ARG.
 */
w4_status w4a8_gemm_schedule(int64_t M, int64_t N, int64_t K, int group, int sms, int64_t *out);
w4_status w4a8_gemm_split_segment(int64_t R, int64_t KT, int64_t PS, int64_t c, int s,
                                  int64_t *out);

/*
 * w4a8_grouped_gemm -- w4a8_gemm for E experts at once (mixture-of-experts layers whose
 *   expert weights are 4-bit; the blog post "4-bit by default", gpt-oss paragraph). Rows
 *   [off[e], off[e+1]) of X_e4m3 / X_f16 / row_scale / gsum_op / Y belong to expert e and are
 *   multiplied by expert e's weight.
 *   expert_row_offsets  device, int32 [E+1], non-decreasing, off[0] == 0, off[E] == M_total
 *   packed              device, E slabs of w4_prepack_bytes(N, K, group, W4_LAYOUT_GEMM)
 *                       bytes each, slab e at packed + e * that size
 *   Y                   device, bf16 [M_total, N]
 *   1 <= E <= 1024. Errors: NULL / SHAPE / GROUP / ALIGN / ARG.
 */
w4_status w4a8_grouped_gemm(const uint8_t *X_e4m3, const uint16_t *X_f16, const float *row_scale,
                            const uint16_t *gsum_op, const int32_t *expert_row_offsets, int E,
                            int64_t M_total, const void *packed, int64_t N, int64_t K, int group,
                            int mode, void *Y, cudaStream_t stream);

/*
 * Mixture-of-experts layer around w4a8_grouped_gemm ("4-bit by default", opening section:
 * MoE expert weights as the 4-bit target, gpt-oss). The pages leave the router, the
 * activation between the two expert projections and the combine open; this library takes
 * top-k routing with softmax gates over the selected logits, SwiGLU on [gate | up] halves,
 * and the gate-weighted sum. A layer is: w4_moe_route; fp8_row_quant_gather of the tokens
 * in expert order; w4a8_grouped_gemm (gate_up); w4_moe_swiglu_quant; w4a8_grouped_gemm
 * (down); w4_moe_combine.
 *
 * w4_moe_route -- logits fp32 [T, E] (device). For each token the k largest logits in
 *   descending order (equal logits in ascending expert order; a NaN logit is taken only where
 *   a scan in expert order that replaces its choice by a strictly larger logit would take it)
 *   -> experts int32 [T, k]; gates fp32 [T, k] = softmax over those k logits (fp32, expf);
 *   expert_row_offsets int32 [E+1], rows of expert e being [off[e], off[e+1]) of the grouped
 *   layout; token_of_row int32 [T*k], the token of every grouped row (tokens ascending inside
 *   an expert); row_of int32 [T, k], the grouped row of token t's i-th expert. Deterministic
 *   (no dependence on thread timing). workspace: device scratch of at least
 *   w4_moe_route_workspace_bytes(T, E) bytes (ceil(T/32) * E int32 expert counts), owned by
 *   the caller, contents irrelevant between calls. Two launches on `stream`; the second reads
 *   every earlier block's counts, so its work grows as (T/32)^2 * E (0.5 M reads at T = 4096,
 *   E = 32).
 *   1 <= E <= 1024, 1 <= k <= min(8, E), T * k < 2^31. Errors: NULL / SHAPE / WORKSPACE /
 *   ALIGN (4-byte) / CUDA.
 */
int64_t w4_moe_route_workspace_bytes(int64_t T, int E);
w4_status w4_moe_route(const float *logits, int64_t T, int E, int k, int32_t *experts,
                       float *gates, int32_t *expert_row_offsets, int32_t *token_of_row,
                       int32_t *row_of, void *workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/*
 * w4_moe_swiglu_quant -- SwiGLU between the expert projections, then the per-row E4M3
 *   quantization of its result for the down projection (TAHOMA "Achievement 2" row scale):
 *   gate_up_bf16 [R, 2H] holds [gate | up] per row; h = gate * up / (1 + exp(-gate)) in fp32;
 *   row_scale[r] = max(max|h|, 1e-8) / 448; X_e4m3 [R, H] = e4m3(h / row_scale) with IEEE
 *   division, RNE, saturation. gsum_op (optional, bf16 [R, w4a8_gsum_op_cols(H, group)]) as
 *   fp8_row_quant writes it, for down projections with group 64 or 128; X_f16 (optional,
 *   fp16 [R, H]) the same E4M3 values as binary16, for groups 32 and 256 (X_e4m3 may then
 *   be NULL). 16 <= H <= 16384, H % 16 == 0. Errors: NULL / SHAPE / GROUP / ALIGN.
 */
w4_status w4_moe_swiglu_quant(const void *gate_up_bf16, int64_t R, int64_t H, int group,
                              uint8_t *X_e4m3, float *row_scale, uint16_t *gsum_op,
                              uint16_t *X_f16, cudaStream_t stream);

/*
 * w4_moe_combine -- y[t, :] = sum_{i < k} gates[t, i] * rows[row_of[t, i], :], fp32 products
 *   and sums in i order, rounded once to bf16. rows_bf16 [R, N] (the down projection's
 *   output in grouped order), row_of int32 [T, k], gates fp32 [T, k], y_bf16 [T, N].
 *   A row index outside [0, R) is recorded as W4_ERR_DEVICE_CHECK and skipped.
 *   N % 8 == 0, 1 <= k <= 8. Errors: NULL / SHAPE / ALIGN.
 */
w4_status w4_moe_combine(const void *rows_bf16, int64_t N, int64_t R, const int32_t *row_of,
                         const float *gates, int64_t T, int k, void *y_bf16, cudaStream_t stream);

/*
 * NF4 comparator (QLWG, NF4 paragraph: 16 levels that are quantiles of a normal distribution,
 * blocks of 64; TAHOMA: the NF4 operating point its W4A8 path is measured against). The
 * levels follow the QLoRA construction (the pages leave it open): with delta = (1/32 + 1/30)/2,
 * the normal quantiles at eight equal probability steps from 1 - delta down to 1/2 (exclusive),
 * the negatives of seven such steps, and an exact zero, divided by the largest, in fp32,
 * ascending. Each block of 64 consecutive weights of a row keeps its max|w| as an fp32 scale
 * (single-level scales: the pages' double quantization of the scales is not built).
 *
 * w4_nf4_levels -- the 16 levels (host array).
 * w4_nf4_quantize -- W_bf16 [N, K] -> codes uint8 [N, K/2] (packed like the INT4 codes: byte
 *   j = q[2j] | q[2j+1] << 4) and absmax fp32 [N, K/64]. The code of w is the level nearest to
 *   w / a (IEEE fp32 division and fp32 distances; ties to the lower level); an all-zero block
 *   gets a = 0 and the zero level. K % 64 == 0. Errors: NULL / SHAPE / ALIGN.
 * w4_nf4_gemv -- y[m, n] = sum_k x[m, k] * level[q[n, k]] * a[n, k / 64] with fp32
 *   accumulation, output bf16 (or fp32 with W4_OUT_FP32); W4_OVERLAP_PREVIOUS as for
 *   w4a16_gemv. Reads the quantizer's codes and absmax directly (no prepack). 1 <= M <= 4,
 *   M * K * 4 bytes of activations staged in shared memory (K <= 57,000 at M = 1).
 *   Errors: NULL / SHAPE / ALIGN / ARG.
 */
w4_status w4_nf4_levels(float *levels_host);
w4_status w4_nf4_quantize(const void *W_bf16, int64_t N, int64_t K, uint8_t *codes, float *absmax,
                          cudaStream_t stream);
w4_status w4_nf4_gemv(const void *x_bf16, int64_t M, const uint8_t *codes, const float *absmax,
                      int64_t N, int64_t K, void *y, int flags, cudaStream_t stream);

/*
 * w4_device_status -- synchronizes `stream`, then reads and clears the device status word
 *   of the current device. *code_out receives W4_OK or the first W4_ERR_TIMEOUT /
 *   W4_ERR_DEVICE_CHECK recorded since the last call. Returns W4_ERR_CUDA if the
 *   synchronization itself fails.
 */
w4_status w4_device_status(cudaStream_t stream, int *code_out);

/*
 * w4_selftest_bounded_wait -- diagnostic (no counterpart in the source pages): launches one
 *   block whose thread waits, with the same bounded mbarrier wait the W4A8 GEMM and the
 *   W4A16 GEMV use, for a barrier phase that nothing completes. After limit_ns nanoseconds
 *   (1e3 .. 1e9) the wait gives up and records W4_ERR_TIMEOUT in the device status word, and
 *   the kernel returns normally; the context stays usable. It lets a test check the failure
 *   path of every bounded wait without faulting or hanging a GPU.
 *   Errors: ARG (limit out of range) / CUDA (launch).
 */
w4_status w4_selftest_bounded_wait(int64_t limit_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* W4_H_ */
