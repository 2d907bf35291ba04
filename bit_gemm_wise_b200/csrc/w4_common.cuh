// Shared device/host helpers of libw4 (sm_100a). Internal header: not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "w4.h"

#define W4_API extern "C" __attribute__((visibility("default")))

namespace w4 {

constexpr unsigned FULL = 0xffffffffu;

// ------------------------------------------------------------------ host-side checks

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool valid_group(int g) { return g == 32 || g == 64 || g == 128 || g == 256; }
inline bool valid_mode(int m) { return m == W4_SYM || m == W4_ASYM; }

// Address of this device's status word (kernels record timeouts / failed checks there).
int *device_status_ptr();

inline w4_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

inline int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// ------------------------------------------------------------------ device helpers

__device__ __forceinline__ void record_status(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// mbarrier helpers (CTA scope)
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// try_wait with a suspend-time hint: a thread whose phase is not complete sleeps until the
// phase completes or about 0.5 ms have passed, instead of spinning and taking issue slots
// from the working warps of its SM sub-partition.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(500000u)
        : "memory");
    return ok != 0;
}

// try_wait without a hint (the hardware's own short time limit), for a single latency-critical
// thread that should resume as soon as the phase completes.
__device__ __forceinline__ bool mbar_try_wait_short(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for an mbarrier phase, bounded by wall-clock time. If `abort` (shared, may be null)
// becomes non-zero the wait gives up at once; if the time runs out it sets *abort, records
// W4_ERR_TIMEOUT in the device status word and returns false.
template <bool SHORT = false>
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t *bar, uint32_t parity, int *abort, int *status,
                                                    uint64_t limit_ns) {
    if (SHORT ? mbar_try_wait_short(bar, parity) : mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (SHORT ? mbar_try_wait_short(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if (abort && *(volatile int *)abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            if (abort) *(volatile int *)abort = 1;
            record_status(status, W4_ERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait without an abort flag (default limit 2 s).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, int *status,
                                                  uint64_t limit_ns = 2000000000ull) {
    return mbar_wait_abortable(bar, parity, nullptr, status, limit_ns);
}

// 1-D bulk copy global -> shared, completing on an mbarrier (size % 16 == 0, both
// addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// The same copy with an L2 evict-first policy: for data read exactly once (a GEMV's weight
// stream), so that it does not push activations and outputs out of L2.
__device__ __forceinline__ void bulk_g2s_stream(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

// Hint to bring `bytes` (a multiple of 16) at src (16-byte aligned) into L2; nothing waits for
// it and nothing lands in shared memory.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Named barrier over `n` threads (a multiple of 32); id 0 is __syncthreads.
__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Streaming 128-bit global load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

}  // namespace w4
