// Status strings, version and the per-device status word of libw4.
#include "w4_common.cuh"

#include <mutex>

namespace w4 {

// One status word per device. Kernels that run a bounded wait or a self-check get its
// address as an argument and record the first failure with atomicCAS.
static __device__ int g_status_word;

static constexpr int kMaxDevices = 64;
static int *g_status_ptr[kMaxDevices];
static std::mutex g_status_mu;

int *device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_status_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    return g_status_ptr[dev];
}

}  // namespace w4

W4_API const char *w4_status_str(int status) {
    switch (status) {
        case W4_OK: return "ok";
        case W4_ERR_NULL: return "null pointer";
        case W4_ERR_SHAPE: return "unsupported shape";
        case W4_ERR_GROUP: return "bad group size";
        case W4_ERR_ALIGN: return "pointer not 16-byte aligned";
        case W4_ERR_ARG: return "bad argument";
        case W4_ERR_UNSUPPORTED: return "unsupported";
        case W4_ERR_CUDA: return "CUDA error";
        case W4_ERR_TIMEOUT: return "device wait timed out";
        case W4_ERR_DEVICE_CHECK: return "device check failed";
        case W4_ERR_WORKSPACE: return "workspace missing or too small";
        case W4_ERR_SCRATCH_LIMIT: return "request exceeds the fixed scratch of the allocation-free entry point";
        default: return "unknown status";
    }
}

W4_API int w4_version(void) { return 100; }

W4_API w4_status w4_device_status(cudaStream_t stream, int *code_out) {
    if (!code_out) return W4_ERR_NULL;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return W4_ERR_CUDA;
    int *p = w4::device_status_ptr();
    if (!p) return W4_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return W4_ERR_CUDA;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return W4_ERR_CUDA;
    *code_out = v;
    return W4_OK;
}

// ------------------------------------------------------------------ bounded-wait self-test
namespace w4 {

// One thread initializes an mbarrier that expects one arrival and waits for its first phase
// without ever arriving: the bounded wait must expire, record W4_ERR_TIMEOUT and return.
__global__ void selftest_wait_kernel(uint64_t limit_ns, int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    (void)mbar_wait_bounded(&bar, 0, status, limit_ns);
}

}  // namespace w4

W4_API w4_status w4_selftest_bounded_wait(int64_t limit_ns, cudaStream_t stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000LL) return W4_ERR_ARG;
    int *status = w4::device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    w4::selftest_wait_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_ns, status);
    return w4::launch_status();
}
