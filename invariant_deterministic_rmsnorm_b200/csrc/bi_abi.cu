// bi_abi.cu -- status strings, ABI version and the device error word of libbi.so.
#include <atomic>

#include "bi_common.cuh"
#include "bi_ctrl.h"
#include "bi_sm100.cuh"

namespace {

// One CTA waits, with the kernels' bounded wait, on an mbarrier that nothing arrives on.  The
// wait must give up after limit_ns; the kernel then reports it the way every kernel reports a
// wait that ran out, and returns.
__global__ void wait_probe_kernel(uint64_t limit_ns, uint32_t* err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        bi::sm100::mbar_init(bi::sm100::smem_u32(&bar), 1);
        bi::sm100::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !bi::sm100::mbar_wait_ns(bi::sm100::smem_u32(&bar), 0u, nullptr, limit_ns))
        atomicOr(err, bi::DEVERR_WAIT_FULL);
}

// One word per device.  Kernels whose bounded waits run out OR a cause bit into it.
__device__ uint32_t g_device_error;

constexpr int kMaxDevices = 64;
std::atomic<uintptr_t> g_word_addr[kMaxDevices];
std::atomic<int> g_pdl{1};

}  // namespace

namespace bi {

bool pdl_enabled() { return g_pdl.load(std::memory_order_relaxed) != 0; }

// Device address of the error word on the current device.  The address is looked
// up once per device and cached.  Returns nullptr on a CUDA error.
uint32_t* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    uintptr_t a = g_word_addr[dev].load(std::memory_order_acquire);
    if (a == 0) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        a = reinterpret_cast<uintptr_t>(p);
        g_word_addr[dev].store(a, std::memory_order_release);
    }
    return reinterpret_cast<uint32_t*>(a);
}

}  // namespace bi

BI_API const char* bi_status_str(int status) {
    switch (status) {
        case BI_OK: return "BI_OK";
        case BI_ERR_INVALID_ARG: return "BI_ERR_INVALID_ARG";
        case BI_ERR_UNSUPPORTED_SHAPE: return "BI_ERR_UNSUPPORTED_SHAPE";
        case BI_ERR_MISALIGNED: return "BI_ERR_MISALIGNED";
        case BI_ERR_WORKSPACE: return "BI_ERR_WORKSPACE";
        case BI_ERR_CUDA: return "BI_ERR_CUDA";
        case BI_ERR_TIMEOUT: return "BI_ERR_TIMEOUT";
        default: return "BI_ERR_UNKNOWN";
    }
}

BI_API int bi_abi_version(void) { return 1; }

BI_API int bi_get_device_error(uint32_t* code, void* stream) {
    if (!code) return BI_ERR_INVALID_ARG;
    uint32_t* word = bi::device_error_word();
    if (!word) return BI_ERR_CUDA;
    cudaStream_t s = bi::as_stream(stream);
    uint32_t host = 0;
    if (cudaMemcpyAsync(&host, word, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess) return BI_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BI_ERR_CUDA;
    *code = host;
    return host ? BI_ERR_TIMEOUT : BI_OK;
}

BI_API int bi_clear_device_error(void* stream) {
    uint32_t* word = bi::device_error_word();
    if (!word) return BI_ERR_CUDA;
    return cudaMemsetAsync(word, 0, sizeof(uint32_t), bi::as_stream(stream)) == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

BI_API int bi_ctrl_wait_timeout_probe(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000ull || limit_ns > 2000000000ull) return BI_ERR_INVALID_ARG;
    uint32_t* err = bi::device_error_word();
    if (!err) return BI_ERR_CUDA;
    wait_probe_kernel<<<1, 32, 0, bi::as_stream(stream)>>>(limit_ns, err);
    return bi::launch_status();
}

BI_API int bi_ctrl_set_pdl(int enable) {
    const int old = g_pdl.exchange(enable ? 1 : 0);
    return old;
}
