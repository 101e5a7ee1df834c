// bi_abi.cu -- status strings, ABI version and the device error word of libbi.so.
#include <atomic>

#include "bi_common.cuh"

namespace {

// One word per device.  Kernels whose bounded waits run out OR a cause bit into it.
__device__ uint32_t g_device_error;

constexpr int kMaxDevices = 64;
std::atomic<uintptr_t> g_word_addr[kMaxDevices];

}  // namespace

namespace bi {

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
