// bi_common.cuh -- shared host/device helpers for the libbi.so kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "bi.h"

#define BI_API extern "C" __attribute__((visibility("default")))

namespace bi {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

// Device address of the library's error word on the current device (bi_abi.cu).
uint32_t* device_error_word();

// Whether launches may use programmatic dependent launch (bi_abi.cu; on unless
// bi_ctrl_set_pdl(0) turned it off).
bool pdl_enabled();

// Launch `kernel` on `s`.  With programmatic dependent launch on, it may begin while the kernel
// before it on the stream finishes; every kernel launched this way calls pdl_wait() (bi_sm100.cuh)
// before it reads or writes global memory.  cluster_y: CTAs per cluster along y; 0 = launched
// without a cluster shape.  A kernel that uses cluster-scope instructions (mapa, st.async,
// barrier.cluster) is always given one, even a cluster of a single CTA.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              unsigned cluster_y, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_y >= 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = 1;
        attr[n].val.clusterDim.y = cluster_y;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = n ? attr : nullptr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline int elem_size(int dtype) { return dtype == BI_F32 ? 4 : (dtype == BI_BF16 ? 2 : 0); }

// Device error word bits (OR-ed by kernels whose bounded waits ran out).
enum : uint32_t {
    DEVERR_WAIT_TMA = 1u << 0,      // producer waited too long for a free stage
    DEVERR_WAIT_FULL = 1u << 1,     // MMA issuer waited too long for a loaded stage
    DEVERR_WAIT_ACCUM = 1u << 2,    // epilogue waited too long for the accumulator
    DEVERR_WAIT_CLUSTER = 1u << 3,  // cluster barrier / DSMEM handshake ran out
    DEVERR_BAD_LAYOUT = 1u << 8,    // decode attention: kv_indptr / kv_len violate the documented layout
    DEVERR_BAD_TOKEN = 1u << 9,     // embedding: token id outside [0, vocab)
    DEVERR_BAD_DST_ROW = 1u << 10,  // KV append: destination row outside the cache
    DEVERR_BAD_PREFILL = 1u << 11,  // prefill attention: indptr / positions outside the buffers
    DEVERR_BAD_POSITION = 1u << 12, // RoPE: position outside the cos/sin table
};

// ------------------------------------------------------------------ device helpers
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 ld_cached_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// bf16 pair <-> two floats.  The unpack is exact: a bf16 is the top half of a binary32.
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Two floats -> packed bf16x2, each rounded to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace bi
