// bi_rmsnorm.cu -- batch-invariant RMSNorm: one CTA per row, reduction tree fixed by H.
//
// Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section
// "Diseño de kernels invariantes al batch", RMSNorm.  That section asks for a
// data-parallel strategy in which one core handles each batch element.  The
// strategy must not change with batch size.  The small-batch split-reduction
// variant the section mentions gives up invariance and is not used here.
//
// Launch plan, a function of (H, dtypes) only:
//   vec     = 16 bytes / element size (8 bf16 or 4 fp32 elements per 128-bit load)
//   nvec    = H / vec
//   threads = nvec / 2 rounded up to a warp, clamped to [32, 256]
//   vpt     = ceil(nvec / threads) vectors per thread (compile-time 1, 2, 4, 8 or 16)
// Thread t owns vectors t, t + threads, t + 2*threads, ...  It keeps them in
// registers (one HBM read of x), sums their squares sequentially with fused
// multiply-adds, then joins a butterfly shuffle tree within its warp and a second
// fixed tree over the warps.  Because the plan depends on H alone, every row is
// reduced in exactly the same order at every M and every row position.
#include "bi_common.cuh"
#include "bi_sm100.cuh"

using bi::sm100::pdl_trigger;
using bi::sm100::pdl_wait;

namespace {

constexpr int kMaxThreads = 256;

template <typename TIO>
struct IoTraits;
template <>
struct IoTraits<float> {
    static constexpr int kVec = 4;
    static __device__ __forceinline__ void unpack(const uint4& u, float (&f)[4]) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    static __device__ __forceinline__ uint4 pack(const float (&f)[4]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};
template <>
struct IoTraits<__nv_bfloat16> {
    static constexpr int kVec = 8;
    static __device__ __forceinline__ void unpack(const uint4& u, float (&f)[8]) {
        f[0] = bi::bf16_lo(u.x); f[1] = bi::bf16_hi(u.x); f[2] = bi::bf16_lo(u.y); f[3] = bi::bf16_hi(u.y);
        f[4] = bi::bf16_lo(u.z); f[5] = bi::bf16_hi(u.z); f[6] = bi::bf16_lo(u.w); f[7] = bi::bf16_hi(u.w);
    }
    static __device__ __forceinline__ uint4 pack(const float (&f)[8]) {
        return make_uint4(bi::pack_bf16x2(f[0], f[1]), bi::pack_bf16x2(f[2], f[3]),
                          bi::pack_bf16x2(f[4], f[5]), bi::pack_bf16x2(f[6], f[7]));
    }
};

// Load kVec weights of type TW starting at element index e0 and widen to fp32.
template <typename TW, int V>
__device__ __forceinline__ void load_w(const TW* w, int64_t e0, float (&f)[V]) {
    if constexpr (sizeof(TW) == 4) {
#pragma unroll
        for (int i = 0; i < V; i += 4) {
            uint4 u = bi::ld_cached_v4(reinterpret_cast<const float*>(w) + e0 + i);
            f[i] = __uint_as_float(u.x); f[i + 1] = __uint_as_float(u.y);
            f[i + 2] = __uint_as_float(u.z); f[i + 3] = __uint_as_float(u.w);
        }
    } else if constexpr (V == 4) {  // fp32 rows with bf16 weights: 4 weights = 8 bytes
        uint2 u;
        asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(u.x), "=r"(u.y)
                     : "l"(reinterpret_cast<const __nv_bfloat16*>(w) + e0));
        f[0] = bi::bf16_lo(u.x); f[1] = bi::bf16_hi(u.x); f[2] = bi::bf16_lo(u.y); f[3] = bi::bf16_hi(u.y);
    } else {
#pragma unroll
        for (int i = 0; i < V; i += 8) {
            uint4 u = bi::ld_cached_v4(reinterpret_cast<const __nv_bfloat16*>(w) + e0 + i);
            f[i] = bi::bf16_lo(u.x); f[i + 1] = bi::bf16_hi(u.x); f[i + 2] = bi::bf16_lo(u.y);
            f[i + 3] = bi::bf16_hi(u.y); f[i + 4] = bi::bf16_lo(u.z); f[i + 5] = bi::bf16_hi(u.z);
            f[i + 6] = bi::bf16_lo(u.w); f[i + 7] = bi::bf16_hi(u.w);
        }
    }
}

// Row r's arithmetic: thread t owns vectors t, t + threads, ... of the row; sequential FMAs
// per thread, a warp butterfly, then a fixed tree over the warps.  The CTA walks rows
// r = blockIdx.x, blockIdx.x + gridDim.x, ... and keeps the next row's loads in flight
// while it reduces the current one.  Which CTA handles a row never changes its arithmetic.
template <typename TIO, typename TW, int VPT>
__global__ void __launch_bounds__(kMaxThreads)
rmsnorm_rows_kernel(const TIO* __restrict__ x, const TW* __restrict__ w, TIO* __restrict__ y, int64_t M, int nvec,
                    int64_t ldx, int64_t ldy, float h_float, float eps) {
    constexpr int V = IoTraits<TIO>::kVec;
    __shared__ float warp_sums[2][kMaxThreads / 32];
    __shared__ float row_total[2];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int nthreads = blockDim.x;
    const int nwarps = nthreads >> 5;

    uint4 xv[VPT], xn[VPT];
    int64_t row = blockIdx.x;
    // Every CTA waits for the kernel before it (x and w may come from it) before anything else,
    // so this grid never completes ahead of that one: a later kernel's wait then covers both.
    pdl_wait();
    pdl_trigger();  // the next kernel may start its set-up; it waits for this grid before it reads y
    if (row >= M) return;
    // the weights are the same for every row: when a thread's share is small, keep their raw
    // bits in registers for the CTA's lifetime (widened per use); otherwise re-read them per row
    constexpr bool kWInRegs = VPT * V <= 32;
    constexpr int WWORDS = V * (int)sizeof(TW) / 4;  // 32-bit words of weights per vector
    uint32_t wr[kWInRegs ? VPT : 1][WWORDS];
    if constexpr (kWInRegs) {
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = tid + i * nthreads;
            if (v < nvec) {
                const uint32_t* src = reinterpret_cast<const uint32_t*>(w + (int64_t)v * V);
#pragma unroll
                for (int k = 0; k < WWORDS; ++k) wr[i][k] = __ldg(src + k);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int v = tid + i * nthreads;
        xv[i] = (v < nvec) ? bi::ld_stream_v4(x + row * ldx + (int64_t)v * V) : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int buf = 0; row < M; row += gridDim.x, buf ^= 1) {
        // 1. prefetch the next row of this CTA
        const int64_t nrow = row + gridDim.x;
        if (nrow < M) {
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = tid + i * nthreads;
                xn[i] = (v < nvec) ? bi::ld_stream_v4(x + nrow * ldx + (int64_t)v * V) : make_uint4(0u, 0u, 0u, 0u);
            }
        }

        // 2. per-thread sum of squares, vectors in order, elements in order
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            float f[V];
            IoTraits<TIO>::unpack(xv[i], f);
#pragma unroll
            for (int e = 0; e < V; ++e) ss = __fmaf_rn(f[e], f[e], ss);
        }

        // 3. warp butterfly: partners add the same two values, so every lane ends with the same bits
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
        if (lane == 0) warp_sums[buf][warp] = ss;
        __syncthreads();

        // 4. fixed tree over the warps (missing warps contribute +0, which is exact)
        if (warp == 0) {
            float t = (lane < nwarps) ? warp_sums[buf][lane] : 0.0f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, off));
            if (lane == 0) row_total[buf] = t;
        }
        __syncthreads();
        // (the buffers alternate between rows, so the next row's writes cannot race these reads)

        const float inv = __frsqrt_rn(__fadd_rn(__fdiv_rn(row_total[buf], h_float), eps));

        // 5. y = (x * inv) * w, one rounding to the output type
        TIO* yr = y + row * ldy;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = tid + i * nthreads;
            if (v < nvec) {
                float f[V], wf[V];
                IoTraits<TIO>::unpack(xv[i], f);
                if constexpr (kWInRegs) {
                    if constexpr (sizeof(TW) == 4) {
#pragma unroll
                        for (int e = 0; e < V; ++e) wf[e] = __uint_as_float(wr[i][e]);
                    } else {
#pragma unroll
                        for (int k = 0; k < WWORDS; ++k) {
                            wf[2 * k] = bi::bf16_lo(wr[i][k]);
                            wf[2 * k + 1] = bi::bf16_hi(wr[i][k]);
                        }
                    }
                } else {
                    load_w<TW, V>(w, (int64_t)v * V, wf);
                }
#pragma unroll
                for (int e = 0; e < V; ++e) f[e] = __fmul_rn(__fmul_rn(f[e], inv), wf[e]);
                bi::st_stream_v4(yr + (int64_t)v * V, IoTraits<TIO>::pack(f));
            }
        }
#pragma unroll
        for (int i = 0; i < VPT; ++i) xv[i] = xn[i];
    }
}

// Grid: as many CTAs as fit on the GPU at once (at most one per row); each loops over rows.
template <typename TIO, typename TW, int VPT>
int launch_rows(const TIO* x, const TW* w, TIO* y, int64_t M, int nvec, int threads, int64_t ldx, int64_t ldy,
                float hf, float eps, cudaStream_t s) {
    static int resident[64][kMaxThreads / 32 + 1];  // CTAs per SM, per device and block size
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BI_ERR_CUDA;
    int& per_sm = resident[dev][threads / 32];
    if (per_sm == 0) {
        int n = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, rmsnorm_rows_kernel<TIO, TW, VPT>, threads, 0) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BI_ERR_CUDA;
        per_sm = (n > 0 ? n : 1) * sms;
    }
    const int64_t grid = M < per_sm ? M : per_sm;
    if (bi::launch_pdl(rmsnorm_rows_kernel<TIO, TW, VPT>, dim3((unsigned)grid), dim3(threads), 0, s, 0u, x, w, y, M,
                       nvec, ldx, ldy, hf, eps) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

template <typename TIO, typename TW>
int launch_typed(const void* x, const void* w, void* y, int64_t M, int64_t H, int64_t ldx, int64_t ldy, float eps,
                 cudaStream_t s) {
    constexpr int V = IoTraits<TIO>::kVec;
    const int nvec = (int)(H / V);
    int threads = ((nvec / 2 + 31) / 32) * 32;  // about two 16-byte vectors per thread
    if (threads < 32) threads = 32;
    if (threads > kMaxThreads) threads = kMaxThreads;
    const int vpt = (nvec + threads - 1) / threads;
    const TIO* xp = static_cast<const TIO*>(x);
    const TW* wp = static_cast<const TW*>(w);
    TIO* yp = static_cast<TIO*>(y);
    const float hf = (float)H;
    switch (vpt) {
        case 1: return launch_rows<TIO, TW, 1>(xp, wp, yp, M, nvec, threads, ldx, ldy, hf, eps, s);
        case 2: return launch_rows<TIO, TW, 2>(xp, wp, yp, M, nvec, threads, ldx, ldy, hf, eps, s);
        case 3: case 4: return launch_rows<TIO, TW, 4>(xp, wp, yp, M, nvec, threads, ldx, ldy, hf, eps, s);
        case 5: case 6: case 7: case 8: return launch_rows<TIO, TW, 8>(xp, wp, yp, M, nvec, threads, ldx, ldy, hf, eps, s);
        default: return launch_rows<TIO, TW, 16>(xp, wp, yp, M, nvec, threads, ldx, ldy, hf, eps, s);
    }
}

}  // namespace

BI_API int bi_rmsnorm(const void* x, const void* w, void* y, int64_t M, int64_t H, int64_t ldx, int64_t ldy,
                      float eps, int io_dtype, int w_dtype, void* stream) {
    const int es = bi::elem_size(io_dtype);
    const int ws = bi::elem_size(w_dtype);
    if (es == 0 || ws == 0) return BI_ERR_INVALID_ARG;
    if (M < 0 || H <= 0 || ldx < H || ldy < H || !(eps >= 0.0f)) return BI_ERR_INVALID_ARG;
    if (M == 0) return BI_OK;
    if (!x || !w || !y) return BI_ERR_INVALID_ARG;
    if (M > 0x7fffffffLL) return BI_ERR_UNSUPPORTED_SHAPE;
    const int vec = 16 / es;
    if (H % vec != 0 || H % (16 / ws) != 0) return BI_ERR_MISALIGNED;
    if ((ldx * es) % 16 != 0 || (ldy * es) % 16 != 0) return BI_ERR_MISALIGNED;
    if (!bi::aligned16(x) || !bi::aligned16(w) || !bi::aligned16(y)) return BI_ERR_MISALIGNED;
    if (H / vec > (int64_t)kMaxThreads * 16) return BI_ERR_UNSUPPORTED_SHAPE;
    if (y == x && ldy != ldx) return BI_ERR_INVALID_ARG;
    cudaStream_t s = bi::as_stream(stream);
    if (io_dtype == BI_F32 && w_dtype == BI_F32) return launch_typed<float, float>(x, w, y, M, H, ldx, ldy, eps, s);
    if (io_dtype == BI_F32 && w_dtype == BI_BF16)
        return launch_typed<float, __nv_bfloat16>(x, w, y, M, H, ldx, ldy, eps, s);
    if (io_dtype == BI_BF16 && w_dtype == BI_BF16)
        return launch_typed<__nv_bfloat16, __nv_bfloat16>(x, w, y, M, H, ldx, ldy, eps, s);
    return launch_typed<__nv_bfloat16, float>(x, w, y, M, H, ldx, ldy, eps, s);
}

// ------------------------------------------------------------------ comparator: split reduction
//
// The small-batch alternative the RMSNorm section mentions: when the batch is small, cut each
// row across S CTAs (a thread-block cluster), reduce the slices in parallel and exchange the
// partial sums over distributed shared memory.  S is chosen from M, so a row's reduction tree
// changes with the batch size: faster for small batches, and not batch-invariant.
namespace {

int split_for(int64_t M, int64_t nvec) {
    int S = M <= 148 ? 8 : (M <= 296 ? 4 : (M <= 592 ? 2 : 1));
    while (S > 1 && (nvec % S != 0 || nvec / S < 32)) S >>= 1;
    return S;
}

template <typename TIO, typename TW>
__global__ void __launch_bounds__(128)
rmsnorm_split_kernel(const TIO* __restrict__ x, const TW* __restrict__ w, TIO* __restrict__ y, int nvec_slice,
                     int64_t ldx, int64_t ldy, float h_float, float eps) {
    constexpr int V = IoTraits<TIO>::kVec;
    constexpr int MAXV = 8;
    __shared__ float warp_sums[4];
    __shared__ float slice_sum;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = bi::sm100::cluster_ctarank();
    const uint32_t S = gridDim.x;
    const int64_t row = blockIdx.y;
    const int64_t v0 = (int64_t)rank * nvec_slice;
    uint4 xv[MAXV];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int v = tid + i * 128;
        xv[i] = make_uint4(0u, 0u, 0u, 0u);
        if (v < nvec_slice) {
            xv[i] = bi::ld_stream_v4(x + row * ldx + (v0 + v) * V);
            float f[V];
            IoTraits<TIO>::unpack(xv[i], f);
#pragma unroll
            for (int e = 0; e < V; ++e) ss = __fmaf_rn(f[e], f[e], ss);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
    if (lane == 0) warp_sums[warp] = ss;
    __syncthreads();
    if (tid == 0) slice_sum = __fadd_rn(__fadd_rn(warp_sums[0], warp_sums[1]), __fadd_rn(warp_sums[2], warp_sums[3]));
    bi::sm100::cluster_sync();
    float total = 0.0f;
    const uint32_t local = bi::sm100::smem_u32(&slice_sum);
    for (uint32_t s = 0; s < S; ++s) {
        float p;
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(p) : "r"(bi::sm100::mapa(local, s)) : "memory");
        total = __fadd_rn(total, p);
    }
    const float inv = __frsqrt_rn(__fadd_rn(__fdiv_rn(total, h_float), eps));
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int v = tid + i * 128;
        if (v < nvec_slice) {
            float f[V], wf[V];
            IoTraits<TIO>::unpack(xv[i], f);
            load_w<TW, V>(w, (v0 + v) * V, wf);
#pragma unroll
            for (int e = 0; e < V; ++e) f[e] = __fmul_rn(__fmul_rn(f[e], inv), wf[e]);
            bi::st_stream_v4(y + row * ldy + (v0 + v) * V, IoTraits<TIO>::pack(f));
        }
    }
    bi::sm100::cluster_sync();  // peers keep their partial sums until every CTA has read them
}

template <typename TIO, typename TW>
int launch_split(const void* x, const void* w, void* y, int64_t M, int64_t H, int64_t ldx, int64_t ldy, float eps,
                 cudaStream_t s) {
    constexpr int V = IoTraits<TIO>::kVec;
    const int64_t nvec = H / V;
    const int S = split_for(M, nvec);
    const int64_t nvs = nvec / S;
    if (nvs > 128 * 8 || M > 65535) return BI_ERR_UNSUPPORTED_SHAPE;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, (unsigned)M, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, rmsnorm_split_kernel<TIO, TW>, static_cast<const TIO*>(x), static_cast<const TW*>(w),
                           static_cast<TIO*>(y), (int)nvs, ldx, ldy, (float)H, eps) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

}  // namespace

BI_API int bi_ctrl_rmsnorm_split(const void* x, const void* w, void* y, int64_t M, int64_t H, int64_t ldx,
                                 int64_t ldy, float eps, int io_dtype, int w_dtype, void* stream) {
    const int es = bi::elem_size(io_dtype);
    const int ws = bi::elem_size(w_dtype);
    if (es == 0 || ws == 0) return BI_ERR_INVALID_ARG;
    if (M < 0 || H <= 0 || ldx < H || ldy < H || !(eps >= 0.0f)) return BI_ERR_INVALID_ARG;
    if (M == 0) return BI_OK;
    if (!x || !w || !y) return BI_ERR_INVALID_ARG;
    if (H % (16 / es) != 0 || H % (16 / ws) != 0 || (ldx * es) % 16 != 0 || (ldy * es) % 16 != 0)
        return BI_ERR_MISALIGNED;
    if (!bi::aligned16(x) || !bi::aligned16(w) || !bi::aligned16(y)) return BI_ERR_MISALIGNED;
    cudaStream_t s = bi::as_stream(stream);
    if (io_dtype == BI_F32 && w_dtype == BI_F32) return launch_split<float, float>(x, w, y, M, H, ldx, ldy, eps, s);
    if (io_dtype == BI_F32) return launch_split<float, __nv_bfloat16>(x, w, y, M, H, ldx, ldy, eps, s);
    if (w_dtype == BI_BF16) return launch_split<__nv_bfloat16, __nv_bfloat16>(x, w, y, M, H, ldx, ldy, eps, s);
    return launch_split<__nv_bfloat16, float>(x, w, y, M, H, ldx, ldy, eps, s);
}
