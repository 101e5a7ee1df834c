// bi_lora.cu -- batch-invariant LoRA shrink (deterministic split-K) and expand.
//
// Source: "Reproducible LoRA Inference Through Deterministic Split-K Reduction" (abstract).
// Split-K kernels parallelise the low-rank LoRA products.  If they combine partial results
// with floating-point atomic additions, repeated runs differ.  The deterministic variant
// keeps Split-K = 8 and combines the partials in a fixed order, so the FP32 shrink output
// is identical under replay.
//
// Shrink, t[M, r] = x[M, K] . A[K, r]:
//   One thread-block cluster of `split` CTAs per 64-row tile.  CTA s of the cluster computes
//   the partial P_s over its contiguous K slice [s*K/split, (s+1)*K/split).  A producer warp
//   streams 64-wide K chunks of x and A into a 6-stage shared-memory ring with TMA.  Four
//   warps accumulate with mma.sync m16n8k16 (bf16 in, fp32 accumulate), K ascending.  The
//   partial lands in the CTA's shared memory.  After a cluster barrier, CTA 0 reads the
//   partials of CTAs 1..split-1 over distributed shared memory and adds them in slice order:
//   t = ((P_0 + P_1) + P_2) + ... + P_{split-1}, every add rounded to nearest.  There is no
//   workspace, no atomic and no extra HBM traffic.  The split count and slice size depend
//   only on (K, split), never on M.
//
// Expand, y[M, N] += scale * bf16(t)[M, r] . B[r, N]:
//   64 x 128 tiles of y per CTA.  t is rounded to bf16 (nearest even) into shared memory,
//   zero-padded to 16 when r = 8.  The product comes from mma.sync into fp32 and is staged
//   in shared memory.  Then y is read and written with coalesced 128-bit accesses:
//   y = round(fma(scale, delta, y)).
#include <mutex>

#include "bi_common.cuh"
#include "bi_sm100.cuh"
#include "bi_tma_host.cuh"

using namespace bi::sm100;

namespace {

// ------------------------------------------------------------------ shrink
constexpr int SH_TM = 128;          // rows per CTA (8 warps x 16)
constexpr int SH_KC = 64;           // K per pipeline stage
constexpr int SH_CWARPS = 8;        // compute warps
constexpr int SH_THREADS = (SH_CWARPS + 1) * 32;
constexpr int SH_MAX_STAGES = 6;
constexpr int SH_MAX_SPLIT = 8;     // the largest cluster the shrink launches (portable cluster size)

template <int R>
struct ShrinkLayout {
    static constexpr int X_STAGE = SH_TM * SH_KC * 2;  // 16 KB, 128B-swizzled rows of 64 K
    static constexpr int A_STAGE = SH_KC * R * 2;      // 64 K-rows of R
    static constexpr int STAGE = X_STAGE + A_STAGE;    // multiple of 1024
    // as many stages as leave room for two CTAs per SM (about 113 KB each)
    static constexpr int STAGES = (110 * 1024) / STAGE < SH_MAX_STAGES ? (110 * 1024) / STAGE : SH_MAX_STAGES;
    static constexpr int PART = SH_TM * R * 4;         // the partial reuses the stage memory
    static_assert(PART <= STAGES * STAGE, "partial must fit in the stage memory");
    static constexpr size_t BYTES = 1024 + (size_t)STAGES * STAGE + 2 * SH_MAX_STAGES * 8 + 16;
    // swizzle of the A stage: inner extent 2R bytes
    static constexpr uint32_t A_MASK = R == 64 ? 7u : (R == 32 ? 3u : (R == 16 ? 1u : 0u));
};

template <int R, bool ATOMIC>
__global__ void __launch_bounds__(SH_THREADS, 1)
lora_shrink_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                   float* __restrict__ t, int M, int KS, int split, uint32_t* err) {
    using L = ShrinkLayout<R>;
    extern __shared__ uint8_t smem_raw[];
    constexpr int SH_STAGES = L::STAGES;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* part = reinterpret_cast<float*>(base);  // written only after every stage has been consumed
    uint64_t* full = reinterpret_cast<uint64_t*>(base + SH_STAGES * L::STAGE);
    uint64_t* empty = full + SH_STAGES;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + SH_STAGES);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t slice = ATOMIC ? blockIdx.y : cluster_ctarank();
    const int m0 = blockIdx.x * SH_TM;
    const int kbase = (int)slice * KS;
    const int nchunks = KS / SH_KC;

    if (tid == 0) {
        for (int i = 0; i < SH_STAGES; ++i) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), SH_CWARPS);
        }
        *abort = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    __syncthreads();

    if (warp == SH_CWARPS) {
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmA);
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % SH_STAGES;
                const uint32_t round = (uint32_t)(c / SH_STAGES);
                if (!mbar_wait(smem_u32(&empty[st]), (round & 1u) ^ 1u, abort)) {
                    atomicOr(err, bi::DEVERR_WAIT_TMA);
                    *abort = 1;
                    break;
                }
                uint8_t* sx = base + st * L::STAGE;
                const uint32_t fb = smem_u32(&full[st]);
                mbar_arrive_expect_tx(fb, L::STAGE);
                tma_load_2d(smem_u32(sx), &tmX, kbase + c * SH_KC, m0, fb);
                tma_load_2d(smem_u32(sx + L::X_STAGE), &tmA, 0, kbase + c * SH_KC, fb);
                ++issued;
            }
            if (*abort) {
                for (int c = issued > SH_STAGES ? issued - SH_STAGES : 0; c < issued; ++c)
                    (void)mbar_wait(smem_u32(&full[c % SH_STAGES]), (uint32_t)(c / SH_STAGES) & 1u, nullptr);
            }
        }
    } else {
        float acc[R / 8][4];
#pragma unroll
        for (int nt = 0; nt < R / 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
        for (int c = 0; c < nchunks; ++c) {
            const int st = c % SH_STAGES;
            const uint32_t round = (uint32_t)(c / SH_STAGES);
            // ldmatrix / mma.sync are warp-collective: the whole warp leaves together on a timeout
            const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), round & 1u, abort));
            if (!ok) {
                if (lane == 0) atomicOr(err, bi::DEVERR_WAIT_FULL);
                *abort = 1;
                break;
            }
            const uint32_t xs = smem_u32(base + st * L::STAGE);
            const uint32_t as = xs + L::X_STAGE;
#pragma unroll
            for (int kk = 0; kk < SH_KC / 16; ++kk) {
                uint32_t a[4];
                const int row = warp * 16 + (lane & 15);
                const int kb = (kk * 16 + (lane >> 4) * 8) * 2;
                ldmatrix_x4(swz(xs + row * 128 + kb, 7u), a);
#pragma unroll
                for (int nt = 0; nt < R / 8; ++nt) {
                    uint32_t b[2];
                    const int krow = kk * 16 + (lane & 15);
                    ldmatrix_x2_trans(swz(as + krow * (2 * R) + nt * 16, L::A_MASK), b);
                    mma_m16n8k16_bf16(acc[nt], a, b);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty[st]));
        }
        // every warp is done reading the stages before any partial overwrites them
        asm volatile("bar.sync 1, %0;" :: "n"(SH_CWARPS * 32) : "memory");
        const int g = lane >> 2, q = lane & 3;
#pragma unroll
        for (int nt = 0; nt < R / 8; ++nt) {
            const int col = nt * 8 + q * 2;
            float* p0 = part + (warp * 16 + g) * R + col;
            float* p1 = part + (warp * 16 + g + 8) * R + col;
            p0[0] = acc[nt][0];
            p0[1] = acc[nt][1];
            p1[0] = acc[nt][2];
            p1[1] = acc[nt][3];
        }
    }

    __syncwarp();  // reconverge each warp before the block / cluster barriers below
    if constexpr (ATOMIC) {
        // Comparator only: partials are added to t in whatever order the CTAs arrive.
        __syncthreads();
        for (int i = tid; i < SH_TM * R; i += SH_THREADS) {
            const int row = i / R, col = i % R;
            if (m0 + row < M) atomicAdd(t + (size_t)(m0 + row) * R + col, part[i]);
        }
    } else {
        cluster_sync();  // every partial of the cluster is complete and visible
        if (slice == 0) {
            for (int i = tid; i < SH_TM * R / 4; i += SH_THREADS) {
                const uint32_t la = smem_u32(part + 4 * i);
                float4 v = *reinterpret_cast<const float4*>(part + 4 * i);
                // every peer's piece is requested before the first is used (one round trip, not
                // split - 1); the adds below still run in slice order
                float4 p[SH_MAX_SPLIT];
#pragma unroll
                for (int s = 1; s < SH_MAX_SPLIT; ++s)
                    if (s < split) p[s] = ld_dsmem_v4(mapa(la, (uint32_t)s));
#pragma unroll
                for (int s = 1; s < SH_MAX_SPLIT; ++s) {
                    if (s < split) {
                        v.x = __fadd_rn(v.x, p[s].x);
                        v.y = __fadd_rn(v.y, p[s].y);
                        v.z = __fadd_rn(v.z, p[s].z);
                        v.w = __fadd_rn(v.w, p[s].w);
                    }
                }
                const int row = (4 * i) / R, col = (4 * i) % R;
                if (m0 + row < M) *reinterpret_cast<float4*>(t + (size_t)(m0 + row) * R + col) = v;
            }
        }
        cluster_sync();  // peers keep their shared memory until the leader has read it
    }
}

// ------------------------------------------------------------------ expand
constexpr int EX_TM = 64;
constexpr int EX_TN = 128;
constexpr int EX_THREADS = 256;

template <int R>
struct ExpandLayout {
    static constexpr int RP = R < 16 ? 16 : R;       // K of the MMA, padded with zeros
    static constexpr int T_PITCH = RP * 2 + 16;       // bytes per row of bf16(t); +16 avoids bank conflicts
    static constexpr int B_PITCH = EX_TN * 2 + 16;    // bytes per K-row of the B tile
    static constexpr int D_PITCH = EX_TN + 8;         // floats per row of the staged product (conflict-free)
    static constexpr int T_BYTES = EX_TM * T_PITCH;
    static constexpr int B_BYTES = RP * B_PITCH;
    static constexpr size_t BYTES = (size_t)T_BYTES + B_BYTES + EX_TM * D_PITCH * 4;
};

template <int R, bool YBF16>
__global__ void __launch_bounds__(EX_THREADS)
lora_expand_kernel(const float* __restrict__ t, const __nv_bfloat16* __restrict__ B, void* __restrict__ y, int M,
                   int N, int64_t ldy, float scale) {
    using L = ExpandLayout<R>;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* sT = smem;
    uint8_t* sB = smem + L::T_BYTES;
    float* sD = reinterpret_cast<float*>(smem + L::T_BYTES + L::B_BYTES);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int m0 = blockIdx.y * EX_TM;
    const int n0 = blockIdx.x * EX_TN;

    // 0. Issue this thread's loads of the y tile first: their HBM latency overlaps steps 1-3.
    //    A chunk is 4 consecutive elements of a row (8 bytes of bf16 or 16 of fp32), so that the
    //    matching 16 bytes of the staged product are read without bank conflicts.
    constexpr int CPR = EX_TN / 4;                              // chunks per tile row
    constexpr int NCH = EX_TM * CPR / EX_THREADS;               // chunks per thread (8)
    uint4 yv[NCH];
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
        const int i = tid + k * EX_THREADS;
        const int row = i / CPR, cc = i % CPR;
        const int col = n0 + cc * 4;
        yv[k] = make_uint4(0u, 0u, 0u, 0u);
        if (m0 + row < M && col < N) {
            if constexpr (YBF16) {
                const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(y) +
                                                                 (size_t)(m0 + row) * ldy + col);
                yv[k].x = u.x;
                yv[k].y = u.y;
            } else {
                yv[k] = *reinterpret_cast<const uint4*>(static_cast<const float*>(y) + (size_t)(m0 + row) * ldy + col);
            }
        }
    }

    // 1. bf16(t) rows into shared memory (rows past M and columns past R are zero).
    for (int i = tid; i < EX_TM * L::RP / 4; i += EX_THREADS) {
        const int row = (4 * i) / L::RP, k = (4 * i) % L::RP;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (m0 + row < M && k < R) v = *reinterpret_cast<const float4*>(t + (size_t)(m0 + row) * R + k);
        uint2 p = make_uint2(bi::pack_bf16x2(v.x, v.y), bi::pack_bf16x2(v.z, v.w));
        *reinterpret_cast<uint2*>(sT + row * L::T_PITCH + k * 2) = p;
    }
    // 2. The B tile [R, 128] (columns past N and rows past R are zero).
    for (int i = tid; i < L::RP * (EX_TN / 8); i += EX_THREADS) {
        const int k = i / (EX_TN / 8), cc = i % (EX_TN / 8);
        const int col = n0 + cc * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (k < R && col < N) v = bi::ld_cached_v4(B + (size_t)k * N + col);
        *reinterpret_cast<uint4*>(sB + k * L::B_PITCH + cc * 16) = v;
    }
    __syncthreads();

    // 3. delta[16 rows x 64 cols] per warp with mma.sync.
    const int wr = warp >> 1, wc = warp & 1;
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
    const uint32_t sTa = smem_u32(sT), sBa = smem_u32(sB);
#pragma unroll
    for (int kk = 0; kk < L::RP / 16; ++kk) {
        uint32_t a[4];
        ldmatrix_x4(sTa + (wr * 16 + (lane & 15)) * L::T_PITCH + (kk * 16 + (lane >> 4) * 8) * 2, a);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            uint32_t b[2];
            ldmatrix_x2_trans(sBa + (kk * 16 + (lane & 15)) * L::B_PITCH + (wc * 64 + nt * 8) * 2, b);
            mma_m16n8k16_bf16(acc[nt], a, b);
        }
    }
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int col = wc * 64 + nt * 8 + q * 2;
        *reinterpret_cast<float2*>(sD + (wr * 16 + g) * L::D_PITCH + col) = make_float2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<float2*>(sD + (wr * 16 + g + 8) * L::D_PITCH + col) = make_float2(acc[nt][2], acc[nt][3]);
    }
    __syncthreads();

    // 4. y = round(fma(scale, delta, y)) with coalesced 128-bit accesses.
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
        const int i = tid + k * EX_THREADS;
        const int row = i / CPR, cc = i % CPR;
        const int col = n0 + cc * 4;
        if (m0 + row >= M || col >= N) continue;
        const float4 d = *reinterpret_cast<const float4*>(sD + row * L::D_PITCH + cc * 4);
        if constexpr (YBF16) {
            const float a0 = __fmaf_rn(scale, d.x, bi::bf16_lo(yv[k].x));
            const float a1 = __fmaf_rn(scale, d.y, bi::bf16_hi(yv[k].x));
            const float a2 = __fmaf_rn(scale, d.z, bi::bf16_lo(yv[k].y));
            const float a3 = __fmaf_rn(scale, d.w, bi::bf16_hi(yv[k].y));
            __nv_bfloat16* p = static_cast<__nv_bfloat16*>(y) + (size_t)(m0 + row) * ldy + col;
            *reinterpret_cast<uint2*>(p) = make_uint2(bi::pack_bf16x2(a0, a1), bi::pack_bf16x2(a2, a3));
        } else {
            float4 v = make_float4(__uint_as_float(yv[k].x), __uint_as_float(yv[k].y), __uint_as_float(yv[k].z),
                                   __uint_as_float(yv[k].w));
            v.x = __fmaf_rn(scale, d.x, v.x);
            v.y = __fmaf_rn(scale, d.y, v.y);
            v.z = __fmaf_rn(scale, d.z, v.z);
            v.w = __fmaf_rn(scale, d.w, v.w);
            float* p = static_cast<float*>(y) + (size_t)(m0 + row) * ldy + col;
            *reinterpret_cast<float4*>(p) = v;
        }
    }
}

// ------------------------------------------------------------------ host side
template <typename F>
bool set_smem_once(F kernel, size_t bytes) {
    // one attribute call per (kernel, device); cheap enough to guard with a small table
    static std::mutex mu;
    static const void* done_k[256];
    static int done_d[256];
    static int n = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (done_k[i] == (const void*)kernel && done_d[i] == dev) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    if (n < 256) {
        done_k[n] = (const void*)kernel;
        done_d[n] = dev;
        ++n;
    }
    return true;
}

template <int R, bool ATOMIC>
int launch_shrink(const void* x, const void* A, float* t, int64_t M, int64_t K, int split, cudaStream_t s) {
    using L = ShrinkLayout<R>;
    uint32_t* err = bi::device_error_word();
    auto kern = lora_shrink_kernel<R, ATOMIC>;
    if (!err || !set_smem_once(kern, L::BYTES)) return BI_ERR_CUDA;
    CUtensorMap tmX, tmA;
    if (!bi::make_tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2,
                          SH_KC, SH_TM, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    if (!bi::make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)R, (uint64_t)K, (uint64_t)R * 2, R,
                          SH_KC, bi::swizzle_for(R * 2)))
        return BI_ERR_CUDA;
    const int KS = (int)(K / split);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((M + SH_TM - 1) / SH_TM), (unsigned)split, 1);
    cfg.blockDim = dim3(SH_THREADS, 1, 1);
    cfg.dynamicSmemBytes = L::BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (!ATOMIC) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = (unsigned)split;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    if (cudaLaunchKernelEx(&cfg, kern, tmX, tmA, t, (int)M, KS, split, err) != cudaSuccess) return BI_ERR_CUDA;
    return bi::launch_status();
}

template <bool ATOMIC>
int shrink_dispatch(const void* x, const void* A, float* t, int64_t M, int64_t K, int32_t r, int32_t split,
                    cudaStream_t s) {
    switch (r) {
        case 8: return launch_shrink<8, ATOMIC>(x, A, t, M, K, split, s);
        case 16: return launch_shrink<16, ATOMIC>(x, A, t, M, K, split, s);
        case 32: return launch_shrink<32, ATOMIC>(x, A, t, M, K, split, s);
        case 64: return launch_shrink<64, ATOMIC>(x, A, t, M, K, split, s);
        default: return BI_ERR_UNSUPPORTED_SHAPE;
    }
}

int shrink_checks(const void* x, const void* A, const float* t, int64_t M, int64_t K, int32_t r, int32_t split) {
    if (M < 0 || K <= 0 || r <= 0) return BI_ERR_INVALID_ARG;
    if (split != 1 && split != 2 && split != 4 && split != 8) return BI_ERR_UNSUPPORTED_SHAPE;
    if (r != 8 && r != 16 && r != 32 && r != 64) return BI_ERR_UNSUPPORTED_SHAPE;
    if (K % ((int64_t)split * SH_KC) != 0) return BI_ERR_UNSUPPORTED_SHAPE;
    if (M > ((int64_t)1 << 31) - SH_TM || K > (1LL << 30)) return BI_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return -1;  // no-op
    if (!x || !A || !t) return BI_ERR_INVALID_ARG;
    if (!bi::aligned16(x) || !bi::aligned16(A) || !bi::aligned16(t)) return BI_ERR_MISALIGNED;
    return BI_OK;
}

template <int R>
int launch_expand(const float* t, const void* B, void* y, int64_t M, int64_t N, int64_t ldy, float scale, bool ybf16,
                  cudaStream_t s) {
    using L = ExpandLayout<R>;
    dim3 grid((unsigned)((N + EX_TN - 1) / EX_TN), (unsigned)((M + EX_TM - 1) / EX_TM));
    if (ybf16) {
        auto k = lora_expand_kernel<R, true>;
        if (!set_smem_once(k, L::BYTES)) return BI_ERR_CUDA;
        k<<<grid, EX_THREADS, L::BYTES, s>>>(t, static_cast<const __nv_bfloat16*>(B), y, (int)M, (int)N, ldy, scale);
    } else {
        auto k = lora_expand_kernel<R, false>;
        if (!set_smem_once(k, L::BYTES)) return BI_ERR_CUDA;
        k<<<grid, EX_THREADS, L::BYTES, s>>>(t, static_cast<const __nv_bfloat16*>(B), y, (int)M, (int)N, ldy, scale);
    }
    return bi::launch_status();
}

}  // namespace

BI_API size_t bi_lora_shrink_workspace_size(int64_t M, int64_t K, int32_t r, int32_t split_k) {
    (void)M; (void)K; (void)r; (void)split_k;
    return 0;
}

BI_API int bi_lora_shrink(const void* x, const void* A, float* t, int64_t M, int64_t K, int32_t r, int32_t split_k,
                          void* ws, size_t ws_bytes, void* stream) {
    (void)ws; (void)ws_bytes;
    const int c = shrink_checks(x, A, t, M, K, r, split_k);
    if (c < 0) return BI_OK;
    if (c != BI_OK) return c;
    return shrink_dispatch<false>(x, A, t, M, K, r, split_k, bi::as_stream(stream));
}

BI_API int bi_ctrl_lora_shrink_atomic(const void* x, const void* A, float* t, int64_t M, int64_t K, int32_t r,
                                      int32_t split_k, void* stream) {
    const int c = shrink_checks(x, A, t, M, K, r, split_k);
    if (c < 0) return BI_OK;
    if (c != BI_OK) return c;
    cudaStream_t s = bi::as_stream(stream);
    if (cudaMemsetAsync(t, 0, (size_t)M * r * sizeof(float), s) != cudaSuccess) return BI_ERR_CUDA;
    return shrink_dispatch<true>(x, A, t, M, K, r, split_k, s);
}

BI_API int bi_lora_expand(const float* t, const void* B, void* y, int64_t M, int32_t r, int64_t N, int64_t ldy,
                          float scale, int y_dtype, void* stream) {
    if (y_dtype != BI_F32 && y_dtype != BI_BF16) return BI_ERR_INVALID_ARG;
    if (M < 0 || N <= 0 || r <= 0 || ldy < N) return BI_ERR_INVALID_ARG;
    if (r != 8 && r != 16 && r != 32 && r != 64) return BI_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return BI_OK;
    if (!t || !B || !y) return BI_ERR_INVALID_ARG;
    if (!bi::aligned16(t) || !bi::aligned16(B) || !bi::aligned16(y)) return BI_ERR_MISALIGNED;
    if (N % 8 != 0 || (ldy * bi::elem_size(y_dtype)) % 16 != 0) return BI_ERR_MISALIGNED;
    if (M > 65535LL * EX_TM || N > (1LL << 31) - EX_TN) return BI_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = bi::as_stream(stream);
    const bool yb = y_dtype == BI_BF16;
    switch (r) {
        case 8: return launch_expand<8>(t, B, y, M, N, ldy, scale, yb, s);
        case 16: return launch_expand<16>(t, B, y, M, N, ldy, scale, yb, s);
        case 32: return launch_expand<32>(t, B, y, M, N, ldy, scale, yb, s);
        default: return launch_expand<64>(t, B, y, M, N, ldy, scale, yb, s);
    }
}
