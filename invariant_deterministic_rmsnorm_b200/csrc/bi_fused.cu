// bi_fused.cu -- RMSNorm and the LoRA shrink of its output in one pass over x.
//
// Sources: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section "Diseño de
// kernels invariantes al batch", RMSNorm; "Reproducible LoRA Inference Through Deterministic
// Split-K Reduction" (abstract).  The normalised rows y feed the base projection and the LoRA
// shrink t = y . A.  Run apart, the shrink reads y back from HBM right after the RMSNorm wrote
// it.  Here the CTA that normalises a row also multiplies it by A while the row is still in its
// shared memory, so y is read from HBM once (as x) and written once.
//
// Both results are bitwise those of the two separate calls (bi_rmsnorm, then bi_lora_shrink on
// its output), because every output element goes through the same operations in the same
// order:
//   - RMSNorm (H = 4096, bf16): thread t of 256 owns 16-byte vectors t and t + 256 of a row,
//     sums their squares with sequential FMAs, joins the warp's butterfly and then a butterfly
//     over the eight warp sums; inv = rsqrt(sum / H + eps), y = (x * inv) * w with two roundings
//     and one rounding to bf16.  That is bi_rmsnorm's plan for H = 4096, statement for statement.
//   - shrink (split_k = 8, r = 8 or 16): warp s computes the partial of K slice s (512 columns)
//     with mma.sync m16n8k16 in 32 ascending 16-deep steps from zero, on the same fragment
//     contents as bi_lora_shrink's ldmatrix loads give, and t = ((P_0 + P_1) + ...) + P_7 in
//     fp32, each add rounded to nearest.  An m16 fragment holds 16 rows; a tile has 8, and the
//     other 8 rows are zero (a row's MMA result depends on that row alone).
// Warp s keeps the B fragments of its slice of A in registers for the CTA's lifetime (32 steps
// x r / 8 column blocks x 2 registers: 128 registers at r = 16), so A is read once per CTA
// (staged through shared memory and taken with ldmatrix .trans, as the shrink kernel does).
//
// Data flow: persistent CTAs, one per SM, walk tiles of 8 rows (tile i, i + grid, ...).  A ring
// of shared-memory stages holds whole rows of x.  Every thread fetches the 16-byte vectors it
// owns with cp.async (one commit group per tile), so the ring keeps two tiles of loads in flight
// without holding them in registers while the CTA works on the third.  Per tile: sums of
// squares, the inverse norms, y over x in the stage (and from there to HBM, one bulk copy per
// row), the eight slice MMAs, the ordered combine, t stored.  Which CTA handles a tile never changes a row's
// arithmetic.
//
// Measured on a B200 against the two calls launched back to back: the same time at M = 256,
// 9-26 % less at M = 1024 ... 8192 (the spread is between boxes).  A tile costs about 3.4 us of latency-bound row and MMA work: one CTA of
// eight warps per SM (the resident A slices take 128 registers a thread) has far less
// parallelism than bi_rmsnorm's eight CTAs per SM.
#include <mutex>
#include "bi_common.cuh"
#include "bi_sm100.cuh"

using namespace bi::sm100;

namespace {

constexpr int FU_THREADS = 256;   // bi_rmsnorm's block for H = 4096 bf16 (512 vectors, two per thread)
constexpr int FU_WARPS = FU_THREADS / 32;
constexpr int FU_H = 4096;
constexpr int FU_VEC = 8;         // bf16 per 16-byte vector
constexpr int FU_NVEC = FU_H / FU_VEC;
constexpr int FU_VPT = FU_NVEC / FU_THREADS;  // 2
constexpr int FU_ROWS = 8;        // rows per tile: the first 8 rows of every m16 fragment
constexpr int FU_SPLIT = 8;       // K slices: one per warp
constexpr int FU_KS = FU_H / FU_SPLIT;        // 512 columns per slice
constexpr int FU_STEPS = FU_KS / 16;          // 32 mma k-steps per slice
constexpr int FU_ROW_BYTES = FU_H * 2;        // 8 KB
// rows sit 8 KB + 16 B apart in a stage, so that the eight rows of an MMA fragment fall in
// different shared-memory banks
constexpr int FU_PITCH = FU_ROW_BYTES + 16;
constexpr int FU_STAGE = FU_ROWS * FU_PITCH;  // 64 KB + 128 B
constexpr int FU_STAGES = 3;                  // 192 KB of rows in flight

// 16 bytes global -> shared without a register round trip (cached in L2 only)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }
// `bytes` (a multiple of 16, both addresses 16-byte aligned) shared -> global by the copy engine
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :: "l"(reinterpret_cast<uint64_t>(dst)), "r"(src), "r"(bytes) : "memory");
}

template <int R>
struct FusedLayout {
    static constexpr int P_OFF = FU_STAGES * FU_STAGE;
    static constexpr int P_BYTES = FU_SPLIT * FU_ROWS * R * 4;  // the slices' partials of a tile
    static constexpr size_t BYTES = (size_t)P_OFF + P_BYTES;
};

template <int R>
__global__ void __launch_bounds__(FU_THREADS, 1)
rmsnorm_lora_shrink_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w,
                           __nv_bfloat16* __restrict__ y, const __nv_bfloat16* __restrict__ A, float* __restrict__ t,
                           int M, int64_t ldx, int64_t ldy, float eps, int n_tiles) {
    using L = FusedLayout<R>;
    extern __shared__ __align__(16) uint8_t smem[];
    float* P = reinterpret_cast<float*>(smem + L::P_OFF);  // [slice][row][R]
    __shared__ float warp_sums[FU_ROWS][FU_WARPS];
    __shared__ float inv_s[FU_ROWS];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int g = lane >> 2, q = lane & 3;  // the mma fragment's row group and column pair
    const uint32_t sbase = smem_u32(smem);

    // the weights of this thread's two vectors, as raw bf16 pairs (bi_rmsnorm keeps them the same way)
    uint32_t wr[FU_VPT][4];
    // B fragments of this warp's K slice: step j, column block nt, k rows 2q, 2q+1 and 2q+8, 2q+9
    uint32_t bfr[FU_STEPS][R / 8][2];
    pdl_wait();  // x, w and A may come from the kernel before this one; it may still read y or t
    pdl_trigger();
#pragma unroll
    for (int i = 0; i < FU_VPT; ++i) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(w + (int64_t)(tid + i * FU_THREADS) * FU_VEC);
#pragma unroll
        for (int k = 0; k < 4; ++k) wr[i][k] = __ldg(src + k);
    }
    // every thread fetches its own vectors of a tile's rows into a stage: one commit group per
    // tile (empty past the last tile, so that the group count stays the same on every thread)
    auto issue = [&](int tile, int stage) {
        if (tile < n_tiles) {
            const int row0 = tile * FU_ROWS;
            const int rows = M - row0 < FU_ROWS ? M - row0 : FU_ROWS;
            for (int r = 0; r < rows; ++r)
#pragma unroll
                for (int i = 0; i < FU_VPT; ++i) {
                    const int v = tid + i * FU_THREADS;
                    cp_async16(sbase + (uint32_t)(stage * FU_STAGE + r * FU_PITCH + v * 16),
                               x + (int64_t)(row0 + r) * ldx + (int64_t)v * FU_VEC);
                }
        }
        cp_async_commit();
    };
    // A [H, R] into stages 1 and 2 (still empty) while the first tile's rows come into stage 0;
    // then each warp takes its fragments with ldmatrix .trans: the same register contents
    // bi_lora_shrink's kernel loads per step
    const uint32_t a_smem = sbase + (uint32_t)FU_STAGE;
#pragma unroll 4
    for (int i = tid; i < FU_H * R * 2 / 16; i += FU_THREADS)
        cp_async16(a_smem + (uint32_t)(i * 16), reinterpret_cast<const uint8_t*>(A) + (size_t)i * 16);
    cp_async_commit();
    issue(blockIdx.x, 0);
    cp_async_wait<1>();  // A has landed (the first tile may still be in flight)
    __syncthreads();
#pragma unroll
    for (int j = 0; j < FU_STEPS; ++j) {
        const int krow = warp * FU_KS + j * 16 + (lane & 15);
#pragma unroll
        for (int nt = 0; nt < R / 8; ++nt) ldmatrix_x2_trans(a_smem + (uint32_t)(krow * R * 2 + nt * 16), bfr[j][nt]);
    }
    __syncthreads();  // every warp has its fragments before stages 1 and 2 are overwritten
    for (int s = 1; s < FU_STAGES; ++s) issue(blockIdx.x + s * gridDim.x, s);

    const float h_float = (float)FU_H;
    int j = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
        const int stage = j % FU_STAGES;
        const int row0 = tile * FU_ROWS;
        const int rows = M - row0 < FU_ROWS ? M - row0 : FU_ROWS;
        // this thread's vectors of the tile have landed (at most the two later tiles' groups pend);
        // phases 1 and 3 read only those, and the barrier after phase 3 publishes y to the MMA warps
        cp_async_wait<FU_STAGES - 1>();

        const uint8_t* st = smem + stage * FU_STAGE;  // this tile's rows, row r at r * FU_PITCH
        // 1. per row: this thread's sum of squares, vectors in order, elements in order; the warp
        //    butterfly.  A full tile works on four rows at a time so that their loads and chains
        //    overlap; every row still goes through exactly its own sequence of operations.
        if (rows == FU_ROWS) {
#pragma unroll
            for (int rg = 0; rg < FU_ROWS; rg += 4) {
                uint4 u[4][FU_VPT];
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int i = 0; i < FU_VPT; ++i)
                        u[r][i] = *reinterpret_cast<const uint4*>(st + (rg + r) * FU_PITCH + (tid + i * FU_THREADS) * 16);
                float ss[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int i = 0; i < FU_VPT; ++i)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const uint4 v = u[r][i];
                        const float f[8] = {bi::bf16_lo(v.x), bi::bf16_hi(v.x), bi::bf16_lo(v.y), bi::bf16_hi(v.y),
                                            bi::bf16_lo(v.z), bi::bf16_hi(v.z), bi::bf16_lo(v.w), bi::bf16_hi(v.w)};
#pragma unroll
                        for (int e = 0; e < 8; ++e) ss[r] = __fmaf_rn(f[e], f[e], ss[r]);
                    }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int r = 0; r < 4; ++r) ss[r] = __fadd_rn(ss[r], __shfl_xor_sync(0xffffffffu, ss[r], off));
                if (lane == 0) {
#pragma unroll
                    for (int r = 0; r < 4; ++r) warp_sums[rg + r][warp] = ss[r];
                }
            }
        } else {
            for (int r = 0; r < rows; ++r) {
                float ss = 0.0f;
#pragma unroll
                for (int i = 0; i < FU_VPT; ++i) {
                    const uint4 u = *reinterpret_cast<const uint4*>(st + r * FU_PITCH + (tid + i * FU_THREADS) * 16);
                    const float f[8] = {bi::bf16_lo(u.x), bi::bf16_hi(u.x), bi::bf16_lo(u.y), bi::bf16_hi(u.y),
                                        bi::bf16_lo(u.z), bi::bf16_hi(u.z), bi::bf16_lo(u.w), bi::bf16_hi(u.w)};
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = __fmaf_rn(f[e], f[e], ss);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
                if (lane == 0) warp_sums[r][warp] = ss;
            }
        }
        __syncthreads();
        // 2. the fixed tree over the eight warp sums (warp r for row r), then the inverse norm
        if (warp < rows) {
            float s = lane < FU_WARPS ? warp_sums[warp][lane] : 0.0f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
            if (lane == 0) inv_s[warp] = __frsqrt_rn(__fadd_rn(__fdiv_rn(s, h_float), eps));
        }
        __syncthreads();
        // 3. y = (x * inv) * w, rounded once to bf16: to HBM, and over x in the stage for the MMAs
        {
            float wf[FU_VPT][8];
#pragma unroll
            for (int i = 0; i < FU_VPT; ++i)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    wf[i][2 * k] = bi::bf16_lo(wr[i][k]);
                    wf[i][2 * k + 1] = bi::bf16_hi(wr[i][k]);
                }
            auto norm_row = [&](int r, int i, const uint4& u) {
                const float inv = inv_s[r];
                const int v = tid + i * FU_THREADS;
                float f[8] = {bi::bf16_lo(u.x), bi::bf16_hi(u.x), bi::bf16_lo(u.y), bi::bf16_hi(u.y),
                              bi::bf16_lo(u.z), bi::bf16_hi(u.z), bi::bf16_lo(u.w), bi::bf16_hi(u.w)};
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(__fmul_rn(f[e], inv), wf[i][e]);
                const uint4 o = make_uint4(bi::pack_bf16x2(f[0], f[1]), bi::pack_bf16x2(f[2], f[3]),
                                           bi::pack_bf16x2(f[4], f[5]), bi::pack_bf16x2(f[6], f[7]));
                *reinterpret_cast<uint4*>(smem + stage * FU_STAGE + r * FU_PITCH + v * 16) = o;
            };
            if (rows == FU_ROWS) {
#pragma unroll
                for (int rg = 0; rg < FU_ROWS; rg += 4) {
                    uint4 u[4][FU_VPT];
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int i = 0; i < FU_VPT; ++i)
                            u[r][i] = *reinterpret_cast<const uint4*>(st + (rg + r) * FU_PITCH + (tid + i * FU_THREADS) * 16);
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int i = 0; i < FU_VPT; ++i) norm_row(rg + r, i, u[r][i]);
                }
            } else {
                for (int r = 0; r < rows; ++r)
#pragma unroll
                    for (int i = 0; i < FU_VPT; ++i)
                        norm_row(r, i, *reinterpret_cast<const uint4*>(st + r * FU_PITCH + (tid + i * FU_THREADS) * 16));
            }
        }
        // y leaves for HBM from the stage, one bulk copy per row (the copy engine reads what the
        // threads wrote: their generic writes are ordered before its async-proxy reads)
        fence_proxy_async_shared();
        __syncthreads();
        if (tid == 0) {
            for (int r = 0; r < rows; ++r)
                bulk_store(y + (int64_t)(row0 + r) * ldy, sbase + (uint32_t)(stage * FU_STAGE + r * FU_PITCH),
                           (uint32_t)FU_ROW_BYTES);
            bulk_commit();
        }
        // 4. warp s: the partial of K slice s over the tile's rows, 32 mma steps from zero.  Row g of
        //    the fragment is tile row g (zero past the last row), rows g + 8 are zero.
        {
            float acc[R / 8][4];
#pragma unroll
            for (int nt = 0; nt < R / 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
            const bool live = g < rows;
            const uint32_t* yrow = reinterpret_cast<const uint32_t*>(st + g * FU_PITCH + warp * FU_KS * 2) + q;
#pragma unroll
            for (int s = 0; s < FU_STEPS; ++s) {
                uint32_t a[4];
                a[0] = live ? yrow[s * 8] : 0u;      // row g, k 2q, 2q+1 of the step
                a[1] = 0u;                           // row g + 8
                a[2] = live ? yrow[s * 8 + 4] : 0u;  // row g, k 2q+8, 2q+9
                a[3] = 0u;
#pragma unroll
                for (int nt = 0; nt < R / 8; ++nt) mma_m16n8k16_bf16(acc[nt], a, bfr[s][nt]);
            }
            if (live) {
#pragma unroll
                for (int nt = 0; nt < R / 8; ++nt) {
                    float* d = P + (warp * FU_ROWS + g) * R + nt * 8 + 2 * q;
                    d[0] = acc[nt][0];
                    d[1] = acc[nt][1];
                }
            }
        }
        __syncthreads();
        // 5. t = ((P_0 + P_1) + ...) + P_7 per element, in slice order
        if (tid < rows * R) {
            const int r = tid / R, c = tid % R;
            float v = P[r * R + c];
#pragma unroll
            for (int sl = 1; sl < FU_SPLIT; ++sl) v = __fadd_rn(v, P[(sl * FU_ROWS + r) * R + c]);
            t[(int64_t)(row0 + r) * R + c] = v;
        }
        // 6. every read of the stage (the MMA warps' and the copy engine's included) is done: refill it
        if (tid == 0) bulk_wait_read();
        __syncthreads();
        issue(tile + FU_STAGES * (int)gridDim.x, stage);
    }
    cp_async_wait<0>();  // nothing may still write this CTA's shared memory when it exits
    if (tid == 0) bulk_wait_all();  // and y has reached global memory
}

template <int R>
int launch_fused(const void* x, const void* w, void* y, const void* A, float* t, int64_t M, int64_t ldx,
                 int64_t ldy, float eps, cudaStream_t s) {
    using L = FusedLayout<R>;
    static std::once_flag once[64];
    static bool attr_ok[64];
    static int sms_cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BI_ERR_CUDA;
    std::call_once(once[dev], [&] {
        attr_ok[dev] = cudaFuncSetAttribute(rmsnorm_lora_shrink_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)L::BYTES) == cudaSuccess &&
                       cudaDeviceGetAttribute(&sms_cached[dev], cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
    });
    if (!attr_ok[dev] || sms_cached[dev] <= 0) return BI_ERR_CUDA;
    const int64_t n_tiles = (M + FU_ROWS - 1) / FU_ROWS;
    const int64_t grid = n_tiles < sms_cached[dev] ? n_tiles : sms_cached[dev];
    if (bi::launch_pdl(rmsnorm_lora_shrink_kernel<R>, dim3((unsigned)grid), dim3(FU_THREADS), L::BYTES, s, 0u,
                       static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w),
                       static_cast<__nv_bfloat16*>(y), static_cast<const __nv_bfloat16*>(A), t, (int)M, ldx, ldy, eps,
                       (int)n_tiles) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

}  // namespace

BI_API int bi_rmsnorm_lora_shrink(const void* x, const void* w, void* y, const void* A, float* t, int64_t M,
                                  int64_t H, int64_t ldx, int64_t ldy, float eps, int32_t r, int32_t split_k,
                                  void* stream) {
    if (M < 0 || H <= 0 || ldx < H || ldy < H || !(eps >= 0.0f) || r <= 0 || split_k <= 0) return BI_ERR_INVALID_ARG;
    if (M == 0) return BI_OK;
    if (!x || !w || !y || !A || !t) return BI_ERR_INVALID_ARG;
    if (H != FU_H || split_k != FU_SPLIT || (r != 8 && r != 16)) return BI_ERR_UNSUPPORTED_SHAPE;
    if (M > 0x7fffffffLL - FU_ROWS) return BI_ERR_UNSUPPORTED_SHAPE;
    if ((ldx * 2) % 16 != 0 || (ldy * 2) % 16 != 0) return BI_ERR_MISALIGNED;
    if (!bi::aligned16(x) || !bi::aligned16(w) || !bi::aligned16(y) || !bi::aligned16(A) || !bi::aligned16(t))
        return BI_ERR_MISALIGNED;
    if (y == x && ldy != ldx) return BI_ERR_INVALID_ARG;
    cudaStream_t s = bi::as_stream(stream);
    return r == 8 ? launch_fused<8>(x, w, y, A, t, M, ldx, ldy, eps, s)
                  : launch_fused<16>(x, w, y, A, t, M, ldx, ldy, eps, s);
}
