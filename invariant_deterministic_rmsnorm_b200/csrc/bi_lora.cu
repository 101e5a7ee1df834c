// bi_lora.cu -- batch-invariant LoRA shrink (deterministic split-K) and expand.
//
// Source: "Reproducible LoRA Inference Through Deterministic Split-K Reduction" (abstract).
// Split-K kernels parallelise the low-rank LoRA products.  If they combine partial results
// with floating-point atomic additions, repeated runs differ.  The deterministic variant
// keeps Split-K = 8 and combines the partials in a fixed order, so the FP32 shrink output
// is identical under replay.
//
// Shrink, t[M, r] = x[M, K] . A[K, r]:
//   The partial P_s of slice s covers the contiguous K slice [s*K/split, (s+1)*K/split).  It is
//   accumulated in fp32 from bf16 products in 16-deep K steps in ascending order, starting from
//   zero: with mma.sync m16n8k16 at r = 8, 16, 32, with tcgen05.mma at r = 64 (below).  The
//   output is t = ((P_0 + P_1) + P_2) + ... + P_{split-1}, every add rounded to nearest.  There
//   is no atomic, and the split count and slice size depend only on (K, split), never on M.  A
//   thread-block cluster of `split` CTAs computes tiles of 64 or 128 rows (by r): CTA s streams x
//   and A of its slice through a TMA ring, each compute warp owns 16 rows, and the partials meet
//   on chip (distributed shared memory), never in HBM.  The ordered kernel
//   (lora_shrink_ordered_kernel) is persistent and spreads the combine over every CTA of the
//   cluster; the atomic comparator (lora_shrink_atomic_kernel) adds the partials into t with
//   floating-point atomics instead.
//
// Expand, y[M, N] += scale * bf16(t)[M, r] . B[r, N]:
//   64 x 128 tiles of y per CTA.  t is rounded to bf16 (nearest even) into shared memory,
//   zero-padded to 16 when r = 8.  The product comes from mma.sync into fp32 registers and goes
//   straight to y in 16-byte pieces: y = round(fma(scale, delta, y)).
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

// The comparator: one CTA per (128-row tile, K slice), partials added into t by floating-point
// atomics in whatever order the CTAs finish.
template <int R>
__global__ void __launch_bounds__(SH_THREADS, 1)
lora_shrink_atomic_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                          float* __restrict__ t, int M, int KS, uint32_t* err) {
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
    const uint32_t slice = blockIdx.y;
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
            release_stage(smem_u32(&empty[st]), lane);
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

    __syncwarp();
    __syncthreads();
    for (int i = tid; i < SH_TM * R; i += SH_THREADS) {
        const int row = i / R, col = i % R;
        if (m0 + row < M) atomicAdd(t + (size_t)(m0 + row) * R + col, part[i]);
    }
}

// ------------------------------------------------------------------ shrink, ordered combine
// The batch-invariant shrink.  Each output element is computed exactly as described at the top
// of this file: slice s's partial is one mma.sync chain over its K slice, and the partials are
// added in slice order.  What this kernel changes is where and when that happens:
//   - Persistent clusters.  A cluster of `split` CTAs (CTA s = slice s) walks tiles c,
//     c + clusters, ...; its producer warp keeps one TMA ring streaming across tiles, so a
//     cluster's next tile loads while its last one is being exchanged and combined.  Tiles have
//     TM = 64 rows from r = 16 (a cluster then has two at M = 4096 on this GPU, where one tile of
//     128 left that tail bare, and twice the CTAs share a small batch) and 128 rows at r = 8; a
//     row's arithmetic does not depend on the tile height.
//   - Distributed, pushed combine.  Compute warp w owns rows [16w, 16w + 16) of the tile; CTA d
//     combines rows [TM d / split, TM (d + 1) / split).  When its chain ends, a warp stages its
//     rows of the partial in its own shared memory as the combining CTA's buffer holds them and
//     sends them with one bulk copy per combining CTA (two when a CTA combines 8 rows), which
//     completes on that CTA's receive barrier.  A combiner warp in every CTA waits for the bytes,
//     adds its rows' split partials from its own shared memory in slice order, writes t, and
//     hands the buffer back to every sender with a remote arrive.  No CTA reads a peer's shared
//     memory.
// Every wait is bounded.  A cluster barrier at the end keeps each CTA's shared memory alive until
// no peer can still write into it.
constexpr int SO_MAX_STAGES = 8;   // a whole 512-column slice of a tile in flight

// Tile height by rank (a row's arithmetic does not depend on it): 64 rows from r = 16, where
// the measured shrink is 2-20 % faster than with 128-row tiles, and 128 rows at r = 8, where it
// is 2-6 % slower.
template <int R>
struct OrderedShape {
    static constexpr int TM = R >= 16 ? 64 : 128;           // rows per tile
    static constexpr int CWARPS = TM / 16;                   // compute warps, 16 rows each
    static constexpr int THREADS = (CWARPS + 2) * 32;        // compute warps, a producer warp, a combiner warp
};

template <int R>
struct OrderedLayout {
    static constexpr int SO_TM = OrderedShape<R>::TM;
    static constexpr int X_STAGE = SO_TM * SH_KC * 2;  // 8 or 16 KB, 128B-swizzled rows of 64 K
    static constexpr int A_STAGE = SH_KC * R * 2;
    static constexpr int STAGE = X_STAGE + A_STAGE;    // a multiple of 1 KB
    static constexpr int NB = 1;                       // receive buffers
    static constexpr int RECV = SO_TM * R * 4;         // one buffer: [slice][rows this CTA combines][R] fp32
    // every compute warp stages its 16 rows of partials here before its bulk copies send them
    static constexpr int STAGING = SO_TM * R * 4;
    // two CTAs per SM: at most 112 KB each, including the 1 KB alignment pad and the barriers
    static constexpr int BUDGET = 112 * 1024 - 1024 - 256;
    static constexpr int STAGES_FIT = (BUDGET - NB * RECV - STAGING) / STAGE;
    static constexpr int STAGES = STAGES_FIT > SO_MAX_STAGES ? SO_MAX_STAGES : STAGES_FIT;
    static_assert(STAGES >= 3, "the ring needs at least three stages");
    static constexpr int RECV_OFF = STAGES * STAGE;
    static constexpr int STAGING_OFF = RECV_OFF + NB * RECV;
    static constexpr int BAR_OFF = STAGING_OFF + STAGING;
    // full[STAGES], empty[STAGES], rfull[NB], rfree[NB][SH_MAX_SPLIT], then the abort flag
    static constexpr int NBARS = 2 * STAGES + NB + NB * SH_MAX_SPLIT;
    static constexpr size_t BYTES = 1024 + (size_t)BAR_OFF + NBARS * 8 + 16;
    static constexpr uint32_t A_MASK = R == 64 ? 7u : (R == 32 ? 3u : (R == 16 ? 1u : 0u));
};

template <int R>
__global__ void __launch_bounds__(OrderedShape<R>::THREADS, 2)
lora_shrink_ordered_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                           float* __restrict__ t, int M, int KS, int split, int n_tiles, uint32_t* err) {
    using L = OrderedLayout<R>;
    constexpr int SO_TM = OrderedShape<R>::TM;
    constexpr int SO_CWARPS = OrderedShape<R>::CWARPS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* recv = reinterpret_cast<float*>(base + L::RECV_OFF);
    float* staging = reinterpret_cast<float*>(base + L::STAGING_OFF);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L::BAR_OFF);
    uint64_t* empty = full + L::STAGES;
    uint64_t* rfull = empty + L::STAGES;        // [NB]: every slice's partial of this CTA's rows has landed
    uint64_t* rfree = rfull + L::NB;            // [NB][8]: CTA d's receive buffer b may be written again
    volatile int* abort = reinterpret_cast<volatile int*>(rfree + L::NB * SH_MAX_SPLIT);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t slice = cluster_ctarank();
    const int kbase = (int)slice * KS;
    const int nchunks = KS / SH_KC;
    const int rows_per = SO_TM / split;  // rows of a tile that each CTA combines (8 or more)

    if (tid == 0) {
        for (int i = 0; i < L::STAGES; ++i) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), SO_CWARPS);
        }
        for (int b = 0; b < L::NB; ++b) {
            mbar_init(smem_u32(&rfull[b]), 1);  // per tile: this CTA's expected bytes, then the copies
            for (int d = 0; d < SH_MAX_SPLIT; ++d) mbar_init(smem_u32(&rfree[b * SH_MAX_SPLIT + d]), 1);
        }
        *abort = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    __syncthreads();
    cluster_sync();  // every CTA's barriers exist before any signal crosses the cluster
    pdl_wait();      // x and A may come from the kernel before this one; it may still read t
    pdl_trigger();

    if (warp == SO_CWARPS) {
        // ------------------------------------------------ producer: one ring across all tiles
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmA);
            uint32_t it = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x) {
                for (int c = 0; c < nchunks; ++c, ++it) {
                    const int st = (int)(it % L::STAGES);
                    const uint32_t round = it / L::STAGES;
                    if (!mbar_wait(smem_u32(&empty[st]), (round & 1u) ^ 1u, abort)) {
                        atomicOr(err, bi::DEVERR_WAIT_TMA);
                        *abort = 1;
                        break;
                    }
                    uint8_t* sx = base + st * L::STAGE;
                    const uint32_t fb = smem_u32(&full[st]);
                    mbar_arrive_expect_tx(fb, L::STAGE);
                    tma_load_2d(smem_u32(sx), &tmX, kbase + c * SH_KC, tile * SO_TM, fb);
                    tma_load_2d(smem_u32(sx + L::X_STAGE), &tmA, 0, kbase + c * SH_KC, fb);
                }
            }
            if (*abort) {  // let loads already in flight land before the shared memory is released
                for (uint32_t i = it > (uint32_t)L::STAGES ? it - L::STAGES : 0u; i < it; ++i)
                    (void)mbar_wait(smem_u32(&full[i % L::STAGES]), (i / L::STAGES) & 1u, nullptr);
            }
        }
    } else if (warp == SO_CWARPS + 1) {
        // ------------------------------------------------ combiner: this CTA's rows of every tile
        const uint32_t tile_bytes = (uint32_t)(SO_TM * R * 4);  // every slice of this CTA's rows
        if (lane == 0 && (int)blockIdx.x < n_tiles) mbar_arrive_expect_tx(smem_u32(&rfull[0]), tile_bytes);
        int j = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
            const int b = j % L::NB;
            const uint32_t par = (uint32_t)(j / L::NB) & 1u;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_cluster(smem_u32(&rfull[b]), par, abort));
            if (!ok) {
                if (lane == 0) atomicOr(err, bi::DEVERR_WAIT_CLUSTER);
                *abort = 1;
                break;
            }
            const float* rb = recv + b * (SO_TM * R);  // [slice][rows_per][R]
            const int row0 = tile * SO_TM + (int)slice * rows_per;
            for (int i = lane; i < rows_per * R / 4; i += 32) {
                const int row = (4 * i) / R, col = (4 * i) % R;
                float4 v = *reinterpret_cast<const float4*>(rb + row * R + col);
                for (int sl = 1; sl < split; ++sl) {  // ((P0 + P1) + P2) + ...: slice order
                    const float4 p = *reinterpret_cast<const float4*>(rb + (sl * rows_per + row) * R + col);
                    v.x = __fadd_rn(v.x, p.x);
                    v.y = __fadd_rn(v.y, p.y);
                    v.z = __fadd_rn(v.z, p.z);
                    v.w = __fadd_rn(v.w, p.w);
                }
                if (row0 + row < M) *reinterpret_cast<float4*>(t + (size_t)(row0 + row) * R + col) = v;
            }
            __syncwarp();
            // the next tile's bytes, posted before any sender may send them
            if (lane == 0 && tile + (int)gridDim.x < n_tiles) mbar_arrive_expect_tx(smem_u32(&rfull[0]), tile_bytes);
            __syncwarp();
            // buffer b of this CTA has been read: every sender in the cluster may refill it
            if (lane < split) mbar_arrive_cluster(mapa(smem_u32(&rfree[b * SH_MAX_SPLIT + slice]), (uint32_t)lane));
        }
    } else {
        // ------------------------------------------------ compute warps
        // this warp's 16 rows go to one combining CTA, or to two when a CTA combines 8 rows
        const int chunk = rows_per < 16 ? rows_per : 16;   // rows per destination
        const int nd = 16 / chunk;                         // 1 or 2
        const int d0 = warp * 16 / rows_per;               // the CTA that combines the first of them
        const int lrow0 = warp * 16 - d0 * rows_per;       // their first row inside d0's share
        const uint32_t stg = smem_u32(staging + warp * 16 * R);  // this warp's 16 rows, as d holds them
        bool pending = false;  // lane 0 issued a copy whose source may still be read
        const int g = lane >> 2, q = lane & 3;
        uint32_t it = 0;
        int j = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
            float acc[R / 8][4];
#pragma unroll
            for (int nt = 0; nt < R / 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
            bool ok = true;
            for (int c = 0; c < nchunks; ++c, ++it) {
                const int st = (int)(it % L::STAGES);
                const uint32_t round = it / L::STAGES;
                // ldmatrix / mma.sync are warp-collective: the whole warp leaves together on a timeout
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), round & 1u, abort));
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
                        uint32_t bf[2];
                        const int krow = kk * 16 + (lane & 15);
                        ldmatrix_x2_trans(swz(as + krow * (2 * R) + nt * 16, L::A_MASK), bf);
                        mma_m16n8k16_bf16(acc[nt], a, bf);
                    }
                }
                release_stage(smem_u32(&empty[st]), lane);
            }
            if (!ok) break;
            const int b = j % L::NB;
            const uint32_t par = (uint32_t)(j / L::NB) & 1u;
            // every destination has read what this warp pushed into its buffer b for tile j - NB
            for (int k = 0; ok && k < nd; ++k)
                ok = __all_sync(0xffffffffu, mbar_wait_cluster(smem_u32(&rfree[b * SH_MAX_SPLIT + d0 + k]), par ^ 1u,
                                                                abort));
            if (!ok) {
                if (lane == 0) atomicOr(err, bi::DEVERR_WAIT_CLUSTER);
                *abort = 1;
                break;
            }
            // stage rows g and g + 8 of this warp's 16, then one bulk copy puts the block at rows
            // lrow0 .. lrow0 + 15 of this slice in d's buffer b, completing on d's receive barrier
            if (lane == 0 && pending) bulk_wait_read();  // the previous tile's copy has read the staging
            __syncwarp();
#pragma unroll
            for (int nt = 0; nt < R / 8; ++nt) {
                const uint32_t col = (uint32_t)(nt * 8 + q * 2) * 4u;
                asm volatile("st.shared.v2.f32 [%0], {%1, %2};" :: "r"(stg + (uint32_t)(g * R * 4) + col),
                             "f"(acc[nt][0]), "f"(acc[nt][1]) : "memory");
                asm volatile("st.shared.v2.f32 [%0], {%1, %2};" :: "r"(stg + (uint32_t)((g + 8) * R * 4) + col),
                             "f"(acc[nt][2]), "f"(acc[nt][3]) : "memory");
            }
            fence_proxy_async_shared();  // the copy engine reads what these generic stores wrote
            __syncwarp();
            if (lane == 0) {
                for (int k = 0; k < nd; ++k) {
                    const uint32_t d = (uint32_t)(d0 + k);
                    const uint32_t dst = mapa(smem_u32(recv), d) +
                                         (uint32_t)((b * SO_TM * R + ((int)slice * rows_per + lrow0) * R) * 4);
                    bulk_copy_to_peer(dst, stg + (uint32_t)(k * chunk * R * 4), (uint32_t)(chunk * R * 4),
                                      mapa(smem_u32(rfull), d) + (uint32_t)b * 8u);
                }
                bulk_commit();
                pending = true;
            }
        }
    }
    // no CTA leaves while a peer may still store into its shared memory or signal its barriers:
    // every bulk copy of this CTA has landed before it joins the final cluster barrier (on an
    // error path a receiver may have stopped waiting for them)
    if (warp < SO_CWARPS && lane == 0) bulk_wait_all();
    __syncwarp();
    cluster_sync();
}

// ------------------------------------------------------------------ shrink on tcgen05
// The plan's kernel at r = 64, and bi_ctrl_lora_shrink_tc at r = 16 and 32.  At r = 64 the
// mma.sync kernel feeds its warp-level MMAs from shared memory: every warp reloads the whole A
// chunk for its 16 rows.  Here one thread issues tcgen05.mma (M = 128 rows of x, N = r, K = 16)
// straight from the TMA-written tiles into TMEM, and four warps read the partials back.  Each
// warp stages a slice of its 32 rows in shared memory as the combining CTA's buffer holds them
// and sends each CTA's block with one bulk copy (shared::cta to shared::cluster, completing on
// that CTA's barrier); the same four warps then combine a quarter of their CTA's rows each.
//
// A kernel that allocates TMEM gets one CTA per SM from the cluster scheduler, and clusters of 8
// then fit only 15 at a time (120 SMs).  So a cluster holds C CTAs, C = split or split / 2, and
// each CTA computes SPC = split / C slices of K: slice s = SPC * rank + l.  Every slice keeps its
// own TMEM accumulator and its own chain over its 512 (K / split) columns in 16-deep ascending
// steps from zero, exactly as if one CTA computed it, and the combine is the same ((P0 + P1) +
// ...) + P(split-1), so both shapes give the same bits.  The host takes C = split while the
// tiles fit the GPU's clusters of that size at once, and C = split / 2 beyond, where the bigger
// clusters would need a second round.  With one CTA per SM the ring gets about 140 KB.
// The tensor core's accumulation is not the warp-level MMA's, so r = 64 results differ from the
// mma.sync kernel's in the last bits; both are batch-invariant, and parity holds against the
// oracle.
constexpr int ST_THREADS = 6 * 32;  // producer, MMA issuer, four TMEM readers that also combine
constexpr int ST_MAX_CLUSTER = SH_MAX_SPLIT;
constexpr int ST_MAX_SPC = 2;  // slices per CTA

template <int R>
struct TcLayout {
    static_assert(R == 16 || R == 32 || R == 64, "the tcgen05 shrink takes r = 16, 32 or 64 (N = r)");
    // The A chunk is the MMA's N-major B operand: rows of 2r bytes (r contiguous), swizzled by the
    // TMA unit at that width (32, 64 or 128 bytes); UMMA layout codes 6, 4, 2; the stride between
    // 8-row groups of K is 8 rows.
    static constexpr uint32_t B_ROW = 2 * R;
    static constexpr uint32_t B_LAYOUT = R == 64 ? 2u : (R == 32 ? 4u : 6u);
    static constexpr uint32_t B_SBO = 8 * B_ROW;
    static constexpr int X_STAGE = SH_TM * SH_KC * 2;  // 16 KB
    static constexpr int A_STAGE = SH_KC * R * 2;      // 8 KB: one [64 K x 64 r] box
    static constexpr int STAGE = X_STAGE + A_STAGE;
    // one receive buffer: [split slices][128 / C rows this CTA combines][R] fp32, at most 64 KB
    // (split / C <= ST_MAX_SPC)
    static constexpr int RECV = ST_MAX_SPC * SH_TM * R * 4;
    // each reader warp stages one slice of its 32 rows here before a bulk copy sends it
    static constexpr int STAGING = 4 * 32 * R * 4;
    static constexpr int BUDGET = 224 * 1024;  // one CTA per SM
    static constexpr int STAGES_FIT = (BUDGET - 1024 - 512 - RECV - STAGING) / STAGE;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static_assert(STAGES >= 4, "the ring needs at least four stages");
    static constexpr int RECV_OFF = STAGES * STAGE;
    static constexpr int STAGING_OFF = RECV_OFF + RECV;
    static constexpr int BAR_OFF = STAGING_OFF + STAGING;
    // full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, rfull, cdone, rfree[ST_MAX_CLUSTER],
    // then the TMEM address and the abort flag
    static constexpr int NBARS = 2 * STAGES + 5 + 2 + ST_MAX_CLUSTER;
    static constexpr size_t BYTES = 1024 + (size_t)BAR_OFF + NBARS * 8 + 16;
    // two accumulator sets (double-buffered across tiles) of ST_MAX_SPC slices
    static constexpr uint32_t TMEM_COLS = 2 * ST_MAX_SPC * R;
};

template <int R>
__global__ void __launch_bounds__(ST_THREADS, 1)
lora_shrink_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                      float* __restrict__ t, int M, int KS, int split, int C, int n_tiles, uint32_t* err) {
    using L = TcLayout<R>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* recv = reinterpret_cast<float*>(base + L::RECV_OFF);
    float* staging = reinterpret_cast<float*>(base + L::STAGING_OFF);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L::BAR_OFF);
    uint64_t* empty = full + L::STAGES;
    uint64_t* tfull = empty + L::STAGES;  // [2]
    uint64_t* tempty = tfull + 2;         // [2]
    uint64_t* drain = tempty + 2;
    uint64_t* rfull = drain + 1;          // every slice of every row this CTA combines has landed
    uint64_t* cdone = rfull + 1;          // the four combining warps have read the receive buffer
    uint64_t* rfree = cdone + 1;          // [ST_MAX_CLUSTER]: CTA d's receive buffer may be written again
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rfree + ST_MAX_CLUSTER);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int rank = (int)cluster_ctarank();
    const int spc = split / C;  // slices per CTA (C: CTAs of the cluster)
    const int nchunks = KS / SH_KC;
    const int rows_per = SH_TM / C;  // rows of a tile that each CTA combines

    if (tid == 0) {
        for (int i = 0; i < L::STAGES; ++i) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tfull[b]), 1);
            mbar_init(smem_u32(&tempty[b]), 4);
        }
        mbar_init(smem_u32(drain), 1);
        mbar_init(smem_u32(rfull), 1);  // per tile: this CTA's expected bytes, then the peers' copies
        mbar_init(smem_u32(cdone), 4);
        for (int d = 0; d < ST_MAX_CLUSTER; ++d) mbar_init(smem_u32(&rfree[d]), 1);
        *abort = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // every CTA's barriers exist before any signal crosses the cluster
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // x and A may come from the kernel before this one; it may still read t
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------ producer: one ring across all tiles and slices
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmA);
            uint32_t it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < n_tiles && !stop; tile += gridDim.x) {
                for (int l = 0; l < spc && !stop; ++l) {
                    const int kbase = (spc * rank + l) * KS;
                    for (int c = 0; c < nchunks; ++c, ++it) {
                        const int st = (int)(it % L::STAGES);
                        const uint32_t round = it / L::STAGES;
                        if (*abort || !mbar_wait(smem_u32(&empty[st]), (round & 1u) ^ 1u, abort)) {
                            if (!*abort) atomicOr(err, bi::DEVERR_WAIT_TMA);
                            *abort = 1;
                            stop = true;
                            break;
                        }
                        uint8_t* sx = base + st * L::STAGE;
                        const uint32_t fb = smem_u32(&full[st]);
                        mbar_arrive_expect_tx(fb, L::STAGE);
                        tma_load_2d(smem_u32(sx), &tmX, kbase + c * SH_KC, tile * SH_TM, fb);
                        tma_load_2d(smem_u32(sx + L::X_STAGE), &tmA, 0, kbase + c * SH_KC, fb);
                    }
                }
            }
            if (*abort) {  // let loads already in flight land before the shared memory is released
                for (uint32_t i = it > (uint32_t)L::STAGES ? it - L::STAGES : 0u; i < it; ++i)
                    (void)mbar_wait(smem_u32(&full[i % L::STAGES]), (i / L::STAGES) & 1u, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc_bf16_f32(SH_TM, R, 0, 1);
            uint32_t it = 0, local = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < n_tiles && !stop && !*abort; tile += gridDim.x, ++local) {
                const uint32_t acc = local & 1u, use = local >> 1;
                if (!mbar_wait(smem_u32(&tempty[acc]), (use & 1u) ^ 1u, abort)) {
                    atomicOr(err, bi::DEVERR_WAIT_ACCUM);
                    *abort = 1;
                    break;
                }
                tc_fence_after();
                for (int l = 0; l < spc && !stop; ++l) {
                    // slice spc * rank + l: its own accumulator, its own chain from zero
                    const uint32_t d_tmem = tmem_base + (acc * ST_MAX_SPC + (uint32_t)l) * R;
                    for (int c = 0; c < nchunks; ++c, ++it) {
                        const int st = (int)(it % L::STAGES);
                        if (!mbar_wait(smem_u32(&full[st]), (it / L::STAGES) & 1u, abort)) {
                            atomicOr(err, bi::DEVERR_WAIT_FULL);
                            *abort = 1;
                            stop = true;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t xs = smem_u32(base + st * L::STAGE);
                        const uint32_t as = xs + L::X_STAGE;
#pragma unroll
                        for (int k = 0; k < SH_KC / 16; ++k) {
                            // x: K-major, 128-byte swizzle, 32 bytes per 16-deep step along the row
                            const uint64_t adesc = make_smem_desc(xs + k * 32, 16, 1024, 2);
                            // A chunk: N-major (r contiguous), swizzled at its row width, 16 K-rows per step
                            const uint64_t bdesc = make_smem_desc(as + k * 16 * L::B_ROW, 8192, L::B_SBO, L::B_LAYOUT);
                            mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (c | k) != 0 ? 1u : 0u);
                        }
                        mma_commit(smem_u32(&empty[st]));  // the stage is free once these MMAs have read it
                    }
                }
                if (!stop) mma_commit(smem_u32(&tfull[acc]));  // this CTA's slices of the tile are complete
            }
            mma_commit(smem_u32(drain));  // TMEM is released only after every MMA completed
            (void)mbar_wait(smem_u32(drain), 0u, nullptr);
        }
    } else {
        // ------------------------------------------------ TMEM readers, then combiners
        const int quarter = warp & 3;          // this warp may read TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;   // row of the tile
        const int d = row / rows_per;          // the CTA that combines it
        const int lrow = row - d * rows_per;   // its row in d's share
        // The lanes whose rows go to one CTA form one contiguous block of its receive buffer: the
        // whole warp when a CTA combines 32 rows or more, else runs of rows_per lanes.
        const int run = rows_per < 32 ? rows_per : 32;
        const bool issuer = (lane % run) == 0;
        const uint32_t stg_row = smem_u32(staging + (quarter * 32 + lane) * R);
        const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
        const uint32_t tile_bytes = (uint32_t)(split * rows_per * R * 4);  // every slice of this CTA's rows
        const int crow0 = quarter * (rows_per / 4);  // this warp's quarter of this CTA's rows
        const int citems = (rows_per / 4) * R / 4;   // its float4 pieces
        bool pending = false;  // this lane issued bulk copies whose source may still be read
        if (quarter == 0 && lane == 0 && (int)blockIdx.x < n_tiles)
            mbar_arrive_expect_tx(smem_u32(rfull), tile_bytes);
        uint32_t local = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++local) {
            const uint32_t acc = local & 1u, use = local >> 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&tfull[acc]), use & 1u, abort));
            if (!ok || *abort) {
                if (lane == 0 && !ok) atomicOr(err, bi::DEVERR_WAIT_ACCUM);
                *abort = 1;
                break;
            }
            // d has taken what this lane sent for the previous tile out of its buffer
            const bool freed = __all_sync(0xffffffffu, mbar_wait_cluster(smem_u32(&rfree[d]), (local & 1u) ^ 1u, abort));
            if (!freed) {
                if (lane == 0) atomicOr(err, bi::DEVERR_WAIT_CLUSTER);
                *abort = 1;
                break;
            }
            tc_fence_after();
            for (int l = 0; l < spc; ++l) {
                uint32_t v[R];
                {
                    const uint32_t col0 = lane_addr + (acc * ST_MAX_SPC + (uint32_t)l) * R;
                    if constexpr (R == 16) {
                        uint32_t (&v16)[16] = *reinterpret_cast<uint32_t(*)[16]>(&v[0]);
                        tmem_ld16(col0, v16);
                    } else {
#pragma unroll
                        for (int h = 0; h < R / 32; ++h)
                            tmem_ld_32x32b_x32(col0 + 32 * h, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * h]));
                    }
                }
                tmem_wait_ld();
                // the staging rows may still be the source of this warp's previous copies
                if (pending && issuer) bulk_wait_read();
                __syncwarp();
                // row lrow of slice s as d's buffer holds it: 16-byte pieces rotated by the row
#pragma unroll
                for (int i = 0; i < R; i += 4)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                 :: "r"(stg_row + (uint32_t)(((i / 4 + lrow) & (R / 4 - 1)) * 16)),
                                    "r"(v[i]), "r"(v[i + 1]), "r"(v[i + 2]), "r"(v[i + 3])
                                 : "memory");
                fence_proxy_async_shared();  // the copy engine reads what these generic stores wrote
                __syncwarp();
                if (issuer) {
                    const int s = spc * rank + l;
                    const uint32_t dst = mapa(smem_u32(recv) + (uint32_t)((s * rows_per + lrow) * R * 4), (uint32_t)d);
                    bulk_copy_to_peer(dst, stg_row, (uint32_t)(run * R * 4), mapa(smem_u32(rfull), (uint32_t)d));
                    bulk_commit();
                    pending = true;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));  // the accumulators may be reused
            // every slice of this CTA's rows has landed: combine this warp's quarter of them
            const bool landed = __all_sync(0xffffffffu, mbar_wait(smem_u32(rfull), local & 1u, abort));
            if (!landed) {
                if (lane == 0) atomicOr(err, bi::DEVERR_WAIT_CLUSTER);
                *abort = 1;
                break;
            }
            const int row0 = tile * SH_TM + rank * rows_per;
            for (int i = lane; i < citems; i += 32) {
                const int rr = crow0 + (4 * i) / R, col = (4 * i) % R;
                const int piece = (((col >> 2) + rr) & (R / 4 - 1)) * 4;  // where the copy put it
                float4 v = *reinterpret_cast<const float4*>(recv + rr * R + piece);
                for (int sl = 1; sl < split; ++sl) {  // ((P0 + P1) + P2) + ...: slice order
                    const float4 p = *reinterpret_cast<const float4*>(recv + (sl * rows_per + rr) * R + piece);
                    v.x = __fadd_rn(v.x, p.x);
                    v.y = __fadd_rn(v.y, p.y);
                    v.z = __fadd_rn(v.z, p.z);
                    v.w = __fadd_rn(v.w, p.w);
                }
                if (row0 + rr < M) *reinterpret_cast<float4*>(t + (size_t)(row0 + rr) * R + col) = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(cdone));
            if (quarter == 0) {
                // all four warps have read this CTA's buffer: post the next tile's bytes, then let
                // every sender refill it
                const bool read = __all_sync(0xffffffffu, mbar_wait(smem_u32(cdone), local & 1u, abort));
                if (!read) {
                    if (lane == 0) atomicOr(err, bi::DEVERR_WAIT_CLUSTER);
                    *abort = 1;
                    break;
                }
                if (lane == 0 && tile + (int)gridDim.x < n_tiles) mbar_arrive_expect_tx(smem_u32(rfull), tile_bytes);
                __syncwarp();
                if (lane < C) mbar_arrive_cluster(mapa(smem_u32(&rfree[rank]), (uint32_t)lane));
            }
        }
        // the copies have landed (destination writes included) before this CTA joins the final
        // cluster barrier, after which a receiver may leave
        if (pending) bulk_wait_all();
    }
    // no CTA leaves, or frees TMEM, while a peer may still store into it or signal it
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ expand
// A CTA owns a 64 x 128 tile of y; warp (wr, wc) owns rows [16 wr, 16 wr + 16) and columns
// [64 wc, 64 wc + 64) of it.  The B tile is staged with its columns permuted inside each group
// of 32, so that the mma.sync accumulator of lane (g, q) holds, for rows g and g + 8, the 8
// CONSECUTIVE output columns [8q, 8q + 8) of every group: the product goes straight from the
// accumulator registers to y in 16-byte pieces, with no trip through shared memory.  Column
// L = 8p + 2q + e of a group in shared memory (p, e: the MMA's n-tile and pair element) holds
// the weights of output column 8q + 2p + e.  Each output element is still one MMA chain over
// r, so the permutation moves work between lanes and changes no arithmetic.
constexpr int EX_TM = 64;
constexpr int EX_TN = 128;
constexpr int EX_THREADS = 256;

template <int R>
struct ExpandLayout {
    static constexpr int RP = R < 16 ? 16 : R;       // K of the MMA, padded with zeros
    static constexpr int T_PITCH = RP * 2 + 16;       // bytes per row of bf16(t); +16 avoids bank conflicts
    static constexpr int B_PITCH = EX_TN * 2 + 16;    // bytes per K-row of the permuted B tile
    static constexpr int T_BYTES = EX_TM * T_PITCH;
    static constexpr int B_BYTES = RP * B_PITCH;
    static constexpr size_t BYTES = (size_t)T_BYTES + B_BYTES;
};

template <int R, bool YBF16>
__global__ void __launch_bounds__(EX_THREADS)
lora_expand_kernel(const float* __restrict__ t, const __nv_bfloat16* __restrict__ B, void* __restrict__ y, int M,
                   int N, int64_t ldy, float scale) {
    using L = ExpandLayout<R>;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* sT = smem;
    uint8_t* sB = smem + L::T_BYTES;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int wr = warp >> 1, wc = warp & 1;
    const int g = lane >> 2, q = lane & 3;
    const int m0 = blockIdx.y * EX_TM;
    const int n0 = blockIdx.x * EX_TN;

    pdl_wait();  // t and y may come from the kernels just before this one

    // 0. This lane's pieces of y: rows g and g + 8 of the warp's strip, columns [8q, 8q + 8) of
    //    each of the warp's two 32-column groups.  Issued first: their HBM latency overlaps 1-3.
    //    A piece is 8 elements: one 16-byte load in bf16, two in fp32.
    constexpr int W = YBF16 ? 1 : 2;  // 16-byte words per piece
    uint4 yv[2][2][W];                // [row half][group][word]
    bool live[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int G = 0; G < 2; ++G) {
            const int row = m0 + wr * 16 + g + 8 * h;
            const int col = n0 + wc * 64 + G * 32 + 8 * q;
            live[h][G] = row < M && col < N;  // N % 8 == 0: a piece is wholly inside or outside
#pragma unroll
            for (int w = 0; w < W; ++w) yv[h][G][w] = make_uint4(0u, 0u, 0u, 0u);
            if (live[h][G]) {
                if constexpr (YBF16) {
                    yv[h][G][0] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(y) +
                                                                  (size_t)row * ldy + col);
                } else {
                    const float* p = static_cast<const float*>(y) + (size_t)row * ldy + col;
                    yv[h][G][0] = *reinterpret_cast<const uint4*>(p);
                    yv[h][G][1] = *reinterpret_cast<const uint4*>(p + 4);
                }
            }
        }
    }

    // 1-2. Every global load of t and of the B tile is issued before the first shared-memory store,
    //      so that their L2 latencies overlap instead of adding up.
    constexpr int T_ITERS = EX_TM * L::RP / 4 / EX_THREADS;   // float4 pieces of t per thread
    constexpr int B_ITERS = L::RP * (EX_TN / 8) / EX_THREADS;  // 8-column pieces of B per thread
    static_assert(T_ITERS * EX_THREADS * 4 == EX_TM * L::RP && B_ITERS * EX_THREADS * 8 == L::RP * EX_TN,
                  "the staging loops cover their tiles exactly");
    float4 tv[T_ITERS];
    uint4 bv[B_ITERS];
#pragma unroll
    for (int j = 0; j < T_ITERS; ++j) {
        const int i = tid + j * EX_THREADS;
        const int row = (4 * i) / L::RP, k = (4 * i) % L::RP;
        tv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (m0 + row < M && k < R) tv[j] = *reinterpret_cast<const float4*>(t + (size_t)(m0 + row) * R + k);
    }
#pragma unroll
    for (int j = 0; j < B_ITERS; ++j) {
        const int i = tid + j * EX_THREADS;
        const int k = i / (EX_TN / 8), c = i % (EX_TN / 8);
        const int col = n0 + c * 8;
        bv[j] = make_uint4(0u, 0u, 0u, 0u);
        if (k < R && col < N) bv[j] = bi::ld_cached_v4(B + (size_t)k * N + col);
    }
    // 1. bf16(t) rows into shared memory (rows past M and columns past R are zero).
#pragma unroll
    for (int j = 0; j < T_ITERS; ++j) {
        const int i = tid + j * EX_THREADS;
        const int row = (4 * i) / L::RP, k = (4 * i) % L::RP;
        const uint2 p = make_uint2(bi::pack_bf16x2(tv[j].x, tv[j].y), bi::pack_bf16x2(tv[j].z, tv[j].w));
        *reinterpret_cast<uint2*>(sT + row * L::T_PITCH + k * 2) = p;
    }
    // 2. The B tile [R, 128], permuted: the 8 weights of output columns [8c, 8c + 8) (c = 4 gg + qq)
    //    go, two at a time, to shared-memory columns 32 gg + 8 p + 2 qq, p = 0..3.  Columns past N
    //    and rows past R are zero.
#pragma unroll
    for (int j = 0; j < B_ITERS; ++j) {
        const int i = tid + j * EX_THREADS;
        const int k = i / (EX_TN / 8), c = i % (EX_TN / 8);
        uint32_t* dst = reinterpret_cast<uint32_t*>(sB + k * L::B_PITCH) + 16 * (c >> 2) + (c & 3);
        dst[0] = bv[j].x;
        dst[4] = bv[j].y;
        dst[8] = bv[j].z;
        dst[12] = bv[j].w;
    }
    __syncthreads();
    pdl_trigger();

    // 3. delta[16 rows x 64 cols] per warp with mma.sync (shared-memory column order).
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

    // 4. y = round(fma(scale, delta, y)).  In group G, n-tile p = 0..3 of the accumulator holds
    //    output columns 8q + 2p + {0, 1} of row g (elements 0, 1) and row g + 8 (elements 2, 3).
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = m0 + wr * 16 + g + 8 * h;
#pragma unroll
        for (int G = 0; G < 2; ++G) {
            if (!live[h][G]) continue;
            const int col = n0 + wc * 64 + G * 32 + 8 * q;
            float d[8];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                d[2 * p] = acc[G * 4 + p][2 * h];
                d[2 * p + 1] = acc[G * 4 + p][2 * h + 1];
            }
            if constexpr (YBF16) {
                const uint4 u = yv[h][G][0];
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    o[j] = bi::pack_bf16x2(__fmaf_rn(scale, d[2 * j], bi::bf16_lo(w4[j])),
                                           __fmaf_rn(scale, d[2 * j + 1], bi::bf16_hi(w4[j])));
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + (size_t)row * ldy + col) =
                    make_uint4(o[0], o[1], o[2], o[3]);
            } else {
                float* p = static_cast<float*>(y) + (size_t)row * ldy + col;
                const uint4 u0 = yv[h][G][0], u1 = yv[h][G][1];
                *reinterpret_cast<float4*>(p) = make_float4(
                    __fmaf_rn(scale, d[0], __uint_as_float(u0.x)), __fmaf_rn(scale, d[1], __uint_as_float(u0.y)),
                    __fmaf_rn(scale, d[2], __uint_as_float(u0.z)), __fmaf_rn(scale, d[3], __uint_as_float(u0.w)));
                *reinterpret_cast<float4*>(p + 4) = make_float4(
                    __fmaf_rn(scale, d[4], __uint_as_float(u1.x)), __fmaf_rn(scale, d[5], __uint_as_float(u1.y)),
                    __fmaf_rn(scale, d[6], __uint_as_float(u1.z)), __fmaf_rn(scale, d[7], __uint_as_float(u1.w)));
            }
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

template <int R>
int launch_shrink_atomic(const void* x, const void* A, float* t, int64_t M, int64_t K, int split, cudaStream_t s) {
    using L = ShrinkLayout<R>;
    uint32_t* err = bi::device_error_word();
    auto kern = lora_shrink_atomic_kernel<R>;
    if (!err || !set_smem_once(kern, L::BYTES)) return BI_ERR_CUDA;
    CUtensorMap tmX, tmA;
    if (!bi::make_tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2,
                          SH_KC, SH_TM, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    if (!bi::make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)R, (uint64_t)K, (uint64_t)R * 2, R,
                          SH_KC, bi::swizzle_for(R * 2)))
        return BI_ERR_CUDA;
    dim3 grid((unsigned)((M + SH_TM - 1) / SH_TM), (unsigned)split, 1);
    kern<<<grid, SH_THREADS, L::BYTES, s>>>(tmX, tmA, t, (int)M, (int)(K / split), err);
    return bi::launch_status();
}

// Clusters of the ordered kernel that fit on the device at once, per (R, split); queried once per
// device.  The grid never exceeds it, so every cluster is resident and walks its tiles; a larger
// grid would only queue clusters behind the first wave.
template <int R>
int ordered_clusters(int split) {
    static std::mutex mu;
    static int cached[64][4];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    const int si = split == 1 ? 0 : (split == 2 ? 1 : (split == 4 ? 2 : 3));
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev][si] == 0) {
        using L = OrderedLayout<R>;
        int n = 0;
        if (split == 1) {
            int per_sm = 0, sms = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, lora_shrink_ordered_kernel<R>, OrderedShape<R>::THREADS,
                                                              L::BYTES) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return -1;
            n = per_sm * sms;
        } else {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(1, (unsigned)split, 1);
            cfg.blockDim = dim3(OrderedShape<R>::THREADS, 1, 1);
            cfg.dynamicSmemBytes = L::BYTES;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 1;
            attr[0].val.clusterDim.y = (unsigned)split;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, lora_shrink_ordered_kernel<R>, &cfg) != cudaSuccess) return -1;
        }
        cached[dev][si] = n > 0 ? n : 1;
    }
    return cached[dev][si];
}

template <int R>
int launch_shrink_ordered(const void* x, const void* A, float* t, int64_t M, int64_t K, int split, cudaStream_t s) {
    using L = OrderedLayout<R>;
    uint32_t* err = bi::device_error_word();
    auto kern = lora_shrink_ordered_kernel<R>;
    if (!err || !set_smem_once(kern, L::BYTES)) return BI_ERR_CUDA;
    const int fit = ordered_clusters<R>(split);
    if (fit <= 0) return BI_ERR_CUDA;
    CUtensorMap tmX, tmA;
    if (!bi::make_tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2,
                          SH_KC, OrderedShape<R>::TM, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    if (!bi::make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)R, (uint64_t)K, (uint64_t)R * 2, R,
                          SH_KC, bi::swizzle_for(R * 2)))
        return BI_ERR_CUDA;
    const int n_tiles = (int)((M + OrderedShape<R>::TM - 1) / OrderedShape<R>::TM);
    const int clusters = n_tiles < fit ? n_tiles : fit;
    if (bi::launch_pdl(kern, dim3((unsigned)clusters, (unsigned)split), dim3(OrderedShape<R>::THREADS), L::BYTES, s,
                       (unsigned)split, tmX, tmA, t, (int)M, (int)(K / split), (int)split, n_tiles,
                       err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

template <int R>
int launch_shrink_tc(const void* x, const void* A, float* t, int64_t M, int64_t K, int split, cudaStream_t s) {
    using L = TcLayout<R>;
    uint32_t* err = bi::device_error_word();
    auto kern = lora_shrink_tc_kernel<R>;
    if (!err || !set_smem_once(kern, L::BYTES)) return BI_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BI_ERR_CUDA;
    // clusters of c CTAs that fit at once (cached per device and cluster size 1, 2, 4, 8)
    static std::mutex mu;
    static int fit_cache[64][4];
    auto fit = [&](int c) -> int {
        const int ci = c == 1 ? 0 : (c == 2 ? 1 : (c == 4 ? 2 : 3));
        std::lock_guard<std::mutex> lock(mu);
        if (fit_cache[dev][ci] == 0) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(1, (unsigned)c, 1);
            cfg.blockDim = dim3(ST_THREADS, 1, 1);
            cfg.dynamicSmemBytes = L::BYTES;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 1;
            attr[0].val.clusterDim.y = (unsigned)c;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
                (void)cudaGetLastError();
                return -1;
            }
            fit_cache[dev][ci] = n > 0 ? n : 1;
        }
        return fit_cache[dev][ci];
    };
    const int n_tiles = (int)((M + SH_TM - 1) / SH_TM);
    // one slice per CTA while the tiles fit in one round of such clusters, else two
    int C = split;
    int fc = fit(C);
    if (fc < 0) return BI_ERR_CUDA;
    if (split >= 2 && n_tiles > fc) {
        C = split / 2;
        fc = fit(C);
        if (fc < 0) return BI_ERR_CUDA;
    }
    CUtensorMap tmX, tmA;
    if (!bi::make_tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2,
                          SH_KC, SH_TM, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    if (!bi::make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)R, (uint64_t)K, (uint64_t)R * 2, R,
                          SH_KC, bi::swizzle_for((uint32_t)R * 2)))
        return BI_ERR_CUDA;
    const int clusters = n_tiles < fc ? n_tiles : fc;
    if (bi::launch_pdl(kern, dim3((unsigned)clusters, (unsigned)C), dim3(ST_THREADS), L::BYTES, s, (unsigned)C, tmX,
                       tmA, t, (int)M, (int)(K / split), (int)split, C, n_tiles, err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

template <bool ATOMIC>
int shrink_dispatch(const void* x, const void* A, float* t, int64_t M, int64_t K, int32_t r, int32_t split,
                    cudaStream_t s) {
    if constexpr (!ATOMIC) {
        switch (r) {
            case 8: return launch_shrink_ordered<8>(x, A, t, M, K, split, s);
            case 16: return launch_shrink_ordered<16>(x, A, t, M, K, split, s);
            case 32: return launch_shrink_ordered<32>(x, A, t, M, K, split, s);
            // r = 64 on tcgen05: the warp-level MMAs reload the A chunk per warp, and the tensor
            // core does not (20-45 % faster at every batch size measured)
            case 64: return launch_shrink_tc<64>(x, A, t, M, K, split, s);
            default: return BI_ERR_UNSUPPORTED_SHAPE;
        }
    } else {
        switch (r) {
            case 8: return launch_shrink_atomic<8>(x, A, t, M, K, split, s);
            case 16: return launch_shrink_atomic<16>(x, A, t, M, K, split, s);
            case 32: return launch_shrink_atomic<32>(x, A, t, M, K, split, s);
            case 64: return launch_shrink_atomic<64>(x, A, t, M, K, split, s);
            default: return BI_ERR_UNSUPPORTED_SHAPE;
        }
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
    auto k = ybf16 ? lora_expand_kernel<R, true> : lora_expand_kernel<R, false>;
    if (!set_smem_once(k, L::BYTES)) return BI_ERR_CUDA;
    if (bi::launch_pdl(k, grid, dim3(EX_THREADS), L::BYTES, s, 0u, t, static_cast<const __nv_bfloat16*>(B), y,
                       (int)M, (int)N, ldy, scale) != cudaSuccess)
        return BI_ERR_CUDA;
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

BI_API int bi_ctrl_lora_shrink_tc(const void* x, const void* A, float* t, int64_t M, int64_t K, int32_t r,
                                  int32_t split_k, void* stream) {
    const int c = shrink_checks(x, A, t, M, K, r, split_k);
    if (c < 0) return BI_OK;
    if (c != BI_OK) return c;
    cudaStream_t s = bi::as_stream(stream);
    switch (r) {
        case 16: return launch_shrink_tc<16>(x, A, t, M, K, split_k, s);
        case 32: return launch_shrink_tc<32>(x, A, t, M, K, split_k, s);
        case 64: return launch_shrink_tc<64>(x, A, t, M, K, split_k, s);
        default: return BI_ERR_UNSUPPORTED_SHAPE;
    }
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
