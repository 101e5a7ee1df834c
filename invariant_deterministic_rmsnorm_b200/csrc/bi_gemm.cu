// bi_gemm.cu -- batch-invariant dense GEMM on tcgen05 tensor cores (sm_100a).
//
// C[M, N] = A[M, K] . W[K, N], bf16 operands, fp32 accumulation in TMEM, fp32 or bf16 output.
//
// Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section
// "Multiplicación de matrices".  The matmul is tile-parallel over 2-D output tiles.
// Small batches tempt implementations into split-K, and a split chosen by batch size
// breaks batch invariance.  The fix the section gives is to force one kernel
// configuration for every batch size.  Here the configuration is fixed by (N, K) and the
// device alone, never by M:
//   - N up to 256 x (SM pairs) (18944 on a B200): 256 x 256 tiles over a 2-CTA cluster,
//     tcgen05.mma.cta_group::2 256 x 256 x 16;
//   - wider N: 128 x 256 tiles on one CTA, tcgen05.mma.cta_group::1 128 x 256 x 16.
// In both, the K-block order is ascending (64 at a time).  The 256 x 256 tiles can also split K
// into S contiguous slices (the cluster-split kernel): slice s of a tile accumulates its K
// blocks in TMEM like an unsplit tile, on its own CTA pair of a 2S-CTA cluster, and the pairs
// add their partials in slice order, ((P0 + P1) + ...) + P(S-1), through distributed shared
// memory before the output rounding; no floating-point atomic is used.  The plan's S comes from
// splits_for(N, K); other S run through bi_ctrl_gemm_split.  A row's tile position and the batch
// size M change which CTA computes the row.  They never change the instructions that produce
// its bits.  Rows past M are zero-filled by the TMA unit and are never stored.
//
// CTA structure (192 threads; in the pair kernel two CTAs per cluster, 2S in the split kernel):
//   warp 0      TMA producer.  Pair kernel: 128 rows of A [128 x 64] and 128 columns of W
//               [64 x 128] per stage, 6-stage ring, completion bytes of both CTAs counted by
//               the leader.  Single-CTA kernel: A [128 x 64] and W [64 x 256], 4-stage ring.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer (the leader's, in the pair
//               kernel): 4 MMAs of K = 16 per stage
//   warps 2..5  epilogue: tcgen05.ld of this CTA's 128 x 256 fp32 accumulator rows, convert,
//               store
// Shared-memory operand layouts are the 128-byte-swizzled canonical forms that the TMA
// unit writes.  A is K-major (one 128-byte row per M row).  W is N-major: boxes of 64
// N-columns x 64 K-rows; the leading-dimension offset is the box stride (8 KB), and the
// stride offset is 8 K-rows (1 KB).
#include <mutex>

#include "bi_common.cuh"
#include "bi_sm100.cuh"
#include "bi_tma_host.cuh"

using namespace bi::sm100;

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int A_STAGE = BM * BK * 2;  // 16 KB
constexpr int B_BOX = 64 * BK * 2;    // 8 KB: 64 N-columns x 64 K-rows
constexpr int THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr int MAX_STAGES = 8;

// Tile geometry for a tile width BN (64, 128 or 256 output columns).
template <int BN>
struct Tile {
    static constexpr int B_STAGE = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
    static constexpr int STAGES = (196 * 1024) / STAGE_BYTES < MAX_STAGES ? (196 * 1024) / STAGE_BYTES : MAX_STAGES;
    static constexpr int ACC_COLS = BN;  // one fp32 accumulator = BN TMEM columns
    static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;  // two accumulators, a power of two
    static constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
};

struct Bars1 {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tfull[2];   // accumulator b holds a finished tile
    uint64_t tempty[2];  // accumulator b has been read out
    uint32_t tmem_addr;
    int abort;
};

__device__ __forceinline__ void fail(uint32_t* err, volatile int* abort, uint32_t bit) {
    atomicOr(err, bit);
    *abort = 1;
}

// Tile order: groups of `gm` row tiles, walked column by column inside a group, so that the
// tiles in flight at any moment share a few W column blocks and a few A row blocks in L2.
// The order decides only which CTA computes a tile, never how.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int gm, int& m_tile, int& n_tile) {
    const int per_group = gm * tiles_n;
    const int group = t / per_group;
    const int first_m = group * gm;
    const int gsm = min(tiles_m - first_m, gm);
    const int r = t - group * per_group;
    m_tile = first_m + r % gsm;
    n_tile = r / gsm;
}

// ------------------------------------------------------------------ the single-CTA kernel
// One CTA computes a 128 x 256 tile with tcgen05.mma.cta_group::1 (4-stage ring of 48 KB).
template <int BN>
__global__ void __launch_bounds__(THREADS, 1)
bi_gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                       void* __restrict__ C, int M, int N, int K, int c_bf16, int gm, uint32_t* err) {
    constexpr int STAGES = Tile<BN>::STAGES;
    constexpr int B_STAGE = Tile<BN>::B_STAGE;
    constexpr int STAGE_BYTES = Tile<BN>::STAGE_BYTES;
    constexpr int ACC_COLS = Tile<BN>::ACC_COLS;
    constexpr int TMEM_COLS = Tile<BN>::TMEM_COLS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE;
    Bars1* bars = reinterpret_cast<Bars1*>(sB + STAGES * B_STAGE);
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles_m = (M + BM - 1) / BM;
    const int tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bars->tfull[b]), 1);
            mbar_init(smem_u32(&bars->tempty[b]), EPI_WARPS);
        }
        bars->abort = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_addr), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_addr;
    // everything above overlaps the previous kernel's tail; A and W may come from it, and it may
    // still read C
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;  // k-blocks issued by this CTA so far (the ring runs across tiles)
            for (int t = blockIdx.x; t < num_tiles && !*abort; t += gridDim.x) {
                int mt, nt;
                tile_coords(t, tiles_m, tiles_n, gm, mt, nt);
                const int m0 = mt * BM, n0 = nt * BN;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t round = it / STAGES;
                    if (!mbar_wait(smem_u32(&bars->empty[s]), (round & 1u) ^ 1u, abort)) {
                        fail(err, abort, bi::DEVERR_WAIT_TMA);
                        break;
                    }
                    const uint32_t fb = smem_u32(&bars->full[s]);
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(smem_u32(sA + s * A_STAGE), &tmA, kb * BK, m0, fb);
#pragma unroll
                    for (int j = 0; j < BN / 64; ++j)
                        tma_load_2d(smem_u32(sB + s * B_STAGE + j * B_BOX), &tmW, n0 + 64 * j, kb * BK, fb);
                }
            }
            if (*abort) {  // let loads already in flight land before the CTA's shared memory is released
                for (uint32_t i = it > (uint32_t)STAGES ? it - STAGES : 0u; i < it; ++i)
                    (void)mbar_wait(smem_u32(&bars->full[i % STAGES]), (i / STAGES) & 1u, nullptr);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc_bf16_f32(BM, BN, 0, 1);
            uint32_t it = 0, local = 0;
            for (int t = blockIdx.x; t < num_tiles && !*abort; t += gridDim.x, ++local) {
                const uint32_t acc = local & 1u, use = local >> 1;
                if (!mbar_wait(smem_u32(&bars->tempty[acc]), (use & 1u) ^ 1u, abort)) {
                    fail(err, abort, bi::DEVERR_WAIT_ACCUM);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t round = it / STAGES;
                    if (!mbar_wait(smem_u32(&bars->full[s]), round & 1u, abort)) {
                        fail(err, abort, bi::DEVERR_WAIT_FULL);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + s * A_STAGE);
                    const uint32_t b_base = smem_u32(sB + s * B_STAGE);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        // A: K-major, 128B swizzle; the k-th 16-element slice starts 32 bytes along the row.
                        const uint64_t adesc = make_smem_desc(a_base + k * UMMA_K * 2, 16, 1024, 2);
                        // W: N-major, 128B swizzle; 16 K-rows of 128 bytes each per step.
                        const uint64_t bdesc = make_smem_desc(b_base + k * UMMA_K * 128, B_BOX, 1024, 2);
                        mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&bars->empty[s]));  // stage free once these MMAs have read it
                }
                mma_commit(smem_u32(&bars->tfull[acc]));  // accumulator complete
            }
        }
    } else {
        const int quarter = warp & 3;  // this warp may read TMEM lanes 32*quarter .. +31
        uint32_t local = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
            const uint32_t acc = local & 1u, use = local >> 1;
            const bool ok = mbar_wait(smem_u32(&bars->tfull[acc]), use & 1u, abort);
            if (!ok) fail(err, abort, bi::DEVERR_WAIT_ACCUM);
            // tcgen05.ld is warp-collective: the whole warp takes the same branch
            if (!__all_sync(0xffffffffu, ok && !*abort)) break;
            tc_fence_after();
            int mt, nt;
            tile_coords(t, tiles_m, tiles_n, gm, mt, nt);
            const int row = mt * BM + quarter * 32 + lane;
            const uint32_t lane_addr = tmem_base + acc * ACC_COLS + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(lane_addr + (uint32_t)c, r);
                tmem_wait_ld();
                if (c == BN - 32) {  // every column of this accumulator is in registers: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&bars->tempty[acc]));
                }
                const int col = nt * BN + c;
                if (row < M && col < N) {
                    if (!c_bf16) {
                        float* dst = static_cast<float*>(C) + (int64_t)row * N + col;
                        if (col + 32 <= N) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                *reinterpret_cast<uint4*>(dst + i) = make_uint4(r[i], r[i + 1], r[i + 2], r[i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < N - col) dst[i] = __uint_as_float(r[i]);
                        }
                    } else {
                        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(C) + (int64_t)row * N + col;
                        uint32_t p[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            p[i] = bi::pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        if (col + 32 <= N) {
#pragma unroll
                            for (int i = 0; i < 16; i += 4)
                                *reinterpret_cast<uint4*>(dst + 2 * i) = make_uint4(p[i], p[i + 1], p[i + 2], p[i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < N - col) dst[i] = __float2bfloat16_rn(__uint_as_float(r[i]));
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}


// ------------------------------------------------------------------ the CTA-pair kernel
// A 2-CTA cluster computes a 256 x 256 output tile with tcgen05.mma.cta_group::2: CTA r of the
// pair loads rows [128r, 128r + 128) of the A tile and columns [128r, 128r + 128) of the W tile,
// and holds rows [128r, 128r + 128) x all 256 columns of the accumulator in its TMEM.  Per SM
// that is 32 KB of operands per 64-deep K block for the same MMA work the single-CTA 128 x 256
// tile gets from 48 KB; an SM can take in about 64 bytes a cycle from L2, and this is what lets
// the tensor pipe stay busy.  Each output element is still one fp32 chain over K in ascending
// 16-deep steps, and the plan depends on (N, K) only.
namespace pair {
constexpr int ROWS = 128;                 // A rows per CTA
constexpr int COLS = 128;                 // W columns per CTA
constexpr int TILE_M = 2 * ROWS;          // 256
constexpr int TILE_N = 2 * COLS;          // 256
constexpr int A_ST = ROWS * BK * 2;       // 16 KB
constexpr int B_ST = COLS * BK * 2;       // 16 KB: two boxes of 64 columns x 64 K-rows
constexpr int ST_BYTES = A_ST + B_ST;     // 32 KB per CTA per stage
constexpr int STAGES = 6;
constexpr uint32_t ACC_COLS = TILE_N;     // one fp32 accumulator: 256 TMEM columns
constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
struct Bars {
    uint64_t full[STAGES];   // leader: both CTAs' bytes of stage s have landed
    uint64_t empty[STAGES];  // each CTA: the MMAs have read its stage s
    uint64_t tfull[2];       // each CTA: accumulator b holds a finished tile
    uint64_t tempty[2];      // leader: both CTAs' epilogues have read accumulator b
    uint64_t drain;          // leader: every MMA issued has completed
    uint32_t tmem_addr;
    int abort;
};
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * ST_BYTES + sizeof(Bars) + 64;
}  // namespace pair

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
bi_gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                         void* __restrict__ C, int M, int N, int K, int c_bf16, int gm, uint32_t* err) {
    using pair::ROWS;
    using pair::COLS;
    using pair::TILE_M;
    using pair::TILE_N;
    using pair::A_ST;
    using pair::B_ST;
    using pair::ST_BYTES;
    using pair::STAGES;
    using pair::ACC_COLS;
    using pair::TMEM_COLS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_ST;
    pair::Bars* bars = reinterpret_cast<pair::Bars*>(sB + STAGES * B_ST);
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: the leader, which issues the MMAs
    const int pair_id = (int)(blockIdx.x >> 1), n_pairs = (int)(gridDim.x >> 1);
    const int tiles_m = (M + TILE_M - 1) / TILE_M;
    const int tiles_n = (N + TILE_N - 1) / TILE_N;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bars->tfull[b]), 1);
            mbar_init(smem_u32(&bars->tempty[b]), 2 * EPI_WARPS);
        }
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmW);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&bars->tmem_addr), TMEM_COLS);
        tmem_relinquish_pair();
    }
    // both CTAs' barriers are initialised and their TMEM allocated before any signal crosses the pair
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_addr;
    // everything above overlaps the previous kernel's tail; A and W may come from it, and it may
    // still read C
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;  // k-blocks issued by this CTA so far (the ring runs across tiles)
            for (int t = pair_id; t < num_tiles && !*abort; t += n_pairs) {
                int mt, nt;
                tile_coords(t, tiles_m, tiles_n, gm, mt, nt);
                const int m0 = mt * TILE_M + (int)rank * ROWS, n0 = nt * TILE_N + (int)rank * COLS;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = (int)(it % STAGES);
                    const uint32_t round = it / STAGES;
                    if (!mbar_wait(smem_u32(&bars->empty[s]), (round & 1u) ^ 1u, abort)) {
                        fail(err, abort, bi::DEVERR_WAIT_TMA);
                        break;
                    }
                    const uint32_t fb = smem_u32(&bars->full[s]);
                    if (rank == 0) mbar_arrive_expect_tx(fb, 2 * ST_BYTES);  // this stage of both CTAs
                    const uint32_t fb_leader = mapa(fb, 0);
                    tma_load_2d_pair(smem_u32(sA + s * A_ST), &tmA, kb * BK, m0, fb_leader);
                    tma_load_2d_pair(smem_u32(sB + s * B_ST), &tmW, n0, kb * BK, fb_leader);
                    tma_load_2d_pair(smem_u32(sB + s * B_ST + B_BOX), &tmW, n0 + 64, kb * BK, fb_leader);
                }
            }
            if (*abort) {
                // let loads already in flight land before the CTA's shared memory is released: the
                // leader tracks both CTAs' bytes; the peer waits a fixed time
                if (rank == 0) {
                    for (uint32_t i = it > (uint32_t)STAGES ? it - STAGES : 0u; i < it; ++i)
                        (void)mbar_wait(smem_u32(&bars->full[i % STAGES]), (i / STAGES) & 1u, nullptr);
                } else {
                    const uint64_t t0 = globaltimer();
                    while (globaltimer() - t0 < 200000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = make_idesc_bf16_f32(TILE_M, TILE_N, 0, 1);
            const uint32_t peer_empty0 = mapa(smem_u32(&bars->empty[0]), 1);
            const uint32_t peer_tfull0 = mapa(smem_u32(&bars->tfull[0]), 1);
            uint32_t it = 0, local = 0;
            for (int t = pair_id; t < num_tiles && !*abort; t += n_pairs, ++local) {
                const uint32_t acc = local & 1u, use = local >> 1;
                if (!mbar_wait(smem_u32(&bars->tempty[acc]), (use & 1u) ^ 1u, abort)) {
                    fail(err, abort, bi::DEVERR_WAIT_ACCUM);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = (int)(it % STAGES);
                    const uint32_t round = it / STAGES;
                    if (!mbar_wait(smem_u32(&bars->full[s]), round & 1u, abort)) {
                        fail(err, abort, bi::DEVERR_WAIT_FULL);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + s * A_ST);
                    const uint32_t b_base = smem_u32(sB + s * B_ST);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        const uint64_t adesc = make_smem_desc(a_base + k * UMMA_K * 2, 16, 1024, 2);
                        const uint64_t bdesc = make_smem_desc(b_base + k * UMMA_K * 128, B_BOX, 1024, 2);
                        mma_bf16_ss_pair(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    // stage s of both CTAs is free once these MMAs have read it
                    mma_commit_pair(smem_u32(&bars->empty[s]));
                    mma_commit_pair(peer_empty0 + (uint32_t)s * 8u);
                }
                mma_commit_pair(smem_u32(&bars->tfull[acc]));  // both CTAs' accumulator rows complete
                mma_commit_pair(peer_tfull0 + acc * 8u);
            }
            mma_commit_pair(smem_u32(&bars->drain));  // TMEM is released only after every MMA completed
            (void)mbar_wait(smem_u32(&bars->drain), 0u, nullptr);
        }
    } else {
        const int quarter = warp & 3;  // this warp may read TMEM lanes 32*quarter .. +31
        const uint32_t tempty0 = rank == 0 ? smem_u32(&bars->tempty[0]) : mapa(smem_u32(&bars->tempty[0]), 0);
        uint32_t local = 0;
        for (int t = pair_id; t < num_tiles; t += n_pairs, ++local) {
            const uint32_t acc = local & 1u, use = local >> 1;
            const bool ok = mbar_wait(smem_u32(&bars->tfull[acc]), use & 1u, abort);
            if (!ok) fail(err, abort, bi::DEVERR_WAIT_ACCUM);
            // tcgen05.ld is warp-collective: the whole warp takes the same branch
            if (!__all_sync(0xffffffffu, ok && !*abort)) break;
            tc_fence_after();
            int mt, nt;
            tile_coords(t, tiles_m, tiles_n, gm, mt, nt);
            const int row = mt * TILE_M + (int)rank * ROWS + quarter * 32 + lane;
            const uint32_t lane_addr = tmem_base + acc * ACC_COLS + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < TILE_N; c += 32) {
                const int col = nt * TILE_N + c;
                uint32_t r[32];
                tmem_ld_32x32b_x32(lane_addr + (uint32_t)c, r);
                tmem_wait_ld();
                if (c == TILE_N - 32) {  // every column of this accumulator is in registers: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(tempty0 + acc * 8u);
                }
                if (row >= M || col >= N) continue;
                if (!c_bf16) {
                    float* dst = static_cast<float*>(C) + (int64_t)row * N + col;
                    if (col + 32 <= N) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<uint4*>(dst + i) = make_uint4(r[i], r[i + 1], r[i + 2], r[i + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < N - col) dst[i] = __uint_as_float(r[i]);
                    }
                } else {
                    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(C) + (int64_t)row * N + col;
                    uint32_t p[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        p[i] = bi::pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                    if (col + 32 <= N) {
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            *reinterpret_cast<uint4*>(dst + 2 * i) = make_uint4(p[i], p[i + 1], p[i + 2], p[i + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < N - col) dst[i] = __float2bfloat16_rn(__uint_as_float(r[i]));
                    }
                }
            }
        }
    }

    // no CTA of the pair leaves (or frees TMEM) while the other may still signal it
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ the cluster-split kernel
// K cut into S contiguous slices whose partials meet on chip.  A cluster of 2S CTAs is S CTA
// pairs; pair p (ranks 2p, 2p + 1) computes slice p of the cluster's current 256 x 256 tile
// exactly as the pair kernel computes a whole tile: cta_group::2 MMAs, its K blocks in ascending
// order, into one of two TMEM accumulators.  The epilogue then combines the S accumulators
// through distributed shared memory.  The tile's 256 columns are cut into 16 chunks of 16;
// chunk c belongs to slice c % S.  For each chunk, the CTA of the owning slice that holds the
// same 128 rows adds ((P0 + P1) + ...) + P(S-1), element by element in fp32, rounds once and
// stores C; each other CTA pushes its piece of the chunk (st.async) into a two-slot receive
// ring of the owner, whose remote arrive hands the slot back once it has been read.  The
// partials never touch HBM, and no floating-point atomic is used.  A cluster walks tiles
// c, c + clusters, ...; the accumulator double buffer lets the exchange of one tile overlap the
// MMAs of the next.
namespace cs {
constexpr int STAGES = 5;
constexpr int CW = 16;                          // columns per exchanged chunk
constexpr int NCH = pair::TILE_N / CW;          // chunks per tile
constexpr int RING = 2;                         // receive slots per epilogue warp
constexpr int MAX_S = 4;
constexpr int PIECE = 32 * CW * 4;              // one sender's piece for one warp: 32 rows x 16 fp32
constexpr int SLOT = (MAX_S - 1) * PIECE;       // every other slice's piece
constexpr int RECV_BYTES = EPI_WARPS * RING * SLOT;
struct Bars {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint64_t rfull[EPI_WARPS][RING];         // owner: every lane of every other slice stored its piece
    uint64_t rfree[EPI_WARPS][RING][MAX_S];  // sender: slot r of warp w in slice o's CTA may be refilled
    uint32_t tmem_addr;
    int abort;
};
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * pair::ST_BYTES + RECV_BYTES + sizeof(Bars) + 64;
static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
}  // namespace cs

__global__ void __launch_bounds__(THREADS, 1)
bi_gemm_bf16_cluster_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                            void* __restrict__ C, int M, int N, int K, int c_bf16, int gm, int S, uint32_t* err) {
    using pair::ROWS;
    using pair::COLS;
    using pair::TILE_M;
    using pair::TILE_N;
    using pair::A_ST;
    using pair::B_ST;
    using pair::ST_BYTES;
    using pair::ACC_COLS;
    using pair::TMEM_COLS;
    constexpr int STAGES = cs::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_ST;
    uint8_t* recv = sB + STAGES * B_ST;
    cs::Bars* bars = reinterpret_cast<cs::Bars*>(recv + cs::RECV_BYTES);
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int slice = (int)(rank >> 1);
    const uint32_t rp = rank & 1u;            // 0: the pair's leader, which issues the MMAs
    const uint32_t leader = rank & ~1u;
    const int csize = 2 * S;
    const int cluster_id = (int)blockIdx.x / csize, n_clusters = (int)gridDim.x / csize;
    const int tiles_m = (M + TILE_M - 1) / TILE_M;
    const int tiles_n = (N + TILE_N - 1) / TILE_N;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = (K + BK - 1) / BK;
    const int kb0 = (int)((int64_t)slice * num_kb / S), kb1 = (int)((int64_t)(slice + 1) * num_kb / S);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bars->tfull[b]), 1);
            mbar_init(smem_u32(&bars->tempty[b]), 2 * EPI_WARPS);
        }
        mbar_init(smem_u32(&bars->drain), 1);
        for (int w = 0; w < EPI_WARPS; ++w)
            for (int r = 0; r < cs::RING; ++r) {
                mbar_init(smem_u32(&bars->rfull[w][r]), (uint32_t)(32 * (S - 1)));  // every lane of each sender
                for (int o = 0; o < cs::MAX_S; ++o) mbar_init(smem_u32(&bars->rfree[w][r][o]), 1);
            }
        bars->abort = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmW);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&bars->tmem_addr), TMEM_COLS);
        tmem_relinquish_pair();
    }
    // every CTA's barriers are initialised and its TMEM allocated before any signal crosses the cluster
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_addr;
    pdl_wait();  // A and W may come from the kernel before this one, and it may still read C
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;  // k-blocks issued by this CTA so far (the ring runs across tiles)
            for (int t = cluster_id; t < num_tiles && !*abort; t += n_clusters) {
                int mt, nt;
                tile_coords(t, tiles_m, tiles_n, gm, mt, nt);
                const int m0 = mt * TILE_M + (int)rp * ROWS, n0 = nt * TILE_N + (int)rp * COLS;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = (int)(it % STAGES);
                    const uint32_t round = it / STAGES;
                    if (!mbar_wait(smem_u32(&bars->empty[s]), (round & 1u) ^ 1u, abort)) {
                        fail(err, abort, bi::DEVERR_WAIT_TMA);
                        break;
                    }
                    const uint32_t fb = smem_u32(&bars->full[s]);
                    if (rp == 0) mbar_arrive_expect_tx(fb, 2 * ST_BYTES);  // this stage of both CTAs
                    const uint32_t fb_leader = mapa(fb, leader);
                    tma_load_2d_pair(smem_u32(sA + s * A_ST), &tmA, kb * BK, m0, fb_leader);
                    tma_load_2d_pair(smem_u32(sB + s * B_ST), &tmW, n0, kb * BK, fb_leader);
                    tma_load_2d_pair(smem_u32(sB + s * B_ST + B_BOX), &tmW, n0 + 64, kb * BK, fb_leader);
                }
            }
            if (*abort) {  // let loads in flight land before the shared memory is released
                if (rp == 0) {
                    for (uint32_t i = it > (uint32_t)STAGES ? it - STAGES : 0u; i < it; ++i)
                        (void)mbar_wait(smem_u32(&bars->full[i % STAGES]), (i / STAGES) & 1u, nullptr);
                } else {
                    const uint64_t t0 = globaltimer();
                    while (globaltimer() - t0 < 200000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rp == 0) {
            constexpr uint32_t idesc = make_idesc_bf16_f32(TILE_M, TILE_N, 0, 1);
            const uint32_t peer_empty0 = mapa(smem_u32(&bars->empty[0]), rank | 1u);
            const uint32_t peer_tfull0 = mapa(smem_u32(&bars->tfull[0]), rank | 1u);
            uint32_t it = 0, local = 0;
            for (int t = cluster_id; t < num_tiles && !*abort; t += n_clusters, ++local) {
                const uint32_t acc = local & 1u, use = local >> 1;
                if (!mbar_wait(smem_u32(&bars->tempty[acc]), (use & 1u) ^ 1u, abort)) {
                    fail(err, abort, bi::DEVERR_WAIT_ACCUM);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = (int)(it % STAGES);
                    const uint32_t round = it / STAGES;
                    if (!mbar_wait(smem_u32(&bars->full[s]), round & 1u, abort)) {
                        fail(err, abort, bi::DEVERR_WAIT_FULL);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + s * A_ST);
                    const uint32_t b_base = smem_u32(sB + s * B_ST);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        const uint64_t adesc = make_smem_desc(a_base + k * UMMA_K * 2, 16, 1024, 2);
                        const uint64_t bdesc = make_smem_desc(b_base + k * UMMA_K * 128, B_BOX, 1024, 2);
                        mma_bf16_ss_pair(d_tmem, adesc, bdesc, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
                    }
                    mma_commit_pair(smem_u32(&bars->empty[s]));
                    mma_commit_pair(peer_empty0 + (uint32_t)s * 8u);
                }
                mma_commit_pair(smem_u32(&bars->tfull[acc]));
                mma_commit_pair(peer_tfull0 + acc * 8u);
            }
            mma_commit_pair(smem_u32(&bars->drain));  // TMEM is released only after every MMA completed
            (void)mbar_wait(smem_u32(&bars->drain), 0u, nullptr);
        }
    } else {
        const int quarter = warp & 3;  // this warp may read TMEM lanes 32*quarter .. +31
        const uint32_t tempty0 = rp == 0 ? smem_u32(&bars->tempty[0]) : mapa(smem_u32(&bars->tempty[0]), leader);
        const uint32_t ring = smem_u32(recv) + (uint32_t)(quarter * cs::RING * cs::SLOT);  // this warp's slots
        const uint32_t rfull0 = smem_u32(&bars->rfull[quarter][0]);
        bool alive = true;
        uint32_t local = 0;
        for (int t = cluster_id; t < num_tiles && alive; t += n_clusters, ++local) {
            const uint32_t acc = local & 1u, use = local >> 1;
            const bool ok = mbar_wait(smem_u32(&bars->tfull[acc]), use & 1u, abort);
            if (!ok) fail(err, abort, bi::DEVERR_WAIT_ACCUM);
            // tcgen05.ld is warp-collective: the whole warp takes the same branch
            if (!__all_sync(0xffffffffu, ok && !*abort)) break;
            tc_fence_after();
            int mt, nt;
            tile_coords(t, tiles_m, tiles_n, gm, mt, nt);
            const int row = mt * TILE_M + (int)rp * ROWS + quarter * 32 + lane;
            const uint32_t lane_addr = tmem_base + acc * ACC_COLS + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < cs::NCH; ++c) {
                uint32_t r[16];
                tmem_ld16(lane_addr + (uint32_t)(c * cs::CW), r);
                tmem_wait_ld();
                if (c == cs::NCH - 1) {  // every column of this accumulator is in registers: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(tempty0 + acc * 8u);
                }
                const int o = c % S;                                 // the slice that owns chunk c
                const int nown_o = (cs::NCH - o + S - 1) / S;
                const uint32_t n = local * (uint32_t)nown_o + (uint32_t)(c / S);  // o's running chunk count
                const int slot = (int)(n % cs::RING);
                const uint32_t par = (n / cs::RING) & 1u;
                if (o != slice) {
                    // push this piece into o's slot once o has read what was there before
                    const bool free_ok = __all_sync(
                        0xffffffffu, mbar_wait_cluster(smem_u32(&bars->rfree[quarter][slot][o]), par ^ 1u, abort));
                    if (!free_ok) {
                        if (lane == 0) fail(err, abort, bi::DEVERR_WAIT_CLUSTER);
                        alive = false;
                        break;
                    }
                    const uint32_t owner = (uint32_t)(2 * o) + rp;
                    const int idx = slice < o ? slice : slice - 1;
                    const uint32_t dst =
                        mapa(ring + (uint32_t)(slot * cs::SLOT + idx * cs::PIECE + lane * cs::CW * 4), owner);
                    const uint32_t bar = mapa(rfull0 + (uint32_t)slot * 8u, owner);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        st_cluster_v4(dst + 16u * i, r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
                    mbar_arrive_cluster(bar);  // release: this lane's stores are visible before its arrival
                    continue;
                }
                // this slice owns chunk c: wait for the other slices' pieces, add in slice order
                const bool full_ok = __all_sync(0xffffffffu, mbar_wait_cluster(rfull0 + (uint32_t)slot * 8u, par, abort));
                if (!full_ok) {
                    if (lane == 0) fail(err, abort, bi::DEVERR_WAIT_CLUSTER);
                    alive = false;
                    break;
                }
                float v[16];
                for (int q = 0; q < S; ++q) {
                    float p[16];
                    if (q == slice) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) p[i] = __uint_as_float(r[i]);
                    } else {
                        const int idx = q < slice ? q : q - 1;
                        const uint32_t src = ring + (uint32_t)(slot * cs::SLOT + idx * cs::PIECE + lane * cs::CW * 4);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                                         : "=f"(p[4 * i]), "=f"(p[4 * i + 1]), "=f"(p[4 * i + 2]), "=f"(p[4 * i + 3])
                                         : "r"(src + 16u * i));
                    }
                    if (q == 0) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = p[i];
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = __fadd_rn(v[i], p[i]);
                    }
                }
                __syncwarp();
                // the slot has been read: every sender may refill it
                if (lane < S && lane != slice)
                    mbar_arrive_cluster(mapa(smem_u32(&bars->rfree[quarter][slot][slice]), (uint32_t)(2 * lane) + rp));
                const int col = nt * TILE_N + c * cs::CW;
                if (row >= M || col >= N) continue;
                if (!c_bf16) {
                    float* dst = static_cast<float*>(C) + (int64_t)row * N + col;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (col + 4 * i + 4 <= N)
                            *reinterpret_cast<float4*>(dst + 4 * i) = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2],
                                                                                  v[4 * i + 3]);
                } else {
                    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(C) + (int64_t)row * N + col;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        if (col + 8 * h + 8 <= N)
                            *reinterpret_cast<uint4*>(dst + 8 * h) = make_uint4(
                                bi::pack_bf16x2(v[8 * h], v[8 * h + 1]), bi::pack_bf16x2(v[8 * h + 2], v[8 * h + 3]),
                                bi::pack_bf16x2(v[8 * h + 4], v[8 * h + 5]), bi::pack_bf16x2(v[8 * h + 6], v[8 * h + 7]));
                }
            }
        }
    }

    // no CTA leaves (or frees TMEM) while a peer may still store into it or signal it
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side
int num_sms() {
    static int cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        cached[dev] = n;
    }
    return cached[dev];
}

template <int BN>
bool ensure_smem_attr() {
    static std::once_flag once[64];
    static bool ok[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::call_once(once[dev], [&] {
        ok[dev] = cudaFuncSetAttribute(bi_gemm_bf16_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Tile<BN>::SMEM_BYTES) == cudaSuccess;
    });
    return ok[dev];
}

// Launch the GEMM on operands with arbitrary (16-byte multiple) row strides: A [M, K] with
// row stride lda, W [K, N] with row stride ldw, C [M, N] with row stride N.
template <int BN>
int launch_gemm_bn(const void* A, int64_t lda, const void* W, int64_t ldw, void* C, int64_t M, int64_t N, int64_t K,
                   bool c_bf16, cudaStream_t stream) {
    uint32_t* err = bi::device_error_word();
    if (!err || !ensure_smem_attr<BN>()) return BI_ERR_CUDA;
    CUtensorMap tmA, tmW;
    if (!bi::make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, BK,
                          BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    if (!bi::make_tmap_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, (uint64_t)N, (uint64_t)K, (uint64_t)ldw * 2, 64,
                          BK, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int sms = num_sms();
    if (sms <= 0) return BI_ERR_CUDA;
    const int gm = 16;  // ~16 row tiles x ~9 column tiles in flight: A and W blocks balanced within L2
    dim3 grid((unsigned)(tiles < sms ? tiles : sms));
    if (bi::launch_pdl(bi_gemm_bf16_tc_kernel<BN>, grid, dim3(THREADS), Tile<BN>::SMEM_BYTES, stream, 0u, tmA, tmW, C,
                       (int)M, (int)N, (int)K, c_bf16 ? 1 : 0, gm, err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

// Shared-memory attribute of the pair kernel (once per device).
bool pair_smem_attr() {
    static std::once_flag once[64];
    static bool ok[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::call_once(once[dev], [&] {
        ok[dev] = cudaFuncSetAttribute(bi_gemm_bf16_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)pair::SMEM_BYTES) == cudaSuccess;
    });
    return ok[dev];
}

// The CTA-pair kernel: 256 x 256 tiles over 2-CTA clusters, one cluster per SM pair at most.
int launch_gemm_pair(const void* A, int64_t lda, const void* W, int64_t ldw, void* C, int64_t M, int64_t N,
                     int64_t K, bool c_bf16, cudaStream_t stream) {
    uint32_t* err = bi::device_error_word();
    if (!err || !pair_smem_attr()) return BI_ERR_CUDA;
    const int sms = num_sms();
    if (sms < 2) return BI_ERR_CUDA;
    const int64_t clusters = sms / 2;
    CUtensorMap tmA, tmW;
    if (!bi::make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, BK,
                          pair::ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    if (!bi::make_tmap_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, (uint64_t)N, (uint64_t)K, (uint64_t)ldw * 2, 64,
                          BK, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    const int64_t tiles = ((M + pair::TILE_M - 1) / pair::TILE_M) * ((N + pair::TILE_N - 1) / pair::TILE_N);
    const int gm = 16;  // row tiles per group of the tile walk (L2 reuse of A and W blocks)
    const int64_t pairs = tiles < clusters ? tiles : clusters;
    // the pair kernel's cluster shape is compiled in (__cluster_dims__)
    if (bi::launch_pdl(bi_gemm_bf16_pair_kernel, dim3((unsigned)(2 * pairs)), dim3(THREADS), pair::SMEM_BYTES, stream,
                       0u, tmA, tmW, C, (int)M, (int)N, (int)K, c_bf16 ? 1 : 0, gm, err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

// Clusters of 2S CTAs of the cluster-split kernel that fit on the device at once (cached per
// device and S).  The grid never exceeds it, so every cluster is resident and walks its tiles.
int split_clusters(int S) {
    static std::mutex mu;
    static int cached[64][cs::MAX_S + 1];
    int dev = 0;
    if (S < 2 || S > cs::MAX_S || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev][S] == 0) {
        cached[dev][S] = -1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * S));
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = cs::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)(2 * S);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, bi_gemm_bf16_cluster_kernel, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            return -1;
        }
        cached[dev][S] = n > 0 ? n : -1;
    }
    return cached[dev][S];
}

bool cluster_smem_attr() {
    static std::once_flag once[64];
    static bool ok[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::call_once(once[dev], [&] {
        ok[dev] = cudaFuncSetAttribute(bi_gemm_bf16_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)cs::SMEM_BYTES) == cudaSuccess &&
                  cudaFuncSetAttribute(bi_gemm_bf16_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                       1) == cudaSuccess;
    });
    return ok[dev];
}

// The cluster-split kernel: 256 x 256 tiles, K in S slices on S CTA pairs of one cluster.
int launch_gemm_cluster(const void* A, int64_t lda, const void* W, int64_t ldw, void* C, int64_t M, int64_t N,
                        int64_t K, bool c_bf16, int S, cudaStream_t stream) {
    uint32_t* err = bi::device_error_word();
    if (!err || !cluster_smem_attr()) return BI_ERR_CUDA;
    if (S < 2 || S > cs::MAX_S || S > (K + BK - 1) / BK) return BI_ERR_INVALID_ARG;
    const int fit = split_clusters(S);
    if (fit <= 0) return BI_ERR_CUDA;
    CUtensorMap tmA, tmW;
    if (!bi::make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, BK,
                          pair::ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    if (!bi::make_tmap_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, (uint64_t)N, (uint64_t)K, (uint64_t)ldw * 2, 64,
                          BK, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    const int64_t tiles = ((M + pair::TILE_M - 1) / pair::TILE_M) * ((N + pair::TILE_N - 1) / pair::TILE_N);
    const int64_t clusters = tiles < fit ? tiles : fit;
    const int gm = 16;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * S * clusters));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = cs::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned na = 0;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)(2 * S);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    if (bi::pdl_enabled()) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, bi_gemm_bf16_cluster_kernel, tmA, tmW, C, (int)M, (int)N, (int)K, c_bf16 ? 1 : 0, gm,
                           S, err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

// The plan for a weight of shape [K, N], a function of (N, K) and the device only, never of M:
// CTA pairs when a row of 256-wide pair tiles fits the GPU's SM pairs (N <= 18944 on a B200),
// single CTAs with 128 x 256 tiles for wider weights.  A wide weight then has enough column
// tiles to occupy every SM at any M in one round, where pair tiles would need two rounds
// for the small batches of decoding.
bool use_pairs(int64_t N, int64_t K) {
    (void)K;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    return (N + pair::TILE_N - 1) / pair::TILE_N <= sms / 2;
}

// The K split of the plan.  The split kernel is built and tested (bi_ctrl_gemm_split runs it
// with any S), but the plan keeps S = 1 for every shape.  Measured on a B200 for the 4096- and
// 6144-wide projections: a split fills idle SM pairs and pays while M fits one or two rows of
// tiles (K = 14336, M = 8: 35 us at S = 4 against 79 us), but its combine of fp32 partials
// through L2 costs 6 % to 5x once M reaches 1024, and the plan may not depend on M.
int splits_for(int64_t N, int64_t K) {
    (void)N;
    (void)K;
    return 1;
}

int launch_gemm(const void* A, int64_t lda, const void* W, int64_t ldw, void* C, int64_t M, int64_t N, int64_t K,
                bool c_bf16, int splits, cudaStream_t stream) {
    if (use_pairs(N, K)) {
        if (splits == 1) return launch_gemm_pair(A, lda, W, ldw, C, M, N, K, c_bf16, stream);
        return launch_gemm_cluster(A, lda, W, ldw, C, M, N, K, c_bf16, splits, stream);
    }
    if (splits != 1) return BI_ERR_INVALID_ARG;
    return launch_gemm_bn<256>(A, lda, W, ldw, C, M, N, K, c_bf16, stream);
}

int gemm_shape_checks(const void* A, const void* W, const void* C, int64_t M, int64_t N, int64_t K, int c_dtype) {
    if (c_dtype != BI_F32 && c_dtype != BI_BF16) return BI_ERR_INVALID_ARG;
    if (M < 0 || N <= 0 || K <= 0) return BI_ERR_INVALID_ARG;
    if (M == 0) return -1;  // no-op
    if (!A || !W || !C) return BI_ERR_INVALID_ARG;
    if (!bi::aligned16(A) || !bi::aligned16(W) || !bi::aligned16(C)) return BI_ERR_MISALIGNED;
    if (K % 8 != 0 || N % 8 != 0) return BI_ERR_MISALIGNED;  // 16-byte row strides for the TMA unit
    if (M > (1LL << 30) || N > (1LL << 30) || K > (1LL << 30)) return BI_ERR_UNSUPPORTED_SHAPE;
    if (((M + pair::TILE_M - 1) / pair::TILE_M) * ((N + pair::TILE_N - 1) / pair::TILE_N) > 0x7fffffffLL)
        return BI_ERR_UNSUPPORTED_SHAPE;
    return BI_OK;
}

// ------------------------------------------------------------------ comparator: split-K chosen by M
// Sum of S fp32 partials in order s = 0, 1, ..., S-1, then the output rounding.
__global__ void splitk_reduce_kernel(const float* __restrict__ part, void* __restrict__ C, int64_t MN, int S,
                                     int c_bf16) {
    const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (i >= MN) return;
    float4 acc = *reinterpret_cast<const float4*>(part + i);
    for (int s = 1; s < S; ++s) {
        const float4 p = *reinterpret_cast<const float4*>(part + (int64_t)s * MN + i);
        acc.x = __fadd_rn(acc.x, p.x);
        acc.y = __fadd_rn(acc.y, p.y);
        acc.z = __fadd_rn(acc.z, p.z);
        acc.w = __fadd_rn(acc.w, p.w);
    }
    if (c_bf16) {
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(C) + i) =
            make_uint2(bi::pack_bf16x2(acc.x, acc.y), bi::pack_bf16x2(acc.z, acc.w));
    } else {
        *reinterpret_cast<float4*>(static_cast<float*>(C) + i) = acc;
    }
}

// The split a batch-size-adaptive library would pick: enough K slices to fill the GPU's SM
// pairs when the batch alone yields too few output tiles (1, 2, 4 or 8, with K / S a multiple
// of 64).
int splitk_for(int64_t M, int64_t N, int64_t K) {
    const bool pairs = use_pairs(N, K);
    const int64_t tm = pairs ? pair::TILE_M : BM, tn = 256;
    const int64_t tiles = ((M + tm - 1) / tm) * ((N + tn - 1) / tn);
    const int slots = (num_sms() > 0 ? num_sms() : 148) / (pairs ? 2 : 1);
    int S = 1;
    while (S < 8 && tiles * S * 2 <= slots && K % ((int64_t)S * 2 * BK) == 0) S *= 2;
    return S;
}

}  // namespace

BI_API int bi_gemm_splits(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0) return 0;
    return splits_for(N, K);
}

BI_API size_t bi_gemm_counter_bytes(int64_t M, int64_t N, int64_t K) {
    (void)M; (void)N; (void)K;
    return 0;  // a K split meets on chip: no counters
}

BI_API size_t bi_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
    (void)M; (void)N; (void)K;
    return 0;  // a K split meets on chip: no workspace
}

BI_API int bi_gemm(const void* A, const void* W, void* C, int64_t M, int64_t N, int64_t K, int c_dtype, void* ws,
                   size_t ws_bytes, void* stream) {
    (void)ws; (void)ws_bytes;
    const int c = gemm_shape_checks(A, W, C, M, N, K, c_dtype);
    if (c < 0) return BI_OK;
    if (c != BI_OK) return c;
    return launch_gemm(A, K, W, N, C, M, N, K, c_dtype == BI_BF16, splits_for(N, K), bi::as_stream(stream));
}

BI_API size_t bi_ctrl_gemm_split_workspace_size(int64_t M, int64_t N, int64_t K, int32_t splits) {
    (void)M; (void)N; (void)K; (void)splits;
    return 0;
}

BI_API int bi_ctrl_gemm_split(const void* A, const void* W, void* C, int64_t M, int64_t N, int64_t K, int c_dtype,
                              int32_t splits, void* ws, size_t ws_bytes, void* stream) {
    (void)ws; (void)ws_bytes;
    const int c = gemm_shape_checks(A, W, C, M, N, K, c_dtype);
    if (c < 0) return BI_OK;
    if (c != BI_OK) return c;
    if (!use_pairs(N, K) && splits != 1) return BI_ERR_UNSUPPORTED_SHAPE;
    if (splits < 1 || splits > cs::MAX_S || splits > (K + BK - 1) / BK) return BI_ERR_INVALID_ARG;
    return launch_gemm(A, K, W, N, C, M, N, K, c_dtype == BI_BF16, splits, bi::as_stream(stream));
}

BI_API size_t bi_ctrl_gemm_splitk_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    const int S = splitk_for(M, N, K);
    return S > 1 ? (size_t)S * M * N * sizeof(float) : 0;
}

BI_API int bi_ctrl_gemm_splitk(const void* A, const void* W, void* C, int64_t M, int64_t N, int64_t K, int c_dtype,
                               void* ws, size_t ws_bytes, void* stream) {
    const int c = gemm_shape_checks(A, W, C, M, N, K, c_dtype);
    if (c < 0) return BI_OK;
    if (c != BI_OK) return c;
    cudaStream_t s = bi::as_stream(stream);
    const int S = splitk_for(M, N, K);
    if (S == 1) return launch_gemm(A, K, W, N, C, M, N, K, c_dtype == BI_BF16, 1, s);
    const size_t need = (size_t)S * M * N * sizeof(float);
    if (!ws || ws_bytes < need || !bi::aligned16(ws)) return BI_ERR_WORKSPACE;
    const int64_t KS = K / S;
    float* part = static_cast<float*>(ws);
    for (int i = 0; i < S; ++i) {
        const int st = launch_gemm(static_cast<const __nv_bfloat16*>(A) + i * KS, K,
                                   static_cast<const __nv_bfloat16*>(W) + i * KS * N, N, part + (int64_t)i * M * N, M,
                                   N, KS, false, 1, s);
        if (st != BI_OK) return st;
    }
    const int64_t MN = M * N;  // N % 8 == 0, so MN is a multiple of 4
    const int64_t threads = (MN / 4 + 255) / 256;
    splitk_reduce_kernel<<<(unsigned)threads, 256, 0, s>>>(part, C, MN, S, c_dtype == BI_BF16 ? 1 : 0);
    return bi::launch_status();
}
