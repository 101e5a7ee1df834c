// bi_prefill_attn.cu -- batch-invariant causal prefill attention (grouped-query, variable length)
// on the sm_100 tensor cores (tcgen05, accumulators in TMEM).
//
// Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section "Attention".
// FlashAttention-2-style kernels are batch-invariant when they parallelise over queries and
// reduce keys/values inside one program in a fixed order.  The order must not change with
// the batch or with how a sequence is split.  Cached and new keys/values must share one
// layout.
//
// Layout: query rows of sequence b are rows q_indptr[b] .. q_indptr[b+1]-1 of q (row stride
// ldq elements, head h at columns [h*128, h*128 + 128)).  Query row i of the sequence sits at
// position q_pos0[b] + i.  Keys and values of sequence b are rows kv_indptr[b] + p of the packed
// caches [tokens, Hkv, 128], for positions p = 0 .. position of the query (causal).
//
// Persistent CTAs, one per SM, each walking work items (a 128-row query tile of a sequence,
// one query head) in a fixed order; 18 warps:
//   warp 0      TMA producer: each item's Q tile into one of two Q buffers (so the next item's
//               tile arrives while this one runs), then its K and V blocks of 64 positions into
//               a 3-stage ring that runs on across items
//   warp 1      tcgen05.mma issuer (and TMEM owner):
//                 S_j = Q K_j^T into one of two TMEM score buffers;
//                 O += P_hi V_j + P_lo V_j into the TMEM output accumulator
//   warps 2..17 softmax and epilogue, four threads per query row (TMEM lane): thread p takes
//               keys [16p, 16p + 16) of each block and output dims [32p, 32p + 32)
// KV blocks of 64 positions, starting at position 0, are visited in ascending order.  For
// block j, each row computes, in base-2 units:
//   t = S_j * scale * log2(e) (masked to -inf past the row's position)
//   m' = m, or the block max when that exceeds m by more than 8 (then O and l are rescaled
//        by 2^(m - m'), read from and written back to TMEM)
//   p = 2^(t - m') (one fused multiply-add, the hardware's approximate exp2);
//   l += sum p (a fixed summation tree);  P = hi + lo, hi = p cut to bf16, lo = bf16(p - hi)
// and out = O * (1 / l) rounded to bf16.  Every decision above is row-local.  Blocks past a row's
// position contribute exact zeros: masked scores, zeroed values past the tile's last position.
// So the rows a tile shares with a row never change its bits.
#include <mutex>

#include "bi_common.cuh"
#include "bi_model.h"
#include "bi_sm100.cuh"
#include "bi_tma_host.cuh"

using namespace bi::sm100;

namespace {

constexpr int D = 128;
constexpr int QT = 128;               // query rows per CTA (the MMA's M)
constexpr int KB = 64;                // keys per block
constexpr int NST = 3;                // K/V ring stages
constexpr int PARTS = 4;              // softmax threads per query row
constexpr int SM_WARPS = 4 * PARTS;   // softmax warps (each TMEM lane quarter is read by PARTS warps)
constexpr int THREADS = 32 * (2 + SM_WARPS);  // producer, MMA, softmax warps
constexpr int KEYS_PER = KB / PARTS;  // keys of a block per softmax thread
constexpr int DIMS_PER = D / PARTS;   // output dims per softmax thread
constexpr int Q_BOX = 64 * QT * 2;    // 64 dims x 128 rows = 16 KB
constexpr int KV_BOX = 64 * KB * 2;   // 64 dims x 64 keys = 8 KB
constexpr int Q_BYTES = 2 * Q_BOX;    // 32 KB
constexpr int KV_BLOCK = 2 * KV_BOX;  // 16 KB: K (or V) of one block
constexpr int P_BYTES = QT * KB * 2;  // 16 KB: one bf16 P tile
constexpr float RESCALE_GAP = 8.0f;   // raise the reference max only past this margin (base 2: x256)
constexpr uint32_t TMEM_COLS = 256;   // S x 2 (64 columns each) + O (128 columns)
constexpr uint32_t O_COL = 128;

struct Bars {
    uint64_t q_full[2];   // the Q tile of this CTA's item n is in Q buffer n % 2
    uint64_t q_empty[2];  // every QK^T of item n is done: Q buffer n % 2 may take item n + 2's tile
    uint64_t kv_full[NST];
    uint64_t kv_empty[NST];
    uint64_t s_full[2];
    uint64_t p_full;   // the softmax warps wrote P_j (and rescaled O)
    uint64_t p_empty;  // PV_j done: the P tiles are free and O is stable
    uint64_t o_full;   // the last PV of an item is done
    uint64_t drain;    // every MMA this CTA issued has completed
    uint64_t xchg;     // the softmax warps swapped their partial row maxima (or sums)
    float xmax[2][PARTS][QT];  // [block parity][part][row]
    float xsum[PARTS][QT];     // [part][row]
    uint32_t tmem_addr;
    int abort;
};

constexpr size_t SMEM_BYTES = 1024 + 2 * Q_BYTES + 2 * NST * KV_BLOCK + 2 * P_BYTES + sizeof(Bars) + 64;

// One work item: a 128-row query tile of one sequence, for one query head.
struct Item {
    int h, g;              // query head and its kv head
    int q_row0, n_q;       // first query row, live rows
    int pos0, kv_base;     // position of the first row; the sequence's first cache row
    int last_pos, nb;      // the highest position a live row sees; KV blocks visited
    bool live, bad;        // rows to compute; a layout the documentation does not allow
};

// Item i of the launch: the tiles in descending order, every head of a tile in turn, so that
// the longer tiles of each sequence come first.
__device__ __forceinline__ Item item_of(int i, int Hq, int Hkv, int n_tiles, int B, const int32_t* q_indptr,
                                        const int32_t* q_tile_indptr, const int32_t* kv_indptr,
                                        const int32_t* q_pos0, int q_rows, int cache_tokens) {
    Item it;
    const int rank = i / Hq;
    it.h = i - rank * Hq;
    it.g = it.h / (Hq / Hkv);
    const int tile = n_tiles - 1 - rank;
    // the sequence that owns this tile: the last b with q_tile_indptr[b] <= tile
    int lo = 0, hi = B;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (q_tile_indptr[mid] <= tile) lo = mid; else hi = mid;
    }
    const int b = lo;
    const int qt = tile - q_tile_indptr[b];
    it.q_row0 = q_indptr[b] + qt * QT;
    it.n_q = min(QT, q_indptr[b + 1] - it.q_row0);
    it.pos0 = q_pos0[b] + qt * QT;
    it.kv_base = kv_indptr[b];
    it.last_pos = it.pos0 + it.n_q - 1;
    it.nb = it.last_pos / KB + 1;
    it.live = it.n_q > 0;  // a tile index past the last sequence's tiles has none
    // the documented layout, checked before any copy or store
    it.bad = it.live && (q_indptr[b + 1] > q_rows || q_indptr[b] < 0 || it.pos0 < 0 || it.kv_base < 0 ||
                         (int64_t)it.kv_base + it.last_pos >= (int64_t)cache_tokens);
    return it;
}

__device__ __forceinline__ void fail(uint32_t* err, volatile int* abort, uint32_t bit) {
    atomicOr(err, bit);
    *abort = 1;
}

// 2^x with the hardware's approximate base-2 exponential (relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Generic-proxy writes to shared memory become visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Each thread of the warp writes 32 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
           "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
           "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
           "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
// Each thread of the warp reads 16 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(THREADS, 1)
prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ q_indptr,
                       const int32_t* __restrict__ q_tile_indptr, const int32_t* __restrict__ kv_indptr,
                       const int32_t* __restrict__ q_pos0, int B, int Hq, int Hkv, int q_rows, int cache_tokens,
                       int n_tiles, float scale_log2, __nv_bfloat16* __restrict__ out, int64_t ldo, uint32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(base);            // Q buffer i at sQ + i * Q_BYTES
    const uint32_t sK = sQ + 2 * Q_BYTES;          // stage s at sK + s * KV_BLOCK
    const uint32_t sV = sK + NST * KV_BLOCK;       // stage s at sV + s * KV_BLOCK
    const uint32_t sPh = sV + NST * KV_BLOCK;      // P high parts
    const uint32_t sPl = sPh + P_BYTES;            // P low parts
    Bars* bars = reinterpret_cast<Bars*>(base + 2 * Q_BYTES + 2 * NST * KV_BLOCK + 2 * P_BYTES);
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = n_tiles * Hq;
    pdl_wait();  // q, the cache and the index arrays may come from the kernels just before this one
    pdl_trigger();
    auto item = [&](int i) {
        return item_of(i, Hq, Hkv, n_tiles, B, q_indptr, q_tile_indptr, kv_indptr, q_pos0, q_rows, cache_tokens);
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bars->q_full[i]), 1);
            mbar_init(smem_u32(&bars->q_empty[i]), 1);
            mbar_init(smem_u32(&bars->s_full[i]), 1);
        }
        for (int s = 0; s < NST; ++s) {
            mbar_init(smem_u32(&bars->kv_full[s]), 1);
            mbar_init(smem_u32(&bars->kv_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->p_full), SM_WARPS);
        mbar_init(smem_u32(&bars->p_empty), 1);
        mbar_init(smem_u32(&bars->o_full), 1);
        mbar_init(smem_u32(&bars->drain), 1);
        mbar_init(smem_u32(&bars->xchg), SM_WARPS);
        bars->abort = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_addr), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_addr;

    // Every role walks the same items in the same order and counts the same KV blocks: n counts
    // this CTA's items, gb the KV blocks of all its items so far (ring stages, score buffers and
    // barrier phases follow gb, so they run on across items).
    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            uint32_t gb = 0, n = 0;
            bool stop = false;
            for (int ix = blockIdx.x; ix < n_items && !stop; ix += gridDim.x) {
                const Item it = item(ix);
                if (it.bad) atomicOr(err, bi::DEVERR_BAD_PREFILL);
                if (!it.live || it.bad) continue;
                const uint32_t qb = n & 1u;
                // Q buffer qb held item n - 2, whose QK^T MMAs must be done with it
                if (n >= 2 && !mbar_wait(smem_u32(&bars->q_empty[qb]), ((n - 2) >> 1) & 1u, abort)) {
                    fail(err, abort, bi::DEVERR_WAIT_TMA);
                    break;
                }
                const uint32_t qf = smem_u32(&bars->q_full[qb]);
                mbar_arrive_expect_tx(qf, Q_BYTES);
                tma_load_2d(sQ + qb * Q_BYTES, &tmQ, it.h * D, it.q_row0, qf);
                tma_load_2d(sQ + qb * Q_BYTES + Q_BOX, &tmQ, it.h * D + 64, it.q_row0, qf);
                ++n;
                for (int j = 0; j < it.nb; ++j, ++gb) {
                    const uint32_t s = gb % NST;
                    if (!mbar_wait(smem_u32(&bars->kv_empty[s]), ((gb / NST) & 1u) ^ 1u, abort)) {
                        fail(err, abort, bi::DEVERR_WAIT_TMA);
                        stop = true;
                        break;
                    }
                    const uint32_t fb = smem_u32(&bars->kv_full[s]);
                    mbar_arrive_expect_tx(fb, 2 * KV_BLOCK);
                    const int row = it.kv_base + j * KB;
                    tma_load_2d(sK + s * KV_BLOCK, &tmK, it.g * D, row, fb);
                    tma_load_2d(sK + s * KV_BLOCK + KV_BOX, &tmK, it.g * D + 64, row, fb);
                    tma_load_2d(sV + s * KV_BLOCK, &tmV, it.g * D, row, fb);
                    tma_load_2d(sV + s * KV_BLOCK + KV_BOX, &tmV, it.g * D + 64, row, fb);
                }
            }
            if (*abort) {  // let the copies in flight land before the CTA's shared memory is released
                for (uint32_t m = n > 2u ? n - 2u : 0u; m < n; ++m)
                    (void)mbar_wait(smem_u32(&bars->q_full[m & 1u]), (m >> 1) & 1u, nullptr);
                for (uint32_t j = gb > (uint32_t)NST ? gb - NST : 0u; j < gb; ++j)
                    (void)mbar_wait(smem_u32(&bars->kv_full[j % NST]), (j / NST) & 1u, nullptr);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = make_idesc_bf16_f32(QT, KB, 0, 0);  // Q and K both K-major
            constexpr uint32_t idesc_o = make_idesc_bf16_f32(QT, D, 0, 1);   // P K-major, V N-major
            uint32_t gb = 0, n = 0;
            bool ok = true;
            // S for global block b = Q K_b^T into score buffer b % 2 (8 steps of 16 dims; dims
            // 64..127 sit in the second box)
            auto issue_s = [&](uint32_t b, uint32_t q_smem) -> bool {
                const uint32_t s = b % NST;
                if (!mbar_wait(smem_u32(&bars->kv_full[s]), (b / NST) & 1u, abort)) {
                    fail(err, abort, bi::DEVERR_WAIT_FULL);
                    return false;
                }
                tc_fence_after();
                const uint32_t d = tmem + (b & 1u) * KB;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (uint32_t)(k & 3) * 32u;
                    const uint64_t ad = make_smem_desc(q_smem + (uint32_t)(k >> 2) * Q_BOX + off, 16, 1024, 2);
                    const uint64_t bd = make_smem_desc(sK + s * KV_BLOCK + (uint32_t)(k >> 2) * KV_BOX + off, 16, 1024, 2);
                    mma_bf16_ss(d, ad, bd, idesc_s, k > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(&bars->s_full[b & 1u]));
                return true;
            };
            for (int ix = blockIdx.x; ok && ix < n_items; ix += gridDim.x) {
                const Item it = item(ix);
                if (!it.live || it.bad) continue;
                const uint32_t qb = n & 1u, q_smem = sQ + qb * Q_BYTES;
                if (!mbar_wait(smem_u32(&bars->q_full[qb]), (n >> 1) & 1u, abort)) {
                    fail(err, abort, bi::DEVERR_WAIT_FULL);
                    break;
                }
                for (int j = 0; ok && j < it.nb && j < 2; ++j) ok = issue_s(gb + (uint32_t)j, q_smem);
                for (int j = 0; ok && j < it.nb; ++j) {
                    const uint32_t b = gb + (uint32_t)j;
                    if (!mbar_wait(smem_u32(&bars->p_full), b & 1u, abort)) {
                        fail(err, abort, bi::DEVERR_WAIT_FULL);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t s = b % NST;
                    // O += P_hi V_b + P_lo V_b (4 steps of 16 keys each); the item's first block starts O
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        const uint32_t sP = part == 0 ? sPh : sPl;
#pragma unroll
                        for (int k = 0; k < KB / 16; ++k) {
                            const uint64_t ad = make_smem_desc(sP + (uint32_t)k * 32u, 16, 1024, 2);
                            const uint64_t bd = make_smem_desc(sV + s * KV_BLOCK + (uint32_t)k * 16u * 128u,
                                                               KV_BOX, 1024, 2);
                            mma_bf16_ss(tmem + O_COL, ad, bd, idesc_o, (j > 0 || part > 0 || k > 0) ? 1u : 0u);
                        }
                    }
                    mma_commit(smem_u32(&bars->p_empty));
                    mma_commit(smem_u32(&bars->kv_empty[s]));
                    if (j + 2 < it.nb) ok = issue_s(b + 2u, q_smem);
                }
                if (!ok || *abort) break;
                mma_commit(smem_u32(&bars->o_full));      // the item's O is complete
                mma_commit(smem_u32(&bars->q_empty[qb]));  // and its Q buffer is free
                gb += (uint32_t)it.nb;
                ++n;
            }
            // every MMA issued above completes before TMEM is released
            mma_commit(smem_u32(&bars->drain));
            (void)mbar_wait(smem_u32(&bars->drain), 0u, nullptr);
        }
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        // PARTS threads share a query row: `part` p takes keys [16p, 16p + 16) of every block and
        // output dims [32p, 32p + 32).  They swap their partial row maxima (and at the end their
        // partial sums) through shared memory behind an mbarrier.
        const int sw = warp - 2;              // softmax warp 0 .. SM_WARPS - 1
        const int part = sw >> 2;
        const int quarter = warp & 3;         // this warp reads TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;    // query row of the tile
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        uint32_t gb = 0, n = 0, xc = 0;       // KV blocks and items so far; exchanges so far
        bool ok = true;
        for (int ix = blockIdx.x; ok && ix < n_items; ix += gridDim.x) {
            const Item it = item(ix);
            if (!it.live || it.bad) continue;
            const bool live = r < it.n_q;
            const int qpos = it.pos0 + r;
            float m_ref = -INFINITY, l = 0.f;
            for (int j = 0; j < it.nb; ++j) {
                const uint32_t b = gb + (uint32_t)j;  // the CTA's KV block count: buffers and phases
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full[b & 1u]), (b >> 1) & 1u, abort));
                if (!ok) {
                    if (lane == 0) fail(err, abort, bi::DEVERR_WAIT_ACCUM);
                    break;
                }
                tc_fence_after();
                float sv[KEYS_PER];
                {
                    uint32_t r0[KEYS_PER];
                    tmem_ld_32x32b_x16(tmem + lane_off + (b & 1u) * KB + (uint32_t)(part * KEYS_PER), r0);
                    tmem_wait_ld();
    #pragma unroll
                    for (int c = 0; c < KEYS_PER; ++c) sv[c] = __uint_as_float(r0[c]);
                }
                const int kpos0 = j * KB + part * KEYS_PER;  // position of this thread's first key in the block
                // scores in base-2 units are t = s * scale * log2(e); keys past the row's position are
                // -inf.  A warp whose rows all sit at or past its last key of the block needs no mask.
                // The multiply is monotone, so the block max of t is the scaled max of the raw scores.
                const bool unmasked = __all_sync(0xffffffffu, live && kpos0 + KEYS_PER - 1 <= qpos);
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    #pragma unroll
                for (int c = 0; c < KEYS_PER; ++c) {
                    const float v = (unmasked || (live && kpos0 + c <= qpos)) ? sv[c] : -INFINITY;
                    sv[c] = v;
                    mx4[c & 3] = fmaxf(mx4[c & 3], v);
                }
                const float mine = __fmul_rn(fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])), scale_log2);
                bars->xmax[b & 1u][part][r] = mine;
                __threadfence_block();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->xchg));
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->xchg), xc & 1u, abort));
                ++xc;
                if (!ok) {
                    if (lane == 0) fail(err, abort, bi::DEVERR_WAIT_CLUSTER);
                    break;
                }
                float mx = bars->xmax[b & 1u][0][r];
    #pragma unroll
                for (int q = 1; q < PARTS; ++q) mx = fmaxf(mx, bars->xmax[b & 1u][q][r]);
                float m_new = m_ref;
                if (m_ref == -INFINITY || mx > m_ref + RESCALE_GAP) m_new = fmaxf(m_ref, mx);
                const bool need = m_new != m_ref && m_ref != -INFINITY;
                const float c_fac = need ? ex2_approx(__fsub_rn(m_ref, m_new)) : 1.0f;
                // the previous block's PV (of this item or the one before) must be done before P is
                // overwritten or O is rescaled
                if (b > 0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->p_empty), (b - 1u) & 1u, abort));
                    if (!ok) {
                        if (lane == 0) fail(err, abort, bi::DEVERR_WAIT_ACCUM);
                        break;
                    }
                    tc_fence_after();
                }
                if (__any_sync(0xffffffffu, need)) {  // a warp-collective TMEM round trip; c_fac is 1 where not needed
                    const uint32_t col = O_COL + (uint32_t)(part * DIMS_PER);
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(tmem + lane_off + col, o);
                    tmem_wait_ld();
    #pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__fmul_rn(__uint_as_float(o[i]), c_fac));
                    tmem_st_32x32b_x32(tmem + lane_off + col, o);
                    tmem_wait_st();
                }
                if (need) l = __fmul_rn(l, c_fac);
                m_ref = m_new;
                // p = 2^(s * scale * log2(e) - m_ref), one fused multiply-add and the hardware exp2;
                // P = hi + lo with hi = p cut to bf16 (exact top 8 significant bits)
                // and lo = bf16(p - hi) (p - hi is exact in fp32); both go to the 128B-swizzled
                // K-major P tiles.  The partial row sum is four interleaved sums, added in a fixed order.
                const uint32_t row_off = (uint32_t)r * 128u;
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll
                for (int cc = 0; cc < KEYS_PER / 8; ++cc) {
                    uint32_t ph[4], pl[4];
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float p0 = ex2_approx(__fmaf_rn(sv[cc * 8 + 2 * e], scale_log2, -m_ref));
                        const float p1 = ex2_approx(__fmaf_rn(sv[cc * 8 + 2 * e + 1], scale_log2, -m_ref));
                        l4[e] = __fadd_rn(__fadd_rn(l4[e], p0), p1);
                        const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
                        ph[e] = __byte_perm(u0, u1, 0x7632);  // the top halves: bf16(p0) | bf16(p1) << 16, cut
                        pl[e] = bi::pack_bf16x2(__fsub_rn(p0, __uint_as_float(u0 & 0xFFFF0000u)),
                                                __fsub_rn(p1, __uint_as_float(u1 & 0xFFFF0000u)));
                    }
                    const int ch = part * (KEYS_PER / 8) + cc;  // 16-byte chunk (8 keys) of the row
                    const uint32_t off = row_off + ((uint32_t)(ch ^ (r & 7)) << 4);
                    st_shared_v4(sPh + off, ph[0], ph[1], ph[2], ph[3]);
                    st_shared_v4(sPl + off, pl[0], pl[1], pl[2], pl[3]);
                }
                l = __fadd_rn(l, __fadd_rn(__fadd_rn(l4[0], l4[1]), __fadd_rn(l4[2], l4[3])));
                // values past the tile's last position (another sequence's rows, or never written) are
                // zeroed, so that a zero P never meets a non-finite V; part p clears 64 of the row's 256 bytes
                if (j * KB + KB - 1 > it.last_pos && r < KB && j * KB + r > it.last_pos) {
                    const uint32_t s = b % NST;
                    // the stage's copy completed before S_j was issued; this wait makes its bytes
                    // visible to this thread before they are overwritten
                    if (mbar_wait(smem_u32(&bars->kv_full[s]), (b / NST) & 1u, abort)) {
                        const uint32_t v0 = sV + (uint32_t)s * KV_BLOCK + (uint32_t)(part >> 1) * KV_BOX + (uint32_t)r * 128u +
                                            (uint32_t)(part & 1) * 64u;
    #pragma unroll
                        for (int q = 0; q < 4; ++q) st_shared_v4(v0 + q * 16, 0u, 0u, 0u, 0u);
                    } else {
                        fail(err, abort, bi::DEVERR_WAIT_FULL);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->p_full));
            }
            // ---------------------------------------------------------------- epilogue: out = O / l
            if (ok) {  // the row sum: the parts' sums added in part order
                bars->xsum[part][r] = l;
                __threadfence_block();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->xchg));
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->xchg), xc & 1u, abort));
                ++xc;
                if (!ok && lane == 0) fail(err, abort, bi::DEVERR_WAIT_CLUSTER);
                l = bars->xsum[0][r];
    #pragma unroll
                for (int q = 1; q < PARTS; ++q) l = __fadd_rn(l, bars->xsum[q][r]);
            }
            if (ok) {
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->o_full), n & 1u, abort));
                if (!ok && lane == 0) fail(err, abort, bi::DEVERR_WAIT_ACCUM);
            }
            if (ok) {
                tc_fence_after();
                const float inv_l = __frcp_rn(l);  // out = O * (1 / l), one reciprocal per row
                __nv_bfloat16* dst = out + (int64_t)(it.q_row0 + r) * ldo + (int64_t)it.h * D + part * DIMS_PER;
                uint32_t o[32];
                tmem_ld_32x32b_x32(tmem + lane_off + O_COL + (uint32_t)(part * DIMS_PER), o);
                tmem_wait_ld();
                if (live) {
                    uint32_t pk[16];
    #pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = bi::pack_bf16x2(__fmul_rn(__uint_as_float(o[2 * i]), inv_l),
                                                __fmul_rn(__uint_as_float(o[2 * i + 1]), inv_l));
    #pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        *reinterpret_cast<uint4*>(dst + 2 * i) = make_uint4(pk[i], pk[i + 1], pk[i + 2], pk[i + 3]);
                }
            }
            gb += (uint32_t)it.nb;
            ++n;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// The kernel's shared-memory size is set once per device; returns the device's SM count (0 on failure).
int ensure_attr() {
    static std::once_flag once[64];
    static int sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::call_once(once[dev], [&] {
        int n = 0;
        if (cudaFuncSetAttribute(prefill_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            sms[dev] = n;
    });
    return sms[dev];
}

}  // namespace

BI_API int bi_prefill_attn(const void* q, int64_t ldq, int64_t q_rows, const void* k_cache, const void* v_cache,
                           int64_t cache_tokens, const int32_t* q_indptr, const int32_t* q_tile_indptr,
                           int32_t n_tiles, const int32_t* kv_indptr, const int32_t* q_pos0, int32_t B, int32_t Hq,
                           int32_t Hkv, int32_t head_dim, float scale, void* out, int64_t ldo, void* stream) {
    if (B < 0 || n_tiles < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || q_rows < 0 || cache_tokens <= 0)
        return BI_ERR_INVALID_ARG;
    if (head_dim != D) return BI_ERR_UNSUPPORTED_SHAPE;
    if (B == 0 || n_tiles == 0 || q_rows == 0) return BI_OK;
    if (!q || !k_cache || !v_cache || !q_indptr || !q_tile_indptr || !kv_indptr || !q_pos0 || !out)
        return BI_ERR_INVALID_ARG;
    if (ldq < (int64_t)Hq * D || ldo < (int64_t)Hq * D) return BI_ERR_INVALID_ARG;
    if (!bi::aligned16(q) || !bi::aligned16(k_cache) || !bi::aligned16(v_cache) || !bi::aligned16(out) ||
        ldq % 8 != 0 || ldo % 8 != 0)
        return BI_ERR_MISALIGNED;
    if (q_rows > 0x7fffffffLL || cache_tokens > 0x7fffffffLL || Hq > 65535) return BI_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)n_tiles * Hq > 0x7fffffffLL) return BI_ERR_UNSUPPORTED_SHAPE;
    uint32_t* err = bi::device_error_word();
    const int sms = ensure_attr();
    if (!err || sms <= 0) return BI_ERR_CUDA;
    CUtensorMap tmQ, tmK, tmV;
    const uint64_t kv_row = (uint64_t)Hkv * D;
    if (!bi::make_tmap_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, (uint64_t)Hq * D, (uint64_t)q_rows,
                          (uint64_t)ldq * 2, 64, QT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !bi::make_tmap_2d(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k_cache, kv_row, (uint64_t)cache_tokens, kv_row * 2,
                          64, KB, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !bi::make_tmap_2d(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v_cache, kv_row, (uint64_t)cache_tokens, kv_row * 2,
                          64, KB, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    // persistent CTAs, one per SM, walking the (tile, head) items
    const int64_t n_items = (int64_t)n_tiles * Hq;
    const dim3 grid((unsigned)(n_items < sms ? n_items : sms));
    if (bi::launch_pdl(prefill_attn_tc_kernel, grid, dim3(THREADS), SMEM_BYTES, bi::as_stream(stream), 0u, tmQ, tmK,
                       tmV, q_indptr, q_tile_indptr, kv_indptr, q_pos0, B, Hq, Hkv, (int)q_rows, (int)cache_tokens,
                       n_tiles, (float)((double)scale * 1.4426950408889634), static_cast<__nv_bfloat16*>(out), ldo,
                       err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}
