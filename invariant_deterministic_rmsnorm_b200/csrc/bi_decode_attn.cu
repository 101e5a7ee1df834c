// bi_decode_attn.cu -- batch-invariant split-KV decode attention with a fixed split size.
//
// Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section "Attention".
// Split-KV (FlashDecoding) stays batch-invariant if the split size is fixed instead of the
// number of splits.  The key/value cache and new tokens must share one consistent layout.
//
// Layout: q [B, Hq, D]; k, v packed [T, Hkv, D] (bf16).  Sequence b owns tokens
// kv_indptr[b] .. kv_indptr[b] + kv_len[b] - 1 of the packed buffer.  kv_indptr[b] must be
// a multiple of the chunk size, so every request's chunks start at its own token 0 and
// never depend on its neighbours.  Query head h reads kv head h / (Hq / Hkv).
//
// Phase 1 (persistent CTAs over the live work items (sequence, chunk, kv head)).  Chunk c of
// sequence b is its tokens [c*256, min(c*256 + 256, L)).  The items are counted on the device
// from kv_indptr and kv_len and cut into one contiguous range per CTA, so a small batch in a
// large cache still spreads over every SM.  For each item the CTA computes, for the group's
// query heads:
//     s_j = scale * q . k_j          (mma.sync m16n8k16: bf16 products, fp32 accumulate)
//     m_c = max_j s_j                (exact; order-free)
//     p_j = exp(s_j - m_c),  l_c = sum_j p_j     (fixed shuffle / shared-memory trees)
//     o_c = sum_j p_j v_j            (fp32 FMAs, fixed token order per thread, fixed tree)
// and stores (o_c, m_c, l_c) to the workspace row of cache slot kv_indptr[b] / 256 + c.  K and
// V reach shared memory through TMA, 128B-swizzled.  V reuses K's buffer once the scores are
// done.
//
// Phase 2 (one warp per (sequence, query head)) merges chunks c = 0, 1, ... in order:
//     m' = max(m, m_c);  l = l e^(m - m') + l_c e^(m_c - m');  o = o e^(m - m') + o_c e^(m_c - m')
// and writes out = o / l.  The arithmetic of request b depends only on its own query, keys
// and values.  The chunk size fixes every split.
#include <mutex>

#include "bi_common.cuh"
#include "bi_sm100.cuh"
#include "bi_tma_host.cuh"

using namespace bi::sm100;

namespace {

constexpr int D = 128;
constexpr int CHUNK = 256;
constexpr int CWARPS = 8;                    // compute warps
constexpr int CTHREADS = CWARPS * 32;        // 256
constexpr int THREADS = CTHREADS + 32;       // + one producer warp
constexpr int SUB = 128;                     // tokens per pipeline stage
constexpr int BOX_TOK = 64;                  // tokens per TMA box
constexpr int BOX_BYTES = BOX_TOK * 64 * 2;  // 64 tokens x 64 dims (one 128-byte half row) = 8 KB
constexpr int STAGE_BYTES = SUB * D * 2;     // 32 KB
constexpr int NSTAGES = 3;

using bi::DEVERR_BAD_LAYOUT;

constexpr int P_PITCH = CHUNK + 8;  // bf16 per head row of the split probabilities (+8: no bank conflicts)

template <int G>
struct AttnLayout {
    static constexpr int S_OFF = NSTAGES * STAGE_BYTES;         // scores [CHUNK][G] fp32
    static constexpr int P_OFF = S_OFF + CHUNK * G * 4;         // p_hi, p_lo: bf16 [8 heads][P_PITCH] each
    static constexpr int P_BYTES = 8 * P_PITCH * 2;
    static constexpr int STAT_OFF = P_OFF + 2 * P_BYTES;        // per-warp partial max / sum [8][G] x 2
    static constexpr int Q_OFF = STAT_OFF + 2 * CWARPS * G * 4;       // per stage: the item's queries, bf16 [G][D]
    static constexpr int Q_BYTES = G * D * 2;
    static constexpr int BAR_OFF = Q_OFF + NSTAGES * Q_BYTES;
    static constexpr size_t BYTES = 1024 + BAR_OFF + 2 * NSTAGES * 8 + 16;
};

// smem address of (token j of a stage, dim d) in a 128B-swizzled stage
__device__ __forceinline__ uint32_t kv_addr(uint32_t stage, int j, int d) {
    const uint32_t box = (uint32_t)((j >> 6) * 2 + (d >> 6));
    return swz(stage + box * BOX_BYTES + (uint32_t)(j & 63) * 128 + (uint32_t)(d & 63) * 2, 7u);
}

__device__ __forceinline__ void compute_barrier() { asm volatile("bar.sync 1, %0;" :: "n"(CTHREADS) : "memory"); }

// Live chunks of sequence b: ceil(len / CH) when its layout is valid, else 0 and *bad.  A
// sequence whose capacity reaches past the cache's T tokens is refused whole, so that the merge
// never reads a slot this phase did not write.
template <int CH>
__device__ __forceinline__ int live_chunks(const int32_t* __restrict__ kv_indptr, const int32_t* __restrict__ kv_len,
                                           int b, int64_t T, bool* bad) {
    const int64_t lo = kv_indptr[b], hi = kv_indptr[b + 1];
    const int len = kv_len[b];
    *bad = lo < 0 || (lo % CHUNK) != 0 || len <= 0 || (int64_t)len > hi - lo || hi > T;
    return *bad ? 0 : (len + CH - 1) / CH;
}

// Block-wide sums and scans of 64-bit counts (every thread of the block calls them).
__device__ __forceinline__ int64_t block_sum(int64_t v, int64_t* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    __syncthreads();  // the scratch may still be read by a previous call
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    int64_t t = 0;
    for (int w = 0; w < nw; ++w) t += scratch[w];
    return t;
}
// inclusive prefix of v over the threads in order; *total is the block's sum
__device__ __forceinline__ int64_t block_scan(int64_t v, int64_t* scratch, int64_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int64_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    __syncthreads();
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    int64_t before = 0, t = 0;
    for (int w = 0; w < nw; ++w) {
        if (w < warp) before += scratch[w];
        t += scratch[w];
    }
    *total = t;
    return before + x;
}

// Walks a CTA's contiguous range of work items in order.  Item order: sequences in order, the
// live chunks of each in order, the kv heads of each chunk in order.  Empty and invalid
// sequences hold no items.  Which CTA computes an item never changes how it is computed.
template <int CH>
struct WorkCursor {
    const int32_t* kv_indptr;
    const int32_t* kv_len;
    int B;
    int64_t T;
    int Hkv;
    int b, c, g, nc, len;
    int64_t lo;

    __device__ __forceinline__ void load() {
        bool bad;
        nc = live_chunks<CH>(kv_indptr, kv_len, b, T, &bad);
        lo = kv_indptr[b];
        len = kv_len[b];
    }
    __device__ __forceinline__ void start(int b0, int c0, int g0) {
        b = b0;
        c = c0;
        g = g0;
        load();
    }
    __device__ __forceinline__ int64_t tok0() const { return lo + (int64_t)c * CH; }
    __device__ __forceinline__ int n_tok() const { return min(CH, len - c * CH); }
    __device__ __forceinline__ void next() {
        if (++g < Hkv) return;
        g = 0;
        if (++c < nc) return;
        c = 0;
        do {
            if (++b >= B) return;
            load();
        } while (nc == 0);
    }
};

// Phase 1, persistent: the batch's live work items, (sequence, chunk, kv head) in that order,
// are cut into one contiguous range per CTA.  Every CTA counts them itself from kv_indptr and
// kv_len, so the cut follows the tokens the batch holds, not the capacity of the cache.
// A producer warp streams each item's K sub-blocks, then its V sub-blocks, through an NSTAGES ring;
// eight compute warps consume them in the same order.
template <int G, int CH>
__global__ void __launch_bounds__(THREADS, 2)
decode_attn_chunk_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ kv_indptr,
                         const int32_t* __restrict__ kv_len, int B, int64_t T, int Hq, int Hkv,
                         float scale, float* __restrict__ o_part, float* __restrict__ ml_part, uint32_t* err) {
    using L = AttnLayout<G>;
    __shared__ int64_t s_scan[THREADS / 32];
    __shared__ int s_first[2];  // sequence and chunk of this CTA's first item
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* sS = reinterpret_cast<float*>(base + L::S_OFF);
    __nv_bfloat16* sPh = reinterpret_cast<__nv_bfloat16*>(base + L::P_OFF);
    __nv_bfloat16* sPl = reinterpret_cast<__nv_bfloat16*>(base + L::P_OFF + L::P_BYTES);
    float* sMax = reinterpret_cast<float*>(base + L::STAT_OFF);
    float* sSum = sMax + CWARPS * G;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L::BAR_OFF);
    uint64_t* empty = full + NSTAGES;
    volatile int* abort = reinterpret_cast<volatile int*>(empty + NSTAGES);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t stage0 = smem_u32(base);
    if (tid == 0) {
        for (int i = 0; i < NSTAGES; ++i) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), CWARPS);
        }
        *abort = 0;
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    __syncthreads();
    pdl_wait();  // q, the cache and the index arrays may come from the kernels just before this one
    pdl_trigger();

    // ---- this CTA's range of the live work items
    // live chunks of every sequence; a decreasing kv_indptr (overlapping sequences) is refused
    int64_t mine = 0;
    int nc_mine = 0;  // sequence tid's live chunks (used when the batch fits one pass)
    bool order_ok = true;
    for (int b = tid; b < B; b += THREADS) {
        bool bad;
        const int nc = live_chunks<CH>(kv_indptr, kv_len, b, T, &bad);
        if (bad && blockIdx.x == 0) atomicOr(err, DEVERR_BAD_LAYOUT);
        order_ok = order_ok && kv_indptr[b + 1] >= kv_indptr[b];
        mine += nc;
        if (b == tid) nc_mine = nc;
    }
    const bool ordered = __syncthreads_and(order_ok) != 0;
    if (!ordered && blockIdx.x == 0 && tid == 0) atomicOr(err, DEVERR_BAD_LAYOUT);
    const int64_t n_items = ordered ? block_sum(mine, s_scan) * Hkv : 0;
    const int64_t per_cta = (n_items + gridDim.x - 1) / gridDim.x;
    const int64_t w_begin = min(n_items, (int64_t)blockIdx.x * per_cta);
    const int64_t w_end = min(n_items, w_begin + per_cta);
    if (w_begin < w_end) {  // uniform across the CTA
        const int64_t j0 = w_begin / Hkv;  // the first item's place among the live chunks
        int64_t before = 0;                // live chunks of the sequences before this pass
        for (int t0 = 0; t0 < B; t0 += THREADS) {
            const int b = t0 + tid;
            int nc = nc_mine;
            if (t0 != 0) {
                bool bad;
                nc = b < B ? live_chunks<CH>(kv_indptr, kv_len, b, T, &bad) : 0;
            }
            int64_t pass_total;
            const int64_t excl = before + block_scan(nc, s_scan, &pass_total) - nc;
            if (nc > 0 && excl <= j0 && j0 < excl + nc) {
                s_first[0] = b;
                s_first[1] = (int)(j0 - excl);
            }
            before += pass_total;
            if (before > j0) break;
        }
        __syncthreads();
    }
    WorkCursor<CH> cur{kv_indptr, kv_len, B, T, Hkv, 0, 0, 0, 0, 0, 0};
    if (w_begin < w_end) cur.start(s_first[0], s_first[1], (int)(w_begin % Hkv));

    if (warp == CWARPS) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            uint32_t it = 0;
            for (int64_t w = w_begin; w < w_end && !*abort; ++w, cur.next()) {
                const int g = cur.g, n_tok = cur.n_tok();
                const int64_t tok0 = cur.tok0();
                const int nsub = (n_tok + SUB - 1) / SUB;
                for (int pass = 0; pass < 2 && !*abort; ++pass) {
                    const CUtensorMap* tm = pass == 0 ? &tmK : &tmV;
                    for (int sb = 0; sb < nsub; ++sb, ++it) {
                        const int st = it % NSTAGES;
                        if (!mbar_wait(smem_u32(&empty[st]), ((it / NSTAGES) & 1u) ^ 1u, abort)) {
                            atomicOr(err, bi::DEVERR_WAIT_TMA);
                            *abort = 1;
                            break;
                        }
                        const int live = min(SUB, n_tok - sb * SUB);
                        const int ngrp = (live + BOX_TOK - 1) / BOX_TOK;
                        const uint32_t fb = smem_u32(&full[st]);
                        const bool with_q = pass == 0 && sb == 0;  // the item's queries ride on its first stage
                        mbar_arrive_expect_tx(fb, (uint32_t)(ngrp * 2 * BOX_BYTES + (with_q ? L::Q_BYTES : 0)));
                        if (with_q)
                            bulk_load(smem_u32(base + L::Q_OFF + st * L::Q_BYTES),
                                      q + ((int64_t)cur.b * Hq + (int64_t)g * G) * D, L::Q_BYTES, fb);
                        const uint32_t dst = stage0 + st * STAGE_BYTES;
                        for (int tg = 0; tg < ngrp; ++tg)
                            for (int hf = 0; hf < 2; ++hf)
                                tma_load_2d(dst + (tg * 2 + hf) * BOX_BYTES, tm, g * D + hf * 64,
                                            (int)(tok0 + sb * SUB + tg * BOX_TOK), fb);
                    }
                }
            }
            if (*abort) {
                for (uint32_t i = it > (uint32_t)NSTAGES ? it - NSTAGES : 0u; i < it; ++i)
                    (void)mbar_wait(smem_u32(&full[i % NSTAGES]), (i / NSTAGES) & 1u, nullptr);
            }
        }
        return;
    }

    // ---------------------------------------------------- compute warps
    uint32_t it = 0;
    for (int64_t w = w_begin; w < w_end; ++w, cur.next()) {
        const int g = cur.g, n_tok = cur.n_tok();
        const int64_t slot = cur.tok0() / CH;  // the item's row of the partials
        const int nsub = (n_tok + SUB - 1) / SUB;

        // ---- scores: in stage sb, warp w owns the 16 tokens [16 w, 16 w + 16)
        bool ok = true;
        uint32_t qf[8][2];
        for (int sb = 0; sb < 2; ++sb) {
            const int t0 = sb * SUB + warp * 16;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (sb < nsub) {
                const int st = it % NSTAGES;
                const bool w_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), (it / NSTAGES) & 1u, abort));
                if (!w_ok) {
                    ok = false;
                    if (lane == 0) {
                        atomicOr(err, bi::DEVERR_WAIT_FULL);
                        *abort = 1;
                    }
                }
                if (sb == 0) {
                    // query fragments from the first stage's query slot (B operand, [16 dims x 8 heads]
                    // per k-step; heads >= G are zero)
                    const int hh = lane >> 2, dq = (lane & 3) * 2;
                    const uint32_t qs = smem_u32(base + L::Q_OFF + st * L::Q_BYTES) + (uint32_t)(hh < G ? hh : 0) * D * 2;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        uint32_t v0 = 0u, v1 = 0u;
                        if (hh < G && w_ok) {
                            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v0) : "r"(qs + (kk * 16 + dq) * 2));
                            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v1) : "r"(qs + (kk * 16 + dq + 8) * 2));
                        }
                        qf[kk][0] = v0;
                        qf[kk][1] = v1;
                    }
                }
                if (w_ok && t0 < n_tok) {
                    const uint32_t sbase = stage0 + st * STAGE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        uint32_t a[4];
                        ldmatrix_x4(kv_addr(sbase, warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8), a);
                        mma_m16n8k16_bf16(acc, a, qf[kk]);
                    }
                }
                release_stage(smem_u32(&empty[st]), lane);
                ++it;
            }
            const int gg = lane >> 2, hq = (lane & 3) * 2;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = t0 + gg + (e >> 1) * 8;
                const int h = hq + (e & 1);
                if (h < G) sS[j * G + h] = (j < n_tok) ? __fmul_rn(acc[e], scale) : -INFINITY;
            }
        }
        // A failed wait never changes the control flow: every compute warp keeps meeting the same
        // named barriers, the abort flag makes the remaining waits return at once, and the
        // kernel runs to its end with the error recorded.
        (void)ok;
        compute_barrier();

        // ---- softmax statistics over the chunk (thread tid owns token tid)
        float sv[G], p[G], mc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) sv[h] = sS[tid * G + h];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float m = sv[h];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            if (lane == 0) sMax[warp * G + h] = m;
        }
        compute_barrier();
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            if (h < G) {
                float m = sMax[h];
#pragma unroll
                for (int ww = 1; ww < CWARPS; ++ww) m = fmaxf(m, sMax[ww * G + h]);
                mc[h] = m;
                p[h] = (tid < n_tok) ? expf(__fsub_rn(sv[h], m)) : 0.0f;
                // p = hi + lo + r with hi, lo bf16 and |r| <= 2^-18 |p|: the tensor-core PV below
                // multiplies the exact bf16 values of V by hi and by lo and adds both in fp32
                const __nv_bfloat16 hi = __float2bfloat16_rn(p[h]);
                const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(p[h], __bfloat162float(hi)));
                sPh[h * P_PITCH + tid] = hi;
                sPl[h * P_PITCH + tid] = lo;
                float sum = p[h];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, off));
                if (lane == 0) sSum[warp * G + h] = sum;
            } else {  // heads past the group: zero columns of the MMA's B operand
                sPh[h * P_PITCH + tid] = __float2bfloat16_rn(0.0f);
                sPl[h * P_PITCH + tid] = __float2bfloat16_rn(0.0f);
            }
        }
        compute_barrier();

        // ---- o_c = sum_j p_j v_j on tensor cores: warp w owns dims [16 w, 16 w + 16) for all 8
        // (padded) heads: O^T[dims x heads] += V^T[dims x 16 tokens] . P[16 tokens x heads], tokens in
        // ascending 16-token steps, the hi then the lo part of P at each step.
        // two independent chains (the hi and the lo part of P), added once at the end
        float oacc[4] = {0.f, 0.f, 0.f, 0.f}, oacc_lo[4] = {0.f, 0.f, 0.f, 0.f};
        const int gq = lane >> 2, cq = lane & 3;
        const uint32_t ph = smem_u32(sPh) + (uint32_t)(gq * P_PITCH + 2 * cq) * 2;
        const uint32_t pl = smem_u32(sPl) + (uint32_t)(gq * P_PITCH + 2 * cq) * 2;
        for (int sb = 0; sb < nsub; ++sb) {
            const int st = it % NSTAGES;
            const bool w_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&full[st]), (it / NSTAGES) & 1u, abort));
            if (!w_ok && lane == 0) {
                atomicOr(err, bi::DEVERR_WAIT_FULL);
                *abort = 1;
            }
            if (w_ok) {
                const uint32_t sbase = stage0 + st * STAGE_BYTES;
                const int live = min(SUB, n_tok - sb * SUB);
                for (int ks = 0; ks * 16 < live; ++ks) {
                    uint32_t a[4];
                    // matrix i = lane / 8: tokens +8 * (i >> 1), dims +8 * (i & 1)
                    const int mi = lane >> 3;
                    ldmatrix_x4_trans(kv_addr(sbase, ks * 16 + (lane & 7) + 8 * (mi >> 1), warp * 16 + 8 * (mi & 1)), a);
                    if (ks * 16 + 16 > live) {  // last, partial step: tokens past the end may hold anything
                        const int t_lo = ks * 16 + 2 * cq;  // tokens of a0/a1 (and +8 for a2/a3)
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int t = t_lo + (r >> 1) * 8;
                            uint32_t m = 0u;
                            if (t < live) m |= 0x0000FFFFu;
                            if (t + 1 < live) m |= 0xFFFF0000u;
                            a[r] &= m;
                        }
                    }
                    const int j0 = sb * SUB + ks * 16;  // token of the chunk at the start of this step
                    uint32_t bh[2], bl[2];
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bh[0]) : "r"(ph + j0 * 2));
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bh[1]) : "r"(ph + (j0 + 8) * 2));
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bl[0]) : "r"(pl + j0 * 2));
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bl[1]) : "r"(pl + (j0 + 8) * 2));
                    mma_m16n8k16_bf16(oacc, a, bh);
                    mma_m16n8k16_bf16(oacc_lo, a, bl);
                }
            }
            release_stage(smem_u32(&empty[st]), lane);
            ++it;
        }

        // oacc: (dim 16w + gq, heads 2cq, 2cq+1) and (dim 16w + gq + 8, same heads)
        const int hq0 = g * G;
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[e] = __fadd_rn(oacc[e], oacc_lo[e]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int h = 2 * cq + (e & 1);
            const int d = warp * 16 + gq + (e >> 1) * 8;
            if (h < G) o_part[((int64_t)slot * Hq + hq0 + h) * D + d] = oacc[e];
        }
        if (tid < G) {
            float l = sSum[tid];
#pragma unroll
            for (int ww = 1; ww < CWARPS; ++ww) l = __fadd_rn(l, sSum[ww * G + tid]);
            // mc[] is uniform across threads; select this head's value without dynamic register indexing
            float m_sel = mc[0];
#pragma unroll
            for (int h = 1; h < G; ++h)
                if (tid == h) m_sel = mc[h];
            *reinterpret_cast<float2*>(ml_part + ((int64_t)slot * Hq + hq0 + tid) * 2) = make_float2(m_sel, l);
        }
        compute_barrier();  // scores, probabilities and statistics are reused by the next item
    }
}

// Phase 2: one warp per (sequence, query head); lane owns dims [4*lane, 4*lane + 4).
template <bool OUT_BF16, int CH>
__global__ void __launch_bounds__(128)
decode_attn_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ ml_part,
                         const int32_t* __restrict__ kv_indptr, const int32_t* __restrict__ kv_len, int64_t T,
                         int Hq, void* __restrict__ out, uint32_t* err) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x * 4 + warp;
    const int b = blockIdx.y;
    pdl_wait();  // the partials come from phase 1, launched just before
    pdl_trigger();
    if (h >= Hq) return;
    const int64_t sbase = kv_indptr[b];
    const int len = kv_len[b];
    const int64_t cap = (int64_t)kv_indptr[b + 1] - sbase;
    // the same checks as phase 1: a sequence past the cache's T tokens has no partials to merge
    if (sbase < 0 || (sbase % CHUNK) != 0 || len <= 0 || (int64_t)len > cap || (int64_t)kv_indptr[b + 1] > T) {
        if (lane == 0) atomicOr(err, DEVERR_BAD_LAYOUT);  // out row left unwritten
        return;
    }
    const int nch = (len + CH - 1) / CH;
    const int64_t slot0 = sbase / CH;
    float m = -INFINITY, l = 0.0f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    // The merge is sequential in c; the loads are not.  Two register buffers of PF chunks: the
    // loads of the next PF chunks are in flight while the current PF are merged, in order.
    constexpr int PF = 8;
    float2 mlA[PF], mlB[PF];
    float4 oA[PF], oB[PF];
    auto fetch = [&](int c0, float2 (&ml)[PF], float4 (&ov)[PF]) {
#pragma unroll
        for (int i = 0; i < PF; ++i) {
            if (c0 + i < nch) {
                const int64_t idx = (slot0 + c0 + i) * Hq + h;
                ml[i] = *reinterpret_cast<const float2*>(ml_part + idx * 2);
                ov[i] = *reinterpret_cast<const float4*>(o_part + idx * D + lane * 4);
            }
        }
    };
    auto merge = [&](int c0, const float2 (&ml)[PF], const float4 (&ov)[PF]) {
#pragma unroll
        for (int i = 0; i < PF; ++i) {
            if (c0 + i < nch) {
                const float mn = fmaxf(m, ml[i].x);
                const float a = expf(__fsub_rn(m, mn));   // 0 on the first chunk (m = -inf)
                const float bsc = expf(__fsub_rn(ml[i].x, mn));
                l = __fmaf_rn(l, a, __fmul_rn(ml[i].y, bsc));
                o.x = __fmaf_rn(o.x, a, __fmul_rn(ov[i].x, bsc));
                o.y = __fmaf_rn(o.y, a, __fmul_rn(ov[i].y, bsc));
                o.z = __fmaf_rn(o.z, a, __fmul_rn(ov[i].z, bsc));
                o.w = __fmaf_rn(o.w, a, __fmul_rn(ov[i].w, bsc));
                m = mn;
            }
        }
    };
    fetch(0, mlA, oA);
    for (int c0 = 0; c0 < nch; c0 += 2 * PF) {
        fetch(c0 + PF, mlB, oB);
        merge(c0, mlA, oA);
        fetch(c0 + 2 * PF, mlA, oA);
        merge(c0 + PF, mlB, oB);
    }
    const float r0 = __fdiv_rn(o.x, l), r1 = __fdiv_rn(o.y, l), r2 = __fdiv_rn(o.z, l), r3 = __fdiv_rn(o.w, l);
    const int64_t off = ((int64_t)b * Hq + h) * D + lane * 4;
    if constexpr (OUT_BF16) {
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + off) =
            make_uint2(bi::pack_bf16x2(r0, r1), bi::pack_bf16x2(r2, r3));
    } else {
        *reinterpret_cast<float4*>(static_cast<float*>(out) + off) = make_float4(r0, r1, r2, r3);
    }
}

// Phase 2 on `s`, allowed to start while phase 1 finishes (it waits for phase 1 before it reads).
template <typename K, typename... Args>
void launch_merge(K kernel, dim3 grid, cudaStream_t s, Args... args) {
    (void)bi::launch_pdl(kernel, grid, dim3(128), 0, s, 0u, args...);
}

template <typename F>
bool set_smem_once(F kernel, size_t bytes) {
    static std::mutex mu;
    static const void* done_k[64];
    static int done_d[64];
    static int n = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (done_k[i] == (const void*)kernel && done_d[i] == dev) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    if (n < 64) {
        done_k[n] = (const void*)kernel;
        done_d[n] = dev;
        ++n;
    }
    return true;
}

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

size_t partial_bytes(int64_t total_tokens, int32_t Hq, int ch = CHUNK) {
    const int64_t slots = (total_tokens + ch - 1) / ch;
    return (size_t)slots * Hq * (D + 2) * sizeof(float);
}

template <int G, int CH = CHUNK>
int launch_chunks(const void* q, const void* k, const void* v, const int32_t* kv_indptr, const int32_t* kv_len,
                  int B, int64_t T, int Hq, int Hkv, float scale, float* o_part, float* ml_part, cudaStream_t s) {
    using L = AttnLayout<G>;
    uint32_t* err = bi::device_error_word();
    auto kern = decode_attn_chunk_kernel<G, CH>;
    if (!err || !set_smem_once(kern, L::BYTES)) return BI_ERR_CUDA;
    CUtensorMap tmK, tmV;
    const uint64_t row = (uint64_t)Hkv * D;  // elements per packed token
    if (!bi::make_tmap_2d(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, row, (uint64_t)T, row * 2, 64, BOX_TOK,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
        !bi::make_tmap_2d(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, row, (uint64_t)T, row * 2, 64, BOX_TOK,
                          CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    // the live items (counted on the device) are at most one per (CH-token slot of the cache, kv head)
    const int64_t items = ((T + CH - 1) / CH) * Hkv;
    const int sms = num_sms();
    if (sms <= 0) return BI_ERR_CUDA;
    const int64_t ctas = 2LL * sms;  // two persistent CTAs per SM: one computes while the other waits
    dim3 grid((unsigned)(items < ctas ? items : ctas));
    if (bi::launch_pdl(kern, grid, dim3(THREADS), L::BYTES, s, 0u, tmK, tmV, static_cast<const __nv_bfloat16*>(q),
                       kv_indptr, kv_len, B, T, Hq, Hkv, scale, o_part, ml_part, err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

}  // namespace

BI_API size_t bi_decode_attn_workspace_size(int64_t total_tokens, int32_t Hq, int32_t head_dim, int32_t chunk) {
    if (total_tokens <= 0 || Hq <= 0 || head_dim != D || chunk != CHUNK) return 0;
    return partial_bytes(total_tokens, Hq);
}

BI_API int bi_decode_attn(const void* q, const void* k, const void* v, const int32_t* kv_indptr, const int32_t* kv_len,
                          int32_t B, int64_t total_tokens, int32_t Hq, int32_t Hkv, int32_t head_dim, float scale,
                          int32_t chunk, void* out, int out_dtype, void* ws, size_t ws_bytes, void* stream) {
    if (out_dtype != BI_F32 && out_dtype != BI_BF16) return BI_ERR_INVALID_ARG;
    if (B < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0 || !(scale == scale)) return BI_ERR_INVALID_ARG;
    if (head_dim != D || chunk != CHUNK || Hq % Hkv != 0) return BI_ERR_UNSUPPORTED_SHAPE;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return BI_ERR_UNSUPPORTED_SHAPE;
    if (B == 0) return BI_OK;
    if (total_tokens == 0) return BI_ERR_INVALID_ARG;
    if (total_tokens > 0x7fffffffLL || B > 65535 || Hq > 4096) return BI_ERR_UNSUPPORTED_SHAPE;
    if (!q || !k || !v || !kv_indptr || !kv_len || !out) return BI_ERR_INVALID_ARG;
    if (!bi::aligned16(q) || !bi::aligned16(k) || !bi::aligned16(v) || !bi::aligned16(out)) return BI_ERR_MISALIGNED;
    const size_t need = partial_bytes(total_tokens, Hq);
    if (!ws || ws_bytes < need || !bi::aligned16(ws)) return BI_ERR_WORKSPACE;
    float* o_part = static_cast<float*>(ws);
    const int64_t slots = (total_tokens + CHUNK - 1) / CHUNK;
    float* ml_part = o_part + (size_t)slots * Hq * D;
    cudaStream_t s = bi::as_stream(stream);
    int st;
    switch (G) {
        case 1: st = launch_chunks<1>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, o_part, ml_part, s); break;
        case 2: st = launch_chunks<2>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, o_part, ml_part, s); break;
        case 4: st = launch_chunks<4>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, o_part, ml_part, s); break;
        default: st = launch_chunks<8>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, o_part, ml_part, s); break;
    }
    if (st != BI_OK) return st;
    dim3 grid((unsigned)((Hq + 3) / 4), (unsigned)B);
    uint32_t* err = bi::device_error_word();
    if (out_dtype == BI_BF16)
        launch_merge(decode_attn_merge_kernel<true, CHUNK>, grid, s, o_part, ml_part, kv_indptr, kv_len,
                     total_tokens, Hq, out, err);
    else
        launch_merge(decode_attn_merge_kernel<false, CHUNK>, grid, s, o_part, ml_part, kv_indptr, kv_len,
                     total_tokens, Hq, out, err);
    return bi::launch_status();
}

// ------------------------------------------------------------------ no-allocation variant
//
// Some callers cannot allocate device memory at all.  Examples: a plugin interface
// that hands a kernel only its input and output buffers and offers no allocator; a
// serving process whose memory pool already owns all of the GPU's free memory; a
// latency-critical loop where cudaMalloc's implicit device synchronisation is not
// acceptable.  bi_decode_attn_noalloc serves them.  It runs the same two kernels as
// bi_decode_attn.  Its per-chunk partials live in the fixed array below, which every
// GPU that loads this library holds until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;  // 16 MiB; mirrored in bi.h

// In host code this name is only a host-side stand-in for the symbol, not a device
// address.  Host code must use the address from cudaGetSymbolAddress (below).
static __device__ __align__(256) unsigned char g_decode_attn_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kNoAllocMaxDevices];

// Device address of the scratch array on the current device.  It is looked up with that
// device current and cached once the lookup has succeeded; a failed lookup (for instance one
// attempted inside a stream capture) caches nothing, so the next call tries again.  Returns
// nullptr if the lookup fails.
void* noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_attn_scratch) == cudaSuccess) g_scratch_ptr[dev] = p;
        else (void)cudaGetLastError();  // the failed lookup must not surface as a later launch's error
    }
    return g_scratch_ptr[dev];
}

}  // namespace

BI_API int bi_decode_attn_noalloc(const void* q, const void* k, const void* v, const int32_t* kv_indptr,
                                  const int32_t* kv_len, int32_t B, int64_t total_tokens, int32_t Hq, int32_t Hkv,
                                  int32_t head_dim, float scale, int32_t chunk, void* out, int out_dtype,
                                  void* stream) {
    if (out_dtype != BI_F32 && out_dtype != BI_BF16) return BI_ERR_INVALID_ARG;
    if (B < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0 || !(scale == scale)) return BI_ERR_INVALID_ARG;
    if (head_dim != D || chunk != CHUNK || Hq % Hkv != 0) return BI_ERR_UNSUPPORTED_SHAPE;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return BI_ERR_UNSUPPORTED_SHAPE;
    if (B == 0) return BI_OK;
    if (total_tokens == 0) return BI_ERR_INVALID_ARG;
    if (total_tokens > 0x7fffffffLL || B > 65535 || Hq > 4096) return BI_ERR_UNSUPPORTED_SHAPE;
    if (!q || !k || !v || !kv_indptr || !kv_len || !out) return BI_ERR_INVALID_ARG;
    if (!bi::aligned16(q) || !bi::aligned16(k) || !bi::aligned16(v) || !bi::aligned16(out)) return BI_ERR_MISALIGNED;
    // The partials must fit in the fixed scratch array; larger caches are refused, not truncated.
    if (partial_bytes(total_tokens, Hq) > kNoAllocScratchBytes) return BI_ERR_WORKSPACE;
    void* scratch = noalloc_scratch();
    if (!scratch) return BI_ERR_CUDA;
    // Nothing in the scratch needs to start at zero: phase 1 writes every partial that
    // phase 2 reads, and slots no sequence covers are never read.
    float* o_part = static_cast<float*>(scratch);
    const int64_t slots = (total_tokens + CHUNK - 1) / CHUNK;
    float* ml_part = o_part + (size_t)slots * Hq * D;
    cudaStream_t s = bi::as_stream(stream);
    int st;
    switch (G) {
        case 1: st = launch_chunks<1>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, o_part, ml_part, s); break;
        case 2: st = launch_chunks<2>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, o_part, ml_part, s); break;
        case 4: st = launch_chunks<4>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, o_part, ml_part, s); break;
        default: st = launch_chunks<8>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, o_part, ml_part, s); break;
    }
    if (st != BI_OK) return st;
    uint32_t* err = bi::device_error_word();
    dim3 grid((unsigned)((Hq + 3) / 4), (unsigned)B);
    if (out_dtype == BI_BF16)
        launch_merge(decode_attn_merge_kernel<true, CHUNK>, grid, s, o_part, ml_part, kv_indptr, kv_len,
                     total_tokens, Hq, out, err);
    else
        launch_merge(decode_attn_merge_kernel<false, CHUNK>, grid, s, o_part, ml_part, kv_indptr, kv_len,
                     total_tokens, Hq, out, err);
    return bi::launch_status();
}

// ------------------------------------------------------------------ comparator: batch-adaptive split
//
// What a batch-size-adaptive split-KV kernel does: when the batch is small, cut the cache into
// more, smaller chunks (128 tokens instead of 256) to fill the GPU.  A request's chunking, and
// so its merge order, then depends on how many other requests share its batch: not batch-invariant.
namespace {

template <int CH>
int run_adaptive(const void* q, const void* k, const void* v, const int32_t* kv_indptr, const int32_t* kv_len,
                 int B, int64_t T, int Hq, int Hkv, float scale, void* out, int out_dtype, float* ws, cudaStream_t s) {
    const int G = Hq / Hkv;
    const int64_t slots = (T + CH - 1) / CH;
    float* o_part = ws;
    float* ml_part = o_part + (size_t)slots * Hq * D;
    int st;
    switch (G) {
        case 1: st = launch_chunks<1, CH>(q, k, v, kv_indptr, kv_len, B, T, Hq, Hkv, scale, o_part, ml_part, s); break;
        case 2: st = launch_chunks<2, CH>(q, k, v, kv_indptr, kv_len, B, T, Hq, Hkv, scale, o_part, ml_part, s); break;
        case 4: st = launch_chunks<4, CH>(q, k, v, kv_indptr, kv_len, B, T, Hq, Hkv, scale, o_part, ml_part, s); break;
        default: st = launch_chunks<8, CH>(q, k, v, kv_indptr, kv_len, B, T, Hq, Hkv, scale, o_part, ml_part, s); break;
    }
    if (st != BI_OK) return st;
    uint32_t* err = bi::device_error_word();
    dim3 grid((unsigned)((Hq + 3) / 4), (unsigned)B);
    if (out_dtype == BI_BF16)
        launch_merge(decode_attn_merge_kernel<true, CH>, grid, s, o_part, ml_part, kv_indptr, kv_len, T, Hq,
                     out, err);
    else
        launch_merge(decode_attn_merge_kernel<false, CH>, grid, s, o_part, ml_part, kv_indptr, kv_len, T, Hq,
                     out, err);
    return bi::launch_status();
}

}  // namespace

BI_API size_t bi_ctrl_decode_attn_adaptive_workspace_size(int64_t total_tokens, int32_t Hq) {
    if (total_tokens <= 0 || Hq <= 0) return 0;
    return partial_bytes(total_tokens, Hq, 128);
}

BI_API int bi_ctrl_decode_attn_adaptive(const void* q, const void* k, const void* v, const int32_t* kv_indptr,
                                        const int32_t* kv_len, int32_t B, int64_t total_tokens, int32_t Hq,
                                        int32_t Hkv, float scale, void* out, int out_dtype, void* ws, size_t ws_bytes,
                                        void* stream) {
    if (out_dtype != BI_F32 && out_dtype != BI_BF16) return BI_ERR_INVALID_ARG;
    if (B < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return BI_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return BI_ERR_UNSUPPORTED_SHAPE;
    if (B == 0) return BI_OK;
    if (total_tokens == 0 || !q || !k || !v || !kv_indptr || !kv_len || !out) return BI_ERR_INVALID_ARG;
    if (total_tokens > 0x7fffffffLL || B > 65535) return BI_ERR_UNSUPPORTED_SHAPE;
    if (!bi::aligned16(q) || !bi::aligned16(k) || !bi::aligned16(v) || !bi::aligned16(out)) return BI_ERR_MISALIGNED;
    const int ch = B < 16 ? 128 : 256;
    if (!ws || ws_bytes < partial_bytes(total_tokens, Hq, ch) || !bi::aligned16(ws)) return BI_ERR_WORKSPACE;
    cudaStream_t s = bi::as_stream(stream);
    if (ch == 128)
        return run_adaptive<128>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, out, out_dtype,
                                 static_cast<float*>(ws), s);
    return run_adaptive<256>(q, k, v, kv_indptr, kv_len, B, total_tokens, Hq, Hkv, scale, out, out_dtype,
                             static_cast<float*>(ws), s);
}
