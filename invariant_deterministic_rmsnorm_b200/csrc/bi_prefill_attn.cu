// bi_prefill_attn.cu -- batch-invariant causal prefill attention (grouped-query, variable length).
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
// One CTA per (64-row query tile of a sequence, query head).  Each of its 4 warps owns 16
// query rows.  KV blocks of 64 positions, starting at position 0, are visited in ascending
// order.  For each block:
//   S = scale * Q K^T                  mma.sync m16n8k16, bf16 products, fp32 sums
//   causal mask, then the online softmax: m' = max(m, rowmax S);  c = e^(m - m');  P = e^(S - m')
//   l = l c + rowsum P;  O = O c + P V  (P split into bf16 hi + lo parts, both multiplied by V)
// and out = O / l rounded to bf16.  Row i's arithmetic depends only on its own sequence's query
// row, keys and values.  Blocks entirely above a row's position contribute exact zeros and
// factors of one, so the tile a row shares with other rows never changes its bits.
#include <mutex>

#include "bi_common.cuh"
#include "bi_model.h"
#include "bi_sm100.cuh"
#include "bi_tma_host.cuh"

using namespace bi::sm100;

namespace {

constexpr int D = 128;
constexpr int QT = 64;                 // query rows per CTA
constexpr int KB = 64;                 // keys per block
constexpr int THREADS = 128;           // 4 warps x 16 query rows
constexpr int HALF_BYTES = 64 * 64 * 2;  // one TMA box: 64 rows x 64 dims = 8 KB
constexpr int TILE_BYTES = 2 * HALF_BYTES;  // 64 rows x 128 dims = 16 KB
constexpr size_t SMEM_BYTES = 1024 + TILE_BYTES /*Q*/ + 2 * 2 * TILE_BYTES /*K,V x 2 stages*/ + 64;

__device__ __forceinline__ uint32_t tile_addr(uint32_t base, int row, int dim) {
    return swz(base + (uint32_t)(dim >> 6) * HALF_BYTES + (uint32_t)row * 128 + (uint32_t)(dim & 63) * 2, 7u);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return bi::pack_bf16x2(lo, hi); }

__global__ void __launch_bounds__(THREADS, 2)
prefill_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ q_indptr,
                    const int32_t* __restrict__ q_tile_indptr, const int32_t* __restrict__ kv_indptr,
                    const int32_t* __restrict__ q_pos0, int B, int Hq, int Hkv, int q_rows, int cache_tokens,
                    float scale, __nv_bfloat16* __restrict__ out, int64_t ldo, uint32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(base);
    const uint32_t sKV = sQ + TILE_BYTES;  // stage s: K at sKV + s*2*TILE, V at + TILE
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + TILE_BYTES + 4 * TILE_BYTES);  // [0] Q, [1..2] stages

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y;
    const int g = h / (Hq / Hkv);

    // the sequence that owns this tile: the last b with q_tile_indptr[b] <= tile
    int lo = 0, hi = B;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (q_tile_indptr[mid] <= tile) lo = mid; else hi = mid;
    }
    const int b = lo;
    const int qt = tile - q_tile_indptr[b];
    const int q_row0 = q_indptr[b] + qt * QT;               // first query row of the tile
    const int n_q = min(QT, q_indptr[b + 1] - q_row0);      // live query rows
    const int pos0 = q_pos0[b] + qt * QT;                   // position of the tile's first row
    const int kv_base = kv_indptr[b];
    const int last_pos = pos0 + n_q - 1;                    // highest position any live row sees
    const int n_blocks = last_pos / KB + 1;
    if (n_q <= 0) return;  // a tile index past the last sequence's tiles
    // the documented layout, checked before any copy or store: rows inside q/out, positions
    // inside the caches
    if (q_indptr[b + 1] > q_rows || q_indptr[b] < 0 || pos0 < 0 || kv_base < 0 ||
        (int64_t)kv_base + last_pos >= (int64_t)cache_tokens) {
        if (tid == 0) atomicOr(err, bi::DEVERR_BAD_PREFILL);
        return;
    }

    __shared__ int s_abort;  // set once a wait has run out: later waits give up at once, no new copies
    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&bars[i]), 1);
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    __syncthreads();
    auto issue_kv = [&](int kb) {
        const int st = kb & 1;
        const uint32_t bar = smem_u32(&bars[1 + st]);
        const uint32_t dk = sKV + st * 2 * TILE_BYTES;
        mbar_arrive_expect_tx(bar, 2 * TILE_BYTES);
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_2d(dk + hf * HALF_BYTES, &tmK, g * D + hf * 64, kv_base + kb * KB, bar);
            tma_load_2d(dk + TILE_BYTES + hf * HALF_BYTES, &tmV, g * D + hf * 64, kv_base + kb * KB, bar);
        }
    };
    if (tid == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        const uint32_t qb = smem_u32(&bars[0]);
        mbar_arrive_expect_tx(qb, TILE_BYTES);
        for (int hf = 0; hf < 2; ++hf) tma_load_2d(sQ + hf * HALF_BYTES, &tmQ, h * D + hf * 64, q_row0, qb);
        issue_kv(0);
    }

    int issued = 0;  // (thread 0) KV blocks whose copies were started
    const int gq = lane >> 2, cq = lane & 3;
    bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars[0]), 0u, &s_abort));
    if (!ok && lane == 0) {
        atomicOr(err, bi::DEVERR_WAIT_FULL);
        s_abort = 1;
    }
    uint32_t qa[8][4];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) ldmatrix_x4(tile_addr(sQ, warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8), qa[kk]);

    // this thread's two query rows and their positions
    const int qpos_a = pos0 + warp * 16 + gq, qpos_b = qpos_a + 8;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    for (int kb = 0; kb < n_blocks; ++kb) {
        // the stage of block kb + 1 was released by the barrier that ended block kb - 1
        if (tid == 0 && kb + 1 < n_blocks && *(volatile int*)&s_abort == 0) {
            issue_kv(kb + 1);
            issued = kb + 1;
        }
        const int st = kb & 1;
        const bool w_ok =
            __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars[1 + st]), (uint32_t)(kb >> 1) & 1u, &s_abort));
        if (!w_ok) {
            ok = false;
            if (lane == 0) {
                atomicOr(err, bi::DEVERR_WAIT_FULL);
                s_abort = 1;
            }
        }
        const uint32_t sK = sKV + st * 2 * TILE_BYTES, sV = sK + TILE_BYTES;
        if (w_ok) {
            // ---- S = Q K^T for this warp's 16 rows x 64 keys
            float s[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
                for (int np = 0; np < 4; ++np) {  // pairs of 8-key n-tiles
                    uint32_t bb[4];
                    const int mi = lane >> 3;
                    ldmatrix_x4(tile_addr(sK, np * 16 + (mi >> 1) * 8 + (lane & 7), kk * 16 + (mi & 1) * 8), bb);
                    const uint32_t b0[2] = {bb[0], bb[1]}, b1[2] = {bb[2], bb[3]};
                    mma_m16n8k16_bf16(s[2 * np], qa[kk], b0);
                    mma_m16n8k16_bf16(s[2 * np + 1], qa[kk], b1);
                }
            }
            // ---- scale, causal mask, online softmax (rows a = gq, b = gq + 8 of this warp)
            float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int kpos = kb * KB + nt * 8 + 2 * cq + (e & 1);
                    const int qpos = (e >> 1) ? qpos_b : qpos_a;
                    const float v = kpos <= qpos ? __fmul_rn(s[nt][e], scale) : -INFINITY;
                    s[nt][e] = v;
                }
                mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]));
                mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]));
            }
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
            const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
            // a fully masked block keeps m: the factor is exactly 1 and P is exactly 0
            const float c_a = (mn_a == -INFINITY) ? 1.f : expf(__fsub_rn(m_a, mn_a));
            const float c_b = (mn_b == -INFINITY) ? 1.f : expf(__fsub_rn(m_b, mn_b));
            float sum_a = 0.f, sum_b = 0.f;
            uint32_t pa_hi[4][4], pa_lo[4][4];  // A fragments of P for the 4 16-key steps
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                float p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float mref = (e >> 1) ? mn_b : mn_a;
                    p[e] = (s[nt][e] == -INFINITY) ? 0.f : expf(__fsub_rn(s[nt][e], mref));
                }
                sum_a = __fadd_rn(sum_a, __fadd_rn(p[0], p[1]));
                sum_b = __fadd_rn(sum_b, __fadd_rn(p[2], p[3]));
                float ph[4], pl[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    ph[e] = __bfloat162float(__float2bfloat16_rn(p[e]));
                    pl[e] = __fsub_rn(p[e], ph[e]);
                }
                const int ks = nt >> 1, half = nt & 1;  // n-tile nt covers keys 8*(nt&1) of step ks
                pa_hi[ks][half * 2 + 0] = pack2(ph[0], ph[1]);
                pa_hi[ks][half * 2 + 1] = pack2(ph[2], ph[3]);
                pa_lo[ks][half * 2 + 0] = pack2(pl[0], pl[1]);
                pa_lo[ks][half * 2 + 1] = pack2(pl[2], pl[3]);
            }
            sum_a = __fadd_rn(sum_a, __shfl_xor_sync(0xffffffffu, sum_a, 1));
            sum_a = __fadd_rn(sum_a, __shfl_xor_sync(0xffffffffu, sum_a, 2));
            sum_b = __fadd_rn(sum_b, __shfl_xor_sync(0xffffffffu, sum_b, 1));
            sum_b = __fadd_rn(sum_b, __shfl_xor_sync(0xffffffffu, sum_b, 2));
            l_a = __fmaf_rn(l_a, c_a, sum_a);
            l_b = __fmaf_rn(l_b, c_b, sum_b);
            m_a = mn_a;
            m_b = mn_b;
#pragma unroll
            for (int dt = 0; dt < 16; ++dt) {
                o[dt][0] = __fmul_rn(o[dt][0], c_a);
                o[dt][1] = __fmul_rn(o[dt][1], c_a);
                o[dt][2] = __fmul_rn(o[dt][2], c_b);
                o[dt][3] = __fmul_rn(o[dt][3], c_b);
            }
            // ---- O += P V (keys past the last live position are masked in the V fragments)
            const int key_limit = last_pos - kb * KB;  // keys j <= key_limit of this block may be read
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                // A operand: rows (gq, gq+8) x keys of step ks; registers: (row a, keys lo),
                // (row b, keys lo), (row a, keys hi), (row b, keys hi)
                const uint32_t ah[4] = {pa_hi[ks][0], pa_hi[ks][1], pa_hi[ks][2], pa_hi[ks][3]};
                const uint32_t al[4] = {pa_lo[ks][0], pa_lo[ks][1], pa_lo[ks][2], pa_lo[ks][3]};
#pragma unroll
                for (int dp = 0; dp < 8; ++dp) {  // pairs of 8-dim n-tiles
                    uint32_t vb[4];
                    const int mi = lane >> 3;
                    ldmatrix_x4_trans(tile_addr(sV, ks * 16 + (lane & 7) + (mi & 1) * 8, dp * 16 + (mi >> 1) * 8), vb);
                    if (ks * 16 + 15 > key_limit) {
                        // keys 2cq, 2cq+1 (+8) of this step: zero the halves past the limit
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int kj = ks * 16 + 2 * cq + (r & 1) * 8;
                            uint32_t m = 0u;
                            if (kj <= key_limit) m |= 0x0000FFFFu;
                            if (kj + 1 <= key_limit) m |= 0xFFFF0000u;
                            vb[r] &= m;
                        }
                    }
                    const uint32_t v0[2] = {vb[0], vb[1]}, v1[2] = {vb[2], vb[3]};
                    mma_m16n8k16_bf16(o[2 * dp], ah, v0);
                    mma_m16n8k16_bf16(o[2 * dp], al, v0);
                    mma_m16n8k16_bf16(o[2 * dp + 1], ah, v1);
                    mma_m16n8k16_bf16(o[2 * dp + 1], al, v1);
                }
            }
        }
        __syncthreads();  // every warp is done with this stage before it is refilled
    }

    if (tid == 0 && *(volatile int*)&s_abort) {
        // a wait ran out: let the copies still in flight land (bounded) before the CTA's shared
        // memory is released.  At most the Q tile and the last two KV blocks can be pending.
        mbar_wait(smem_u32(&bars[0]), 0u, nullptr);
        for (int j = issued > 0 ? issued - 1 : 0; j <= issued; ++j)
            mbar_wait(smem_u32(&bars[1 + (j & 1)]), (uint32_t)(j >> 1) & 1u, nullptr);
    }
    // ---- out = O / l for the live rows of this warp
    const int row_a = warp * 16 + gq, row_b = row_a + 8;
    if (ok) {
#pragma unroll
        for (int dt = 0; dt < 16; ++dt) {
            const int d = dt * 8 + 2 * cq;
            if (row_a < n_q) {
                __nv_bfloat16* p = out + (int64_t)(q_row0 + row_a) * ldo + (int64_t)h * D + d;
                *reinterpret_cast<uint32_t*>(p) = pack2(__fdiv_rn(o[dt][0], l_a), __fdiv_rn(o[dt][1], l_a));
            }
            if (row_b < n_q) {
                __nv_bfloat16* p = out + (int64_t)(q_row0 + row_b) * ldo + (int64_t)h * D + d;
                *reinterpret_cast<uint32_t*>(p) = pack2(__fdiv_rn(o[dt][2], l_b), __fdiv_rn(o[dt][3], l_b));
            }
        }
    }
}

bool ensure_attr() {
    static std::once_flag once[64];
    static bool okd[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::call_once(once[dev], [&] {
        okd[dev] = cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)SMEM_BYTES) == cudaSuccess;
    });
    return okd[dev];
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
    uint32_t* err = bi::device_error_word();
    if (!err || !ensure_attr()) return BI_ERR_CUDA;
    CUtensorMap tmQ, tmK, tmV;
    const uint64_t kv_row = (uint64_t)Hkv * D;
    if (!bi::make_tmap_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, (uint64_t)Hq * D, (uint64_t)q_rows,
                          (uint64_t)ldq * 2, 64, QT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !bi::make_tmap_2d(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k_cache, kv_row, (uint64_t)cache_tokens, kv_row * 2,
                          64, KB, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !bi::make_tmap_2d(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v_cache, kv_row, (uint64_t)cache_tokens, kv_row * 2,
                          64, KB, CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    dim3 grid((unsigned)n_tiles, (unsigned)Hq);
    prefill_attn_kernel<<<grid, THREADS, SMEM_BYTES, bi::as_stream(stream)>>>(
        tmQ, tmK, tmV, q_indptr, q_tile_indptr, kv_indptr, q_pos0, B, Hq, Hkv, (int)q_rows, (int)cache_tokens, scale,
        static_cast<__nv_bfloat16*>(out), ldo, err);
    return bi::launch_status();
}
