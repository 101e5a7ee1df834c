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
// Phase 1 (one CTA per (chunk slot, kv head)).  Slot s covers packed tokens
// [s*256, s*256 + 256).  The CTA finds the sequence that owns the slot.  Its tokens
// [c*256, min(c*256 + 256, L)) are chunk c of that sequence.  The CTA computes, for the
// group's query heads:
//     s_j = scale * q . k_j          (mma.sync m16n8k16: bf16 products, fp32 accumulate)
//     m_c = max_j s_j                (exact; order-free)
//     p_j = exp(s_j - m_c),  l_c = sum_j p_j     (fixed shuffle / shared-memory trees)
//     o_c = sum_j p_j v_j            (fp32 FMAs, fixed token order per thread, fixed tree)
// and stores (o_c, m_c, l_c) to the workspace.  K and V reach shared memory through TMA,
// 128B-swizzled.  V reuses K's buffer once the scores are done.
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
constexpr int THREADS = 256;   // 8 warps
constexpr int BOX_TOK = 64;    // tokens per TMA box
constexpr int BOX_BYTES = BOX_TOK * 64 * 2;  // 64 tokens x 64 dims (one 128-byte half row) = 8 KB
constexpr int KV_BYTES = CHUNK * D * 2;      // 64 KB

constexpr uint32_t DEVERR_BAD_LAYOUT = 1u << 8;  // kv_indptr / kv_len violate the documented layout

template <int G>
struct AttnLayout {
    static constexpr int S_OFF = KV_BYTES;                      // scores / probabilities [CHUNK][G] fp32
    static constexpr int RED_OFF = S_OFF + CHUNK * G * 4;       // [8 warps][G][D] fp32
    static constexpr int STAT_OFF = RED_OFF + 8 * G * D * 4;    // per-warp partial max / sum [8][G] x 2
    static constexpr int BAR_OFF = STAT_OFF + 2 * 8 * G * 4;
    static constexpr size_t BYTES = 1024 + BAR_OFF + 64;
};

// smem address of (token j, dim pair starting at d) in the swizzled K/V buffer
__device__ __forceinline__ uint32_t kv_addr(uint32_t base, int j, int d) {
    const uint32_t box = (uint32_t)((j >> 6) * 2 + (d >> 6));
    return swz(base + box * BOX_BYTES + (uint32_t)(j & 63) * 128 + (uint32_t)(d & 63) * 2, 7u);
}

template <int G>
__global__ void __launch_bounds__(THREADS, 2)
decode_attn_chunk_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ kv_indptr,
                         const int32_t* __restrict__ kv_len, int B, int Hq, int Hkv, float scale,
                         float* __restrict__ o_part, float* __restrict__ ml_part, uint32_t* err) {
    using L = AttnLayout<G>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* sS = reinterpret_cast<float*>(base + L::S_OFF);
    float* sRed = reinterpret_cast<float*>(base + L::RED_OFF);
    float* sMax = reinterpret_cast<float*>(base + L::STAT_OFF);
    float* sSum = sMax + 8 * G;
    uint64_t* bar = reinterpret_cast<uint64_t*>(base + L::BAR_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slot = blockIdx.x;
    const int g = blockIdx.y;
    const int64_t tok0 = (int64_t)slot * CHUNK;

    // Which sequence owns this slot: the last b with kv_indptr[b] <= tok0 (binary search).
    int lo = 0, hi = B;  // invariant: kv_indptr[lo] <= tok0 < kv_indptr[hi] when tok0 < kv_indptr[B]
    if (tok0 < kv_indptr[0] || tok0 >= kv_indptr[B]) return;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (kv_indptr[mid] <= tok0) lo = mid; else hi = mid;
    }
    const int b = lo;
    const int64_t sbase = kv_indptr[b];
    const int len = kv_len[b];
    const int64_t cap = (int64_t)kv_indptr[b + 1] - sbase;
    if ((sbase % CHUNK) != 0 || len <= 0 || (int64_t)len > cap) {
        if (tid == 0 && g == 0 && tok0 - sbase < CHUNK) atomicOr(err, DEVERR_BAD_LAYOUT);
        return;
    }
    const int c = (int)((tok0 - sbase) / CHUNK);
    const int n_tok = min(CHUNK, len - c * CHUNK);
    if (n_tok <= 0) return;  // capacity padding beyond the sequence
    const int n_box_tok = (n_tok + BOX_TOK - 1) / BOX_TOK;  // 64-token groups holding live tokens

    const uint32_t kv_base = smem_u32(base);
    const uint32_t bar_a = smem_u32(bar);
    if (tid == 0) {
        mbar_init(bar_a, 1);
        fence_barrier_init();
        fence_proxy_async_shared();
    }
    __syncthreads();
    if (tid == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        mbar_arrive_expect_tx(bar_a, (uint32_t)(n_box_tok * 2 * BOX_BYTES));
        for (int tg = 0; tg < n_box_tok; ++tg)
            for (int hf = 0; hf < 2; ++hf)
                tma_load_2d(kv_base + (tg * 2 + hf) * BOX_BYTES, &tmK, g * D + hf * 64, (int)(tok0 + tg * BOX_TOK),
                            bar_a);
    }

    // Query fragments (B operand, [16 dims x 8 heads] per k-step; heads >= G are zero).
    uint32_t qf[8][2];
    {
        const int hh = lane >> 2, dq = (lane & 3) * 2;
        const __nv_bfloat16* qh = q + ((int64_t)b * Hq + (int64_t)g * G + (hh < G ? hh : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t v0 = 0u, v1 = 0u;
            if (hh < G) {
                v0 = *reinterpret_cast<const uint32_t*>(qh + kk * 16 + dq);
                v1 = *reinterpret_cast<const uint32_t*>(qh + kk * 16 + dq + 8);
            }
            qf[kk][0] = v0;
            qf[kk][1] = v1;
        }
    }

    const bool k_ok = __all_sync(0xffffffffu, mbar_wait(bar_a, 0u, nullptr));
    if (!k_ok && lane == 0) atomicOr(err, bi::DEVERR_WAIT_FULL);

    // ---- scores: warp w owns tokens [32w, 32w + 32) as two 16-row MMA tiles
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        const int t0 = warp * 32 + mt * 16;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (k_ok && t0 < n_tok) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t a[4];
                ldmatrix_x4(kv_addr(kv_base, t0 + (lane & 15), kk * 16 + (lane >> 4) * 8), a);
                mma_m16n8k16_bf16(acc, a, qf[kk]);
            }
        }
        const int gg = lane >> 2, hq = (lane & 3) * 2;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = t0 + gg + (e >> 1) * 8;
            const int h = hq + (e & 1);
            if (h < G) sS[j * G + h] = (j < n_tok) ? __fmul_rn(acc[e], scale) : -INFINITY;
        }
    }
    __syncthreads();  // K no longer needed; scores complete

    if (tid == 0) {  // V into the same buffer (its previous contents are dead: every ldmatrix has completed)
        fence_proxy_async_shared();
        mbar_arrive_expect_tx(bar_a, (uint32_t)(n_box_tok * 2 * BOX_BYTES));
        for (int tg = 0; tg < n_box_tok; ++tg)
            for (int hf = 0; hf < 2; ++hf)
                tma_load_2d(kv_base + (tg * 2 + hf) * BOX_BYTES, &tmV, g * D + hf * 64, (int)(tok0 + tg * BOX_TOK),
                            bar_a);
    }

    // ---- softmax statistics over the chunk (thread tid owns token tid)
    float s[G], p[G];
#pragma unroll
    for (int h = 0; h < G; ++h) s[h] = sS[tid * G + h];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float m = s[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) sMax[warp * G + h] = m;
    }
    __syncthreads();
    float mc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float m = sMax[h];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = fmaxf(m, sMax[w * G + h]);
        mc[h] = m;
        p[h] = (tid < n_tok) ? expf(__fsub_rn(s[h], m)) : 0.0f;
        sS[tid * G + h] = p[h];
        float sum = p[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, off));
        if (lane == 0) sSum[warp * G + h] = sum;
    }
    __syncthreads();

    // ---- o_c = sum_j p_j v_j: thread owns dims [8*dg, 8*dg + 8) and tokens j = tg + 16 i
    const bool v_ok = __all_sync(0xffffffffu, mbar_wait(bar_a, 1u, nullptr));
    if (!v_ok && lane == 0) atomicOr(err, bi::DEVERR_WAIT_FULL);
    const int dg = tid & 15, tg = tid >> 4;
    float acc[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] = 0.0f;
    if (v_ok) {
#pragma unroll 4
        for (int i = 0; i < CHUNK / 16; ++i) {
            const int j = tg + 16 * i;
            if (j >= n_tok) break;
            uint4 u;
            const uint32_t a = kv_addr(kv_base, j, dg * 8);
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(a));
            const float vf[8] = {bi::bf16_lo(u.x), bi::bf16_hi(u.x), bi::bf16_lo(u.y), bi::bf16_hi(u.y),
                                 bi::bf16_lo(u.z), bi::bf16_hi(u.z), bi::bf16_lo(u.w), bi::bf16_hi(u.w)};
            float pj[G];
#pragma unroll
            for (int h = 0; h < G; ++h) pj[h] = sS[j * G + h];
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[h][e] = __fmaf_rn(pj[h], vf[e], acc[h][e]);
        }
    }
    // pair the two token groups of this warp (lanes l and l ^ 16 share dg), then warps in order
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] = __fadd_rn(acc[h][e], __shfl_xor_sync(0xffffffffu, acc[h][e], 16));
    if (lane < 16) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float4* dst = reinterpret_cast<float4*>(sRed + (warp * G + h) * D + dg * 8);
            dst[0] = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
            dst[1] = make_float4(acc[h][4], acc[h][5], acc[h][6], acc[h][7]);
        }
    }
    __syncthreads();

    const int hq0 = g * G;
    for (int o = tid; o < G * D; o += THREADS) {
        const int h = o / D, d = o % D;
        float v = sRed[h * D + d];
#pragma unroll
        for (int w = 1; w < 8; ++w) v = __fadd_rn(v, sRed[(w * G + h) * D + d]);
        o_part[((int64_t)slot * Hq + hq0 + h) * D + d] = v;
    }
    if (tid < G) {
        float l = sSum[tid];
#pragma unroll
        for (int w = 1; w < 8; ++w) l = __fadd_rn(l, sSum[w * G + tid]);
        float2* ml = reinterpret_cast<float2*>(ml_part + ((int64_t)slot * Hq + hq0 + tid) * 2);
        // mc[] is uniform across threads; select this head's value without dynamic register indexing
        float m_sel = mc[0];
#pragma unroll
        for (int h = 1; h < G; ++h)
            if (tid == h) m_sel = mc[h];
        *ml = make_float2(m_sel, l);
    }
}

// Phase 2: one warp per (sequence, query head); lane owns dims [4*lane, 4*lane + 4).
template <bool OUT_BF16>
__global__ void __launch_bounds__(128)
decode_attn_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ ml_part,
                         const int32_t* __restrict__ kv_indptr, const int32_t* __restrict__ kv_len, int Hq,
                         void* __restrict__ out, uint32_t* err) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x * 4 + warp;
    const int b = blockIdx.y;
    if (h >= Hq) return;
    const int64_t sbase = kv_indptr[b];
    const int len = kv_len[b];
    const int64_t cap = (int64_t)kv_indptr[b + 1] - sbase;
    if ((sbase % CHUNK) != 0 || len <= 0 || (int64_t)len > cap) {
        if (lane == 0) atomicOr(err, DEVERR_BAD_LAYOUT);  // out row left unwritten
        return;
    }
    const int nch = (len + CHUNK - 1) / CHUNK;
    const int64_t slot0 = sbase / CHUNK;
    float m = -INFINITY, l = 0.0f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nch; ++c) {
        const int64_t idx = (slot0 + c) * Hq + h;
        const float2 mlc = *reinterpret_cast<const float2*>(ml_part + idx * 2);
        const float4 oc = *reinterpret_cast<const float4*>(o_part + idx * D + lane * 4);
        const float mn = fmaxf(m, mlc.x);
        const float a = expf(__fsub_rn(m, mn));   // 0 on the first chunk (m = -inf)
        const float bsc = expf(__fsub_rn(mlc.x, mn));
        l = __fmaf_rn(l, a, __fmul_rn(mlc.y, bsc));
        o.x = __fmaf_rn(o.x, a, __fmul_rn(oc.x, bsc));
        o.y = __fmaf_rn(o.y, a, __fmul_rn(oc.y, bsc));
        o.z = __fmaf_rn(o.z, a, __fmul_rn(oc.z, bsc));
        o.w = __fmaf_rn(o.w, a, __fmul_rn(oc.w, bsc));
        m = mn;
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

size_t partial_bytes(int64_t total_tokens, int32_t Hq) {
    const int64_t slots = (total_tokens + CHUNK - 1) / CHUNK;
    return (size_t)slots * Hq * (D + 2) * sizeof(float);
}

template <int G>
int launch_chunks(const void* q, const void* k, const void* v, const int32_t* kv_indptr, const int32_t* kv_len,
                  int B, int64_t T, int Hq, int Hkv, float scale, float* o_part, float* ml_part, cudaStream_t s) {
    using L = AttnLayout<G>;
    uint32_t* err = bi::device_error_word();
    auto kern = decode_attn_chunk_kernel<G>;
    if (!err || !set_smem_once(kern, L::BYTES)) return BI_ERR_CUDA;
    CUtensorMap tmK, tmV;
    const uint64_t row = (uint64_t)Hkv * D;  // elements per packed token
    if (!bi::make_tmap_2d(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, row, (uint64_t)T, row * 2, 64, BOX_TOK,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
        !bi::make_tmap_2d(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, row, (uint64_t)T, row * 2, 64, BOX_TOK,
                          CU_TENSOR_MAP_SWIZZLE_128B))
        return BI_ERR_CUDA;
    dim3 grid((unsigned)((T + CHUNK - 1) / CHUNK), (unsigned)Hkv);
    kern<<<grid, THREADS, L::BYTES, s>>>(tmK, tmV, static_cast<const __nv_bfloat16*>(q), kv_indptr, kv_len, B, Hq,
                                         Hkv, scale, o_part, ml_part, err);
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
        decode_attn_merge_kernel<true><<<grid, 128, 0, s>>>(o_part, ml_part, kv_indptr, kv_len, Hq, out, err);
    else
        decode_attn_merge_kernel<false><<<grid, 128, 0, s>>>(o_part, ml_part, kv_indptr, kv_len, Hq, out, err);
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
std::once_flag g_scratch_once[kNoAllocMaxDevices];
void* g_scratch_ptr[kNoAllocMaxDevices];

// Device address of the scratch array on the current device.  It is looked up on the
// first call made with that device current, then cached.  Returns nullptr if the
// lookup fails.
void* noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
    std::call_once(g_scratch_once[dev], [dev] {
        void* p = nullptr;
        g_scratch_ptr[dev] = (cudaGetSymbolAddress(&p, g_decode_attn_scratch) == cudaSuccess) ? p : nullptr;
    });
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
        decode_attn_merge_kernel<true><<<grid, 128, 0, s>>>(o_part, ml_part, kv_indptr, kv_len, Hq, out, err);
    else
        decode_attn_merge_kernel<false><<<grid, 128, 0, s>>>(o_part, ml_part, kv_indptr, kv_len, Hq, out, err);
    return bi::launch_status();
}
