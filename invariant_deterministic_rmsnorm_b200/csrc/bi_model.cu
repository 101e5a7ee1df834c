// bi_model.cu -- the row-wise model ops a decoder needs around the hot-path kernels:
// embedding gather, rotary position embedding, KV-cache append, residual add, SwiGLU, argmax.
//
// Every op here works on one token row at a time, with no reduction across rows.  An
// output row's bits therefore depend only on that row's inputs, and its position (for
// RoPE), whatever the batch.  Source for why that matters: "Defeating Nondeterminism in
// LLM Inference" (Spanish summary), "La verdadera causa clave".  The batch size changes
// from request to request, so every kernel must give each row the same bits at any batch
// size.
#include <math.h>

#include "bi_common.cuh"
#include "bi_model.h"
#include "bi_sm100.cuh"

using bi::sm100::pdl_trigger;
using bi::sm100::pdl_wait;

namespace {

// ------------------------------------------------------------------ embedding gather
__global__ void embed_kernel(const int32_t* __restrict__ tokens, const __nv_bfloat16* __restrict__ table,
                             __nv_bfloat16* __restrict__ out, int64_t H, int64_t vocab, uint32_t* err) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    const int64_t t = blockIdx.x;
    const int32_t id = tokens[t];
    if (id < 0 || id >= vocab) {
        if (threadIdx.x == 0) atomicOr(err, bi::DEVERR_BAD_TOKEN);  // token id out of range: row left unwritten
        return;
    }
    const uint4* src = reinterpret_cast<const uint4*>(table + (int64_t)id * H);
    uint4* dst = reinterpret_cast<uint4*>(out + t * H);
    for (int64_t i = threadIdx.x; i < H / 8; i += blockDim.x) dst[i] = src[i];
}

// ------------------------------------------------------------------ rotary position embedding
// table[p][i] = (cos, sin) of the angle p * theta^(-2i/D) for pair i < D/2, formed in double
// precision and rounded once to fp32.  Built once per (theta, D, positions); every rotation reads it.
__global__ void rope_table_kernel(float2* __restrict__ table, int64_t rows, int half, double log_theta, int D) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= rows * half) return;
    const int64_t p = k / half;
    const int i = (int)(k % half);
    const double ang = (double)p * exp(-log_theta * (2.0 * i) / (double)D);
    double sd, cd;
    sincos(ang, &sd, &cd);
    table[k] = make_float2((float)cd, (float)sd);
}

// (x_i, x_{i+D/2}) -> (x_i cos - x_{i+D/2} sin, x_{i+D/2} cos + x_i sin) in fp32, rounded once to
// bf16 (the "rotate half" pairing of Llama).  One thread turns pairs i and i+1 of one head.
__global__ void rope_kernel(__nv_bfloat16* __restrict__ x, int64_t ld_row, int heads, int D,
                            const int32_t* __restrict__ pos, const float4* __restrict__ table, int64_t table_rows,
                            uint32_t* err) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    const int64_t t = blockIdx.x;
    const int half = D / 2, quads = half / 2;  // pairs per head, two at a time
    const int j = blockIdx.y * blockDim.x + threadIdx.x;
    if (j >= heads * quads) return;
    const int32_t p = pos[t];
    if (p < 0 || p >= table_rows) {
        if (j == 0) atomicOr(err, bi::DEVERR_BAD_POSITION);  // position outside the table: row left as is
        return;
    }
    const int h = j / quads, i = (j % quads) * 2;
    const float4 cs = table[((int64_t)p * half + i) / 2];  // (cos_i, sin_i, cos_i+1, sin_i+1)
    uint32_t* lo = reinterpret_cast<uint32_t*>(x + t * ld_row + (int64_t)h * D + i);
    uint32_t* hi = reinterpret_cast<uint32_t*>(x + t * ld_row + (int64_t)h * D + half + i);
    const uint32_t av = *lo, bv = *hi;
    const float a0 = bi::bf16_lo(av), a1 = bi::bf16_hi(av), b0 = bi::bf16_lo(bv), b1 = bi::bf16_hi(bv);
    *lo = bi::pack_bf16x2(__fsub_rn(__fmul_rn(a0, cs.x), __fmul_rn(b0, cs.y)),
                          __fsub_rn(__fmul_rn(a1, cs.z), __fmul_rn(b1, cs.w)));
    *hi = bi::pack_bf16x2(__fadd_rn(__fmul_rn(b0, cs.x), __fmul_rn(a0, cs.y)),
                          __fadd_rn(__fmul_rn(b1, cs.z), __fmul_rn(a1, cs.w)));
}

// The same rotation, eight pairs i .. i+7 (i a multiple of 8) of one head per thread, with
// 16-byte loads and stores, for rows that are 16-byte aligned and head_dim a multiple of 16.
// Element for element it runs rope_kernel's operations, so the two give the same bits.
__global__ void rope8_kernel(__nv_bfloat16* __restrict__ x, int64_t ld_row, int heads, int D,
                             const int32_t* __restrict__ pos, const float4* __restrict__ table, int64_t table_rows,
                             uint32_t* err) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    const int64_t t = blockIdx.x;
    const int half = D / 2, octs = half / 8;  // pairs per head, eight at a time
    const int j = blockIdx.y * blockDim.x + threadIdx.x;
    if (j >= heads * octs) return;
    const int32_t p = pos[t];
    if (p < 0 || p >= table_rows) {
        if (j == 0) atomicOr(err, bi::DEVERR_BAD_POSITION);  // position outside the table: row left as is
        return;
    }
    const int h = j / octs, i = (j % octs) * 8;
    const float4* cs = table + ((int64_t)p * half + i) / 2;  // (cos, sin) of pairs i, i+1 per float4
    uint4* lo = reinterpret_cast<uint4*>(x + t * ld_row + (int64_t)h * D + i);
    uint4* hi = reinterpret_cast<uint4*>(x + t * ld_row + (int64_t)h * D + half + i);
    const uint4 av = *lo, bv = *hi;
    const uint32_t a[4] = {av.x, av.y, av.z, av.w}, b[4] = {bv.x, bv.y, bv.z, bv.w};
    uint32_t ro[4], rh[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 c = cs[q];
        const float a0 = bi::bf16_lo(a[q]), a1 = bi::bf16_hi(a[q]), b0 = bi::bf16_lo(b[q]), b1 = bi::bf16_hi(b[q]);
        ro[q] = bi::pack_bf16x2(__fsub_rn(__fmul_rn(a0, c.x), __fmul_rn(b0, c.y)),
                                __fsub_rn(__fmul_rn(a1, c.z), __fmul_rn(b1, c.w)));
        rh[q] = bi::pack_bf16x2(__fadd_rn(__fmul_rn(b0, c.x), __fmul_rn(a0, c.y)),
                                __fadd_rn(__fmul_rn(b1, c.z), __fmul_rn(a1, c.w)));
    }
    *lo = make_uint4(ro[0], ro[1], ro[2], ro[3]);
    *hi = make_uint4(rh[0], rh[1], rh[2], rh[3]);
}

// ------------------------------------------------------------------ KV append
// dst[dst_row[t], :] = src[t, :] for one packed row of `row_elems` bf16 (all kv heads of a token).
__global__ void kv_append_kernel(const __nv_bfloat16* __restrict__ src, int64_t ld_src,
                                 const int32_t* __restrict__ dst_row, __nv_bfloat16* __restrict__ dst,
                                 int64_t row_elems, int64_t dst_rows, uint32_t* err) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    const int64_t t = blockIdx.x;
    const int64_t r = dst_row[t];
    if (r < 0 || r >= dst_rows) {
        if (threadIdx.x == 0) atomicOr(err, bi::DEVERR_BAD_DST_ROW);  // destination row out of range: skipped
        return;
    }
    const uint4* s = reinterpret_cast<const uint4*>(src + t * ld_src);
    uint4* d = reinterpret_cast<uint4*>(dst + r * row_elems);
    for (int64_t i = threadIdx.x; i < row_elems / 8; i += blockDim.x) d[i] = s[i];
}

// ------------------------------------------------------------------ residual add (in place)
__global__ void add_kernel(__nv_bfloat16* __restrict__ h, int64_t ldh, const __nv_bfloat16* __restrict__ d,
                           int64_t ldd, int64_t N) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    const int64_t t = blockIdx.x;
    const int64_t i = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;  // 8-element vector of the row
    if (i < N / 8) {
        uint4* hp = reinterpret_cast<uint4*>(h + t * ldh) + i;
        const uint4 a = *hp;
        const uint4 b = *(reinterpret_cast<const uint4*>(d + t * ldd) + i);
        uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            av[j] = bi::pack_bf16x2(__fadd_rn(bi::bf16_lo(av[j]), bi::bf16_lo(bv[j])),
                                    __fadd_rn(bi::bf16_hi(av[j]), bi::bf16_hi(bv[j])));
        *hp = make_uint4(av[0], av[1], av[2], av[3]);
    }
}

// ------------------------------------------------------------------ SwiGLU
// out[t, j] = silu(gu[t, j]) * gu[t, N + j] with silu(g) = g / (1 + e^-g), fp32, rounded once.
__global__ void swiglu_kernel(const __nv_bfloat16* __restrict__ gu, int64_t ld_gu, __nv_bfloat16* __restrict__ out,
                              int64_t ld_out, int64_t N) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    const int64_t t = blockIdx.x;
    const int64_t i = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;  // 8-element vector of the row
    if (i < N / 8) {
        const uint4 g = *(reinterpret_cast<const uint4*>(gu + t * ld_gu) + i);
        const uint4 u = *(reinterpret_cast<const uint4*>(gu + t * ld_gu + N) + i);
        uint32_t gv[4] = {g.x, g.y, g.z, g.w}, uv[4] = {u.x, u.y, u.z, u.w}, ov[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float g0 = bi::bf16_lo(gv[j]), g1 = bi::bf16_hi(gv[j]);
            const float s0 = __fdiv_rn(g0, __fadd_rn(1.0f, expf(-g0)));
            const float s1 = __fdiv_rn(g1, __fadd_rn(1.0f, expf(-g1)));
            ov[j] = bi::pack_bf16x2(__fmul_rn(s0, bi::bf16_lo(uv[j])), __fmul_rn(s1, bi::bf16_hi(uv[j])));
        }
        *(reinterpret_cast<uint4*>(out + t * ld_out) + i) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
    }
}

// ------------------------------------------------------------------ argmax
// The index of the largest fp32 value of each row; among equal values the smallest index.
// NaN compares as smaller than everything.  One CTA per row, a fixed tree.
constexpr int ARGMAX_THREADS = 1024;
__global__ void __launch_bounds__(ARGMAX_THREADS) argmax_kernel(const float* __restrict__ x, int64_t ld, int64_t N,
                                                                int32_t* __restrict__ out) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    __shared__ float sv[ARGMAX_THREADS];
    __shared__ int32_t si[ARGMAX_THREADS];
    const int64_t t = blockIdx.x;
    float best = -INFINITY;
    int32_t bi_ = 0x7fffffff;
    for (int64_t i = threadIdx.x; i < N; i += blockDim.x) {
        const float v = x[t * ld + i];
        if (v > best || (v == best && (int32_t)i < bi_)) {
            best = v;
            bi_ = (int32_t)i;
        }
    }
    sv[threadIdx.x] = best;
    si[threadIdx.x] = bi_;
    __syncthreads();
    for (int off = ARGMAX_THREADS / 2; off > 0; off >>= 1) {
        if ((int)threadIdx.x < off) {
            const float v = sv[threadIdx.x + off];
            const int32_t j = si[threadIdx.x + off];
            if (v > sv[threadIdx.x] || (v == sv[threadIdx.x] && j < si[threadIdx.x])) {
                sv[threadIdx.x] = v;
                si[threadIdx.x] = j;
            }
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) out[t] = si[0] == 0x7fffffff ? 0 : si[0];
}

int rows_ok(int64_t rows) { return rows >= 0 && rows <= 0x7fffffffLL; }

// v[i] += step: the per-step bookkeeping of a replayed decode step (positions, cache rows, KV
// lengths), so that no device work in the decoder runs outside this library.
__global__ void advance_kernel(int32_t* __restrict__ v, int64_t n, int32_t step) {
    pdl_wait();  // inputs may come from the kernel just before this one
    pdl_trigger();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) v[i] += step;
}

}  // namespace

BI_API int bi_embed(const int32_t* tokens, const void* table, void* out, int64_t T, int64_t H, int64_t vocab,
                    void* stream) {
    if (T < 0 || H <= 0 || vocab <= 0 || !rows_ok(T)) return BI_ERR_INVALID_ARG;
    if (T == 0) return BI_OK;
    if (!tokens || !table || !out) return BI_ERR_INVALID_ARG;
    if (H % 8 != 0 || !bi::aligned16(table) || !bi::aligned16(out)) return BI_ERR_MISALIGNED;
    uint32_t* err = bi::device_error_word();
    if (!err) return BI_ERR_CUDA;
    if (bi::launch_pdl(embed_kernel, dim3((unsigned)T), dim3(256), 0, bi::as_stream(stream), 0u,
                       tokens, static_cast<const __nv_bfloat16*>(table), static_cast<__nv_bfloat16*>(out), H, vocab,
                       err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

BI_API int bi_rope_table(void* table, int64_t positions, int32_t head_dim, double theta, void* stream) {
    if (positions < 0 || head_dim <= 0 || head_dim % 4 != 0 || !(theta > 1.0)) return BI_ERR_INVALID_ARG;
    if (positions == 0) return BI_OK;
    if (!table) return BI_ERR_INVALID_ARG;
    if (!bi::aligned16(table)) return BI_ERR_MISALIGNED;
    const int half = head_dim / 2;
    if (positions > ((int64_t)1 << 38) / half) return BI_ERR_UNSUPPORTED_SHAPE;
    const int64_t n = positions * half;
    if (bi::launch_pdl(rope_table_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, bi::as_stream(stream), 0u,
                       static_cast<float2*>(table), positions, half, log(theta), head_dim) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

BI_API int bi_rope(void* x, int64_t T, int64_t ld_row, int32_t heads, int32_t head_dim, const int32_t* pos,
                   const void* table, int64_t table_rows, void* stream) {
    if (T < 0 || heads <= 0 || head_dim <= 0 || head_dim % 4 != 0 || table_rows <= 0 || !rows_ok(T))
        return BI_ERR_INVALID_ARG;
    if (ld_row < (int64_t)heads * head_dim) return BI_ERR_INVALID_ARG;
    if (T == 0) return BI_OK;
    if (!x || !pos || !table) return BI_ERR_INVALID_ARG;
    if (!bi::aligned16(table) || (reinterpret_cast<uintptr_t>(x) & 3u) || ld_row % 2 != 0) return BI_ERR_MISALIGNED;
    uint32_t* err = bi::device_error_word();
    if (!err) return BI_ERR_CUDA;
    // 16-byte accesses where the layout allows them (the same bits either way)
    const bool vec = bi::aligned16(x) && ld_row % 8 == 0 && head_dim % 16 == 0;
    const int work = heads * (head_dim / (vec ? 16 : 4));
    if ((work + 127) / 128 > 65535) return BI_ERR_UNSUPPORTED_SHAPE;
    dim3 grid((unsigned)T, (unsigned)((work + 127) / 128));
    if (bi::launch_pdl(vec ? rope8_kernel : rope_kernel, dim3(grid), dim3(128), 0, bi::as_stream(stream), 0u,
                       static_cast<__nv_bfloat16*>(x), ld_row, heads, head_dim, pos,
                       static_cast<const float4*>(table), table_rows, err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

BI_API int bi_kv_append(const void* src, int64_t ld_src, const int32_t* dst_row, void* dst, int64_t T,
                        int64_t row_elems, int64_t dst_rows, void* stream) {
    if (T < 0 || row_elems <= 0 || dst_rows < 0 || ld_src < row_elems || !rows_ok(T)) return BI_ERR_INVALID_ARG;
    if (T == 0) return BI_OK;
    if (!src || !dst_row || !dst) return BI_ERR_INVALID_ARG;
    if (row_elems % 8 != 0 || ld_src % 8 != 0 || !bi::aligned16(src) || !bi::aligned16(dst)) return BI_ERR_MISALIGNED;
    uint32_t* err = bi::device_error_word();
    if (!err) return BI_ERR_CUDA;
    if (bi::launch_pdl(kv_append_kernel, dim3((unsigned)T), dim3(256), 0, bi::as_stream(stream), 0u,
                       static_cast<const __nv_bfloat16*>(src), ld_src, dst_row, static_cast<__nv_bfloat16*>(dst),
                       row_elems, dst_rows, err) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

BI_API int bi_add(void* h, int64_t ldh, const void* d, int64_t ldd, int64_t T, int64_t N, void* stream) {
    if (T < 0 || N <= 0 || ldh < N || ldd < N || !rows_ok(T)) return BI_ERR_INVALID_ARG;
    if (T == 0) return BI_OK;
    if (!h || !d) return BI_ERR_INVALID_ARG;
    if (N % 8 != 0 || ldh % 8 != 0 || ldd % 8 != 0 || !bi::aligned16(h) || !bi::aligned16(d)) return BI_ERR_MISALIGNED;
    if ((N / 8 + 255) / 256 > 65535) return BI_ERR_UNSUPPORTED_SHAPE;
    if (bi::launch_pdl(add_kernel, dim3((unsigned)T, (unsigned)((N / 8 + 255) / 256)), dim3(256), 0,
                       bi::as_stream(stream), 0u,
                       static_cast<__nv_bfloat16*>(h), ldh, static_cast<const __nv_bfloat16*>(d), ldd,
                       N) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

BI_API int bi_swiglu(const void* gu, int64_t ld_gu, void* out, int64_t ld_out, int64_t T, int64_t N, void* stream) {
    if (T < 0 || N <= 0 || ld_gu < 2 * N || ld_out < N || !rows_ok(T)) return BI_ERR_INVALID_ARG;
    if (T == 0) return BI_OK;
    if (!gu || !out) return BI_ERR_INVALID_ARG;
    if (N % 8 != 0 || ld_gu % 8 != 0 || ld_out % 8 != 0 || !bi::aligned16(gu) || !bi::aligned16(out))
        return BI_ERR_MISALIGNED;
    if ((N / 8 + 255) / 256 > 65535) return BI_ERR_UNSUPPORTED_SHAPE;
    if (bi::launch_pdl(swiglu_kernel, dim3((unsigned)T, (unsigned)((N / 8 + 255) / 256)), dim3(256), 0,
                       bi::as_stream(stream), 0u,
                       static_cast<const __nv_bfloat16*>(gu), ld_gu, static_cast<__nv_bfloat16*>(out), ld_out,
                       N) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

BI_API int bi_argmax(const float* x, int64_t ld, int64_t T, int64_t N, int32_t* out, void* stream) {
    if (T < 0 || N <= 0 || ld < N || !rows_ok(T) || N > 0x7fffffffLL) return BI_ERR_INVALID_ARG;
    if (T == 0) return BI_OK;
    if (!x || !out) return BI_ERR_INVALID_ARG;
    if (bi::launch_pdl(argmax_kernel, dim3((unsigned)T), dim3(ARGMAX_THREADS), 0, bi::as_stream(stream), 0u,
                       x, ld, N, out) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}

BI_API int bi_advance(int32_t* v, int64_t n, int32_t step, void* stream) {
    if (n < 0 || n > ((int64_t)1 << 40)) return BI_ERR_INVALID_ARG;
    if (n == 0) return BI_OK;
    if (!v) return BI_ERR_INVALID_ARG;
    if (bi::launch_pdl(advance_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, bi::as_stream(stream), 0u,
                       v, n, step) != cudaSuccess)
        return BI_ERR_CUDA;
    return bi::launch_status();
}
