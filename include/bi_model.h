/*
 * bi_model.h -- the decoder ops around the hot-path kernels of bi.h: embedding gather,
 * rotary position embedding, KV-cache append, residual add, SwiGLU, greedy argmax and
 * batch-invariant causal prefill attention.
 *
 * Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), sections "La
 * verdadera causa clave" and "Attention".  Inference is not deterministic for a user
 * because the batch a request shares changes from call to call.  A model is
 * batch-invariant only if every op it runs gives each token row the same bits at any batch
 * size.  The row-wise ops below do no reduction across rows.  The prefill attention fixes
 * the order in which a query row visits its keys by absolute position, so it is invariant
 * both to the batch and to how a prompt is cut into prefill chunks.
 *
 * Conventions are those of bi.h:
 *   - Every pointer is a device pointer unless noted.  The caller owns every buffer.
 *   - Calls are asynchronous on `stream` (a cudaStream_t, NULL = the legacy default stream).
 *   - Argument checks happen on the host and return a bi_status without launching.
 *   - Checks that need device data (token ids, row indices, indptr arrays) are made by the
 *     kernel.  A failing row is skipped, and a bit is OR-ed into the device error word
 *     (bi_get_device_error).
 *   - bf16 tensors are raw 16-bit patterns.  Base pointers and row strides must be 16-byte
 *     aligned (BI_ERR_MISALIGNED otherwise).
 */
#ifndef BI_MODEL_H
#define BI_MODEL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * bi_embed -- out[t, :] = table[tokens[t], :]
 *
 * tokens int32 [T]; table bf16 [vocab, H]; out bf16 [T, H] (row stride H).  A pure copy.
 * An id outside [0, vocab) leaves its row unwritten and sets bit 0x200.
 * H must be a multiple of 8.
 */
int bi_embed(const int32_t* tokens, const void* table, void* out, int64_t T, int64_t H, int64_t vocab,
             void* stream);

/*
 * bi_rope_table -- the cos/sin table that bi_rope reads.
 *
 * table: fp32 pairs [positions, head_dim/2, 2], 16-byte aligned, owned by the caller.
 * Entry (p, i) holds (cos a, sin a) for a = p * theta^(-2i/head_dim).  The angle and its
 * cosine and sine are formed in double precision, then rounded once to fp32.  Build it once
 * per (theta, head_dim) with as many positions as the longest sequence.  The pages give no
 * position encoding; RoPE with theta = 500000 is the Llama-3 choice that the decoder's shapes
 * follow.  head_dim must be a multiple of 4 and theta > 1.
 */
int bi_rope_table(void* table, int64_t positions, int32_t head_dim, double theta, void* stream);

/*
 * bi_rope -- rotary position embedding, in place, rotate-half pairing (Llama form).
 *
 * x bf16: T rows of stride ld_row elements (ld_row even, x 4-byte aligned).  Each row holds
 * `heads` heads of head_dim dims at columns [h*head_dim, (h+1)*head_dim).  pos int32 [T]
 * gives each row's position p.  For pair i < head_dim/2, with (c, s) = table[p][i],
 * (a, b) = (x_i, x_{i+head_dim/2}) becomes (a c - b s, b c + a s).  The math is fp32, and each
 * result is rounded once to bf16.  table comes from bi_rope_table, with table_rows positions.
 * A position outside [0, table_rows) leaves its row unchanged and sets bit 0x1000.
 */
int bi_rope(void* x, int64_t T, int64_t ld_row, int32_t heads, int32_t head_dim, const int32_t* pos,
            const void* table, int64_t table_rows, void* stream);

/*
 * bi_kv_append -- dst[dst_row[t], :] = src[t, :] for t < T
 *
 * src bf16: T rows of stride ld_src elements, of which the first row_elems are copied.
 * dst is a packed cache, bf16 [dst_rows, row_elems].  dst_row int32 [T] must not repeat.
 * A row outside [0, dst_rows) is skipped and sets bit 0x400.  New keys and values are
 * written into the same packed layout that cached ones already have, before attention
 * reads them ("Attention" section: one layout for cached and new tokens).
 * row_elems and ld_src must be multiples of 8.
 */
int bi_kv_append(const void* src, int64_t ld_src, const int32_t* dst_row, void* dst, int64_t T,
                 int64_t row_elems, int64_t dst_rows, void* stream);

/*
 * bi_add -- h[t, :N] = bf16(h[t, :N] + d[t, :N]), in place (the residual connection).
 *
 * bf16, row strides ldh and ldd.  Each sum is formed in fp32 and rounded once.
 * N, ldh and ldd must be multiples of 8.
 */
int bi_add(void* h, int64_t ldh, const void* d, int64_t ldd, int64_t T, int64_t N, void* stream);

/*
 * bi_swiglu -- out[t, j] = bf16(silu(gu[t, j]) * gu[t, N + j]), with silu(g) = g / (1 + e^-g).
 *
 * gu bf16 [T, >= 2N] (row stride ld_gu) holds the gate and the up projections side by side,
 * as one GEMM writes them.  out bf16 [T, >= N] (row stride ld_out).  The math is fp32, with
 * one rounding.  N, ld_gu and ld_out must be multiples of 8.
 */
int bi_swiglu(const void* gu, int64_t ld_gu, void* out, int64_t ld_out, int64_t T, int64_t N, void* stream);

/*
 * bi_argmax -- out[t] = the index of the largest x[t, j], j < N (greedy decoding).
 *
 * x fp32 [T, N] (row stride ld); out int32 [T].  Ties go to the smallest index.  NaN
 * never wins; an all-NaN row gives 0.
 */
int bi_argmax(const float* x, int64_t ld, int64_t T, int64_t N, int32_t* out, void* stream);

/*
 * bi_advance -- v[i] += step for i < n (int32, wrapping as two's complement).
 *
 * The bookkeeping of a replayed greedy decode step: the positions, cache rows and KV lengths
 * of every sequence move on by one token.  Kept in the library so that a captured decode
 * step runs no device work outside it.  v int32 [n], device; n >= 0 (0 is a no-op).
 */
int bi_advance(int32_t* v, int64_t n, int32_t step, void* stream);

/*
 * bi_prefill_attn -- batch-invariant causal attention for prefill (grouped-query, variable length).
 *
 * Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section "Attention".
 * A FlashAttention-2 style kernel is batch-invariant when it splits the work over queries
 * and reduces each query's keys inside one program in an order that does not depend on the
 * batch.  The page adds that cached and new keys must share one layout.  Here the key
 * order is fixed by absolute position: blocks of 64 positions from position 0, visited in
 * ascending order with an online softmax.  A query row's bits therefore depend on its own
 * query vector, its keys and values, and nothing else.  They do not depend on:
 *   - the other sequences in the call;
 *   - how many rows of its sequence the call holds (chunked prefill, a cached prefix).
 *
 * Inputs, for B sequences:
 *   q             bf16, q_rows rows of stride ldq.  Head h of a row is columns [h*128, h*128+128).
 *                 Rows q_indptr[b] .. q_indptr[b+1]-1 belong to sequence b.
 *   q_indptr      int32 [B+1], non-decreasing, q_indptr[B] <= q_rows.
 *   q_tile_indptr int32 [B+1]: q_tile_indptr[0] = 0 and
 *                 q_tile_indptr[b+1] = q_tile_indptr[b] + ceil((q_indptr[b+1] - q_indptr[b]) / 128).
 *                 n_tiles = q_tile_indptr[B].  Built on the host with the lengths.
 *   q_pos0        int32 [B]: the position of sequence b's first query row.  Query row i of
 *                 the sequence is at position q_pos0[b] + i.
 *   k_cache,
 *   v_cache       bf16 [cache_tokens, Hkv, 128], packed.  Position p of sequence b is row
 *                 kv_indptr[b] + p.  Every position up to the sequence's last query must
 *                 already be in the cache (append first with bi_kv_append).
 *   kv_indptr     int32 [B].
 * Output:
 *   out           bf16, rows of stride ldo, the same row numbering as q; head h at
 *                 columns [h*128, h*128+128).
 *
 * Query row i attends to the keys at positions 0 .. q_pos0[b] + i:
 *   out = softmax(scale * q k^T) v.
 * Both products run on the tensor cores (tcgen05, fp32 accumulators in TMEM), one CTA per
 * (128-row query tile, query head).  Scores are fp32, and the softmax works in base 2:
 * p = 2^(s * scale * log2(e) - m), with the hardware's approximate exp2.  Each row keeps a
 * reference max m.  It raises m only when a block's max exceeds it by more than 8 (a factor
 * of 256), and then rescales the accumulated output and sum.  P.V multiplies P as a bf16
 * high part (p cut to 8 significant bits) plus the bf16-rounded remainder.  The sum of P
 * follows a fixed tree.  Values past a tile's last
 * position are zeroed before they meet a zero P.  Every choice is row-local.  Bitwise
 * invariance covers every output bit, except the sign of an output element that is exactly
 * zero.
 *
 * Constraints:
 *   - head_dim must be 128 (BI_ERR_UNSUPPORTED_SHAPE otherwise), and Hq a multiple of Hkv.
 *     q head h uses kv head h / (Hq/Hkv).
 *   - Indptr or position values outside the buffers: the tile is skipped and bit 0x800 is set.
 *   - Nothing is allocated and no workspace is needed.
 */
int bi_prefill_attn(const void* q, int64_t ldq, int64_t q_rows, const void* k_cache, const void* v_cache,
                    int64_t cache_tokens, const int32_t* q_indptr, const int32_t* q_tile_indptr, int32_t n_tiles,
                    const int32_t* kv_indptr, const int32_t* q_pos0, int32_t B, int32_t Hq, int32_t Hkv,
                    int32_t head_dim, float scale, void* out, int64_t ldo, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BI_MODEL_H */
