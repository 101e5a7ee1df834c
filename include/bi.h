/*
 * bi.h -- C ABI of libbi.so: batch-invariant forward kernels for NVIDIA B200 (sm_100a).
 *
 * Batch invariance: for fixed weights and fixed shape parameters (H, N, K, r, D,
 * chunk, eps, scale), the bits of output row m depend only on input row m.  They
 * do not depend on the batch size M, on the row's position in the batch, or on
 * the other rows.  Every kernel gets this by construction.  Its launch plan,
 * reduction tree, tile shape and split counts are functions of the shape
 * parameters alone, never of M.  No kernel uses floating-point atomics.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" must point to device memory (or memory the device
 *     can address) on the current CUDA device.  Pointers marked "host" are read
 *     by the CPU before the call returns.
 *   - The caller allocates and owns every buffer, workspaces included.  The
 *     library never allocates, frees or synchronises, except where an entry point
 *     says otherwise.
 *   - `stream` is a cudaStream_t passed as void*.  NULL means the legacy default
 *     stream.  Work is enqueued asynchronously on it.
 *   - Shapes, dtypes, alignment and workspace are checked on the host before any
 *     launch.  A failed check returns a status and launches nothing.  A failed
 *     launch returns BI_ERR_CUDA.  Kernels that wait on on-chip barriers give up
 *     after a bounded number of polls.  They record a code in a device error word,
 *     read back by bi_get_device_error().
 *   - An empty batch (M == 0 or B == 0) is a valid no-op and returns BI_OK.
 *   - Base pointers and row strides must be 16-byte aligned.  Otherwise the call
 *     returns BI_ERR_MISALIGNED.
 *   - Calls are thread-safe as long as their output buffers do not overlap.
 *
 * dtype codes: BI_F32 = IEEE binary32, BI_BF16 = bfloat16 (round to nearest even
 * on output).
 */
#ifndef BI_H
#define BI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bi_status {
    BI_OK = 0,
    BI_ERR_INVALID_ARG = 1,       /* null pointer, negative size, unknown dtype      */
    BI_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside what the kernel is built for      */
    BI_ERR_MISALIGNED = 3,        /* pointer or stride not 16-byte aligned           */
    BI_ERR_WORKSPACE = 4,         /* workspace missing or smaller than required      */
    BI_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed            */
    BI_ERR_TIMEOUT = 6            /* a device-side bounded wait ran out              */
} bi_status;

typedef enum bi_dtype { BI_F32 = 0, BI_BF16 = 1 } bi_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* bi_status_str(int status);

/* ABI version of this header: 1. */
int bi_abi_version(void);

/*
 * Device error word.  Kernels that spin on an mbarrier or a cluster barrier stop
 * after a bounded number of polls.  They OR a cause bit into a per-library device
 * word and return early, and their outputs are then undefined.
 * bi_get_device_error() synchronises `stream`, then reads the word into *code
 * (0 = no error).  Return value: BI_OK, BI_ERR_TIMEOUT if *code != 0, or
 * BI_ERR_CUDA.  bi_clear_device_error() zeroes the word, ordered on `stream`.
 * Bits: 0x1 a producer's wait for a free stage, 0x2 a wait for a loaded stage,
 * 0x4 a wait for the accumulator, 0x8 a cluster handshake (partials or a receive buffer of
 * another CTA of the cluster); 0x100 decode-attention
 * layout, 0x200 embedding token id, 0x400 KV-append destination row, 0x800
 * prefill-attention layout, 0x1000 RoPE position (the last five are input checks made on
 * the device).
 */
int bi_get_device_error(uint32_t* code, void* stream);
int bi_clear_device_error(void* stream);

/*
 * bi_rmsnorm -- y[m, :] = x[m, :] / sqrt(mean_j x[m, j]^2 + eps) * w
 *
 * Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section
 * "Diseño de kernels invariantes al batch", RMSNorm.  It uses a data-parallel
 * strategy: each batch element is handled by one core, with the same strategy at
 * every batch size.  The page prints no formula.  The Llama form is read here:
 * the mean is over H, eps is inside the square root, and the weight w is applied
 * as is.
 *
 *   x    device, [M, H] row-major, row stride ldx elements, dtype io_dtype
 *   w    device, [H], dtype w_dtype
 *   y    device, [M, H] row-major, row stride ldy elements, dtype io_dtype.
 *        y may alias x only if ldy == ldx (in-place).
 *   M    rows (>= 0).  H: row length, > 0, a multiple of 16 bytes' worth of
 *        elements (8 for bf16, 4 for fp32), at most 32768 (bf16) / 16384 (fp32).
 *   eps  added to the mean square inside the square root.
 *
 * Arithmetic: fp32.  Each row is reduced by one CTA.  The tree is fixed by H:
 * thread -> warp shuffle -> CTA.  Then inv = rsqrt_rn(sum/H + eps) and
 * y = (x * inv) * w, rounded once to io_dtype.
 */
int bi_rmsnorm(const void* x, const void* w, void* y, int64_t M, int64_t H, int64_t ldx, int64_t ldy,
               float eps, int io_dtype, int w_dtype, void* stream);

/*
 * bi_gemm -- C[M, N] = A[M, K] . W[K, N]
 *
 * Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section
 * "Multiplicación de matrices".  The matmul is tile-parallel over 2-D tiles on
 * tensor cores.  A split-K chosen for small batches breaks batch invariance.  The
 * remedy is to force the same kernel configuration for every batch size.
 *
 *   A    device, bf16 [M, K] row-major (K contiguous)
 *   W    device, bf16 [K, N] row-major (N contiguous), the weight
 *   C    device, [M, N] row-major, dtype c_dtype (BI_F32: the fp32 accumulator as is;
 *        BI_BF16: the accumulator rounded to nearest even)
 *   M    >= 0 rows.  N, K > 0, multiples of 8 (16-byte rows for the TMA unit).
 *   ws, ws_bytes  unused: no plan needs a workspace (bi_gemm_workspace_size and
 *        bi_gemm_counter_bytes return 0), so NULL and 0 are fine.  Kept in the signature so that
 *        callers written against a plan with a workspace stay valid.
 *
 * Arithmetic: bf16 x bf16 -> fp32 in tensor memory, K walked in ascending 64-wide
 * blocks.  The plan (tile, MMA shape, K order, split count) is a function of (N, K) and
 * the device only:
 *   - N <= 256 x (SM pairs): 256 x 256 tiles on 2-CTA clusters,
 *     tcgen05.mma.cta_group::2 256x256x16.  K may be cut into S = bi_gemm_splits(N, K)
 *     contiguous slices (S <= 4): slice s accumulates its K blocks in fp32, and the output is
 *     ((P0 + P1) + ...) + P(S-1), summed in that order in fp32 and rounded once.  The S slices
 *     of a tile run on S CTA pairs of one thread-block cluster, and their partials meet in
 *     distributed shared memory, never in HBM.  bi_ctrl_gemm_split runs other S.
 *   - wider N: 128 x 256 tiles on one CTA, tcgen05.mma.cta_group::1 128x256x16, no split.
 * Rows past M and columns past N or K are zero-filled on load and never stored.  C may
 * not alias A or W.
 */
int bi_gemm_splits(int64_t N, int64_t K);
size_t bi_gemm_counter_bytes(int64_t M, int64_t N, int64_t K);
size_t bi_gemm_workspace_size(int64_t M, int64_t N, int64_t K);
int bi_gemm(const void* A, const void* W, void* C, int64_t M, int64_t N, int64_t K, int c_dtype, void* ws,
            size_t ws_bytes, void* stream);

/*
 * bi_lora_shrink -- t[M, r] = x[M, K] . A[K, r], deterministic split-K
 *
 * Source: "Reproducible LoRA Inference Through Deterministic Split-K Reduction"
 * (abstract).  A Split-K = 8 shrink keeps its parallelism but combines the per-slice
 * FP32 partials in a fixed order instead of with floating-point atomic additions.  Its
 * FP32 output is then identical under replay.
 *
 *   x     device, bf16 [M, K] row-major
 *   A     device, bf16 [K, r] row-major (the LoRA down-projection)
 *   t     device, fp32 [M, r] row-major, overwritten
 *   r     8, 16, 32 or 64.  split_k: 1, 2, 4 or 8 (the workloads use 8).
 *         K must be a multiple of 64 * split_k.
 *   ws, ws_bytes  workspace of bi_lora_shrink_workspace_size() bytes.  That size is
 *         always 0, because the partials never leave the chip.  ws may be NULL.
 *
 * Arithmetic: slice s of K (the contiguous range [s K / split_k, (s + 1) K / split_k)) gives
 * the partial P_s, accumulated in fp32 from bf16 products in 16-deep K steps in ascending
 * order, starting from zero: with mma.sync at r = 8, 16 and 32, with tcgen05.mma (one TMEM
 * accumulator per slice) at r = 64.  t = ((P_0 + P_1) + ...) + P_{split_k - 1}, each add
 * rounded to nearest.  No atomics.  The partials meet on chip (distributed shared memory of
 * a thread-block cluster), and every CTA of the cluster adds all slices of its share of a
 * tile's rows (tiles of 128 rows at r = 8 and 64, of 64 rows at r = 16 and 32).  The arithmetic
 * depends on (K, r, split_k) only; neither the tile height nor the cluster shape of the r = 64
 * kernel (split_k CTAs of one slice, or split_k / 2 of two, by the number of tiles) changes a
 * row's bits.
 */
size_t bi_lora_shrink_workspace_size(int64_t M, int64_t K, int32_t r, int32_t split_k);
int bi_lora_shrink(const void* x, const void* A, float* t, int64_t M, int64_t K, int32_t r, int32_t split_k,
                   void* ws, size_t ws_bytes, void* stream);

/*
 * bi_rmsnorm_lora_shrink -- y = RMSNorm(x) . w and t = y . A in one pass
 *
 * Sources: the RMSNorm section of "Defeating Nondeterminism in LLM Inference" (Spanish
 * summary, "Diseño de kernels invariantes al batch") and "Reproducible LoRA Inference Through
 * Deterministic Split-K Reduction" (abstract).  The fused form of bi_rmsnorm followed by
 * bi_lora_shrink on its output, for the case where the normalised rows feed a LoRA-adapted
 * projection: the CTA that normalises a row multiplies it by A from its shared memory, so the
 * shrink does not read y back from HBM.
 *
 *   x, y  device, bf16 [M, H] with row strides ldx, ldy (elements); y may equal x (then ldy = ldx)
 *   w     device, bf16 [H], the RMSNorm weight
 *   A     device, bf16 [H, r] row-major, the LoRA down-projection
 *   t     device, fp32 [M, r] row-major, overwritten
 *   H     4096; r 8 or 16; split_k 8.  Other shapes give BI_ERR_UNSUPPORTED_SHAPE: call bi_rmsnorm
 *         and bi_lora_shrink instead, which give the same bits.
 *   x, y, w, A, t 16-byte aligned, ldx and ldy multiples of 8.
 *
 * Arithmetic: y is bitwise bi_rmsnorm(x, w, eps) (bf16 in and out, bf16 weight) and t is
 * bitwise bi_lora_shrink(y, A, r, split_k): every element goes through the same operations in
 * the same order (bi_rmsnorm's per-row reduction tree for H = 4096; per K slice an mma.sync
 * chain of 16-deep steps from zero, then ((P_0 + P_1) + ...) + P_7).  Batch-invariant like
 * both.  Persistent CTAs walk 8-row tiles; which CTA takes a tile never changes a row's
 * arithmetic.
 */
int bi_rmsnorm_lora_shrink(const void* x, const void* w, void* y, const void* A, float* t, int64_t M, int64_t H,
                           int64_t ldx, int64_t ldy, float eps, int32_t r, int32_t split_k, void* stream);

/*
 * bi_lora_expand -- y[M, N] += scale * bf16(t)[M, r] . B[r, N], in place
 *
 * Source: the same abstract ("low-rank LoRA multiplications").  The low-rank product
 * is added to the base layer's output.
 *
 *   t     device, fp32 [M, r] row-major (the shrink output).  It enters the product
 *         rounded to bf16, nearest even.
 *   B     device, bf16 [r, N] row-major (the LoRA up-projection)
 *   y     device, [M, N] with row stride ldy elements, dtype y_dtype, read and written
 *   r     8, 16, 32 or 64.  N: a multiple of 8.  scale: the LoRA scaling (alpha / r).
 *
 * Arithmetic: mma.sync, bf16 in, fp32 accumulate over r.  Then
 * y = round_to_y_dtype(fma(scale, delta, y)), elementwise.
 */
int bi_lora_expand(const float* t, const void* B, void* y, int64_t M, int32_t r, int64_t N, int64_t ldy,
                   float scale, int y_dtype, void* stream);

/*
 * bi_decode_attn -- one decode step of grouped-query attention over a packed KV cache,
 * split-KV with a FIXED split size.
 *
 * Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), section
 * "Attention".  Split-KV (FlashDecoding) keeps the same reduction order if the split
 * SIZE is fixed rather than the number of splits.  Cached and new keys/values share one
 * consistent layout.
 *
 *   q          device, bf16 [B, Hq, head_dim], one query token per sequence
 *   k, v       device, bf16 [total_tokens, Hkv, head_dim], the packed cache
 *   kv_indptr  device, int32 [B + 1], non-decreasing.  Sequence b owns tokens
 *              kv_indptr[b] .. kv_indptr[b] + kv_len[b] - 1.  Every kv_indptr[b] must be
 *              a multiple of `chunk` and kv_indptr[B] <= total_tokens.  Tokens between
 *              the end of a sequence and kv_indptr[b+1] are never read.
 *   kv_len     device, int32 [B], 1 <= kv_len[b] <= kv_indptr[b+1] - kv_indptr[b]
 *   Hq, Hkv    query / kv heads.  Hq / Hkv must be 1, 2, 4 or 8.  Query head h reads kv
 *              head h / (Hq / Hkv).  head_dim must be 128.  chunk must be 256.
 *   scale      score scale, usually 1/sqrt(head_dim)
 *   out        device, [B, Hq, head_dim], dtype out_dtype
 *   ws         device workspace of at least bi_decode_attn_workspace_size(total_tokens,
 *              Hq, head_dim, chunk) bytes, 16-byte aligned.  It holds one fp32 partial
 *              (head_dim values, the running max and the sum) per (256-token slot of the
 *              cache, query head).  Its contents need no initialisation and are
 *              overwritten.
 *
 * Arithmetic: chunk c of sequence b is its tokens [256c, min(256c + 256, L_b)).  Each
 * chunk yields m_c = max s_j, l_c = sum exp(s_j - m_c) and o_c = sum exp(s_j - m_c) v_j,
 * with s_j = scale * q . k_j (bf16 products, fp32 sums over fixed trees).  The chunks are
 * merged in order c = 0, 1, ... with an fp32 log-sum-exp rescale, and out = o / l.
 *
 * Layout violations that only the device can see (kv_indptr negative or not chunk-aligned,
 * kv_len out of range, kv_indptr[b + 1] > total_tokens) set bit 0x100 of the device error
 * word.  The affected rows of out are then left unwritten; the other rows are computed as
 * usual.  A decreasing kv_indptr (sequences that overlap) also sets bit 0x100 and voids the
 * whole call: no chunk is computed and out holds no result.
 *
 * Work split: the live chunks of the batch (ceil(kv_len[b] / 256) per sequence), not the
 * cache's capacity, are divided among the persistent CTAs, so a few requests in a large
 * cache still use every SM.  Which CTA computes a chunk never changes its arithmetic.
 */
size_t bi_decode_attn_workspace_size(int64_t total_tokens, int32_t Hq, int32_t head_dim, int32_t chunk);
int bi_decode_attn(const void* q, const void* k, const void* v, const int32_t* kv_indptr, const int32_t* kv_len,
                   int32_t B, int64_t total_tokens, int32_t Hq, int32_t Hkv, int32_t head_dim, float scale,
                   int32_t chunk, void* out, int out_dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * bi_decode_attn_noalloc -- bi_decode_attn without a caller-provided workspace.
 *
 * The pages have no counterpart for this entry point.  It exists for callers that
 * cannot allocate device memory.  Examples: a plugin interface that hands the kernel
 * only its input and output buffers and offers no allocator; a serving process whose
 * memory pool already owns all of the GPU's free memory; a latency-critical loop where
 * cudaMalloc's implicit device synchronisation is not acceptable.
 *
 * Arguments, layout, arithmetic and results are those of bi_decode_attn, minus ws and
 * ws_bytes.  The per-chunk partials live in one fixed array of
 * BI_DECODE_ATTN_NOALLOC_SCRATCH_BYTES (16 MiB) of device memory inside libbi.so.  Every
 * GPU that loads the library holds that array until the process exits.  The call
 * allocates and frees nothing.
 *
 *   - Limit: the partials need bi_decode_attn_workspace_size(total_tokens, Hq, 128, 256)
 *     bytes.  Beyond 16 MiB the call returns BI_ERR_WORKSPACE and launches nothing.
 *     At Hq = 32 that is about 258,000 cache tokens; use bi_decode_attn for larger caches.
 *   - The first call on each device looks up the array's device address with that
 *     device current, then caches it.  Make that first call before any stream capture.  A
 *     lookup that fails returns BI_ERR_CUDA and is tried again by the next call.
 *   - A sequence whose kv_indptr[b + 1] exceeds total_tokens is a layout error (bit 0x100,
 *     row left unwritten), as in bi_decode_attn: the call never reads partials it did not
 *     write in this call.
 *   - Every call on a device shares the one array, which keeps whatever the last call
 *     left there.  Nothing in it needs to start at zero.  Calls whose work overlaps on
 *     the GPU (on different streams, or from different host threads without ordering)
 *     race on the array and corrupt each other's results: serialise them.
 */
#define BI_DECODE_ATTN_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int bi_decode_attn_noalloc(const void* q, const void* k, const void* v, const int32_t* kv_indptr,
                           const int32_t* kv_len, int32_t B, int64_t total_tokens, int32_t Hq, int32_t Hkv,
                           int32_t head_dim, float scale, int32_t chunk, void* out, int out_dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BI_H */
