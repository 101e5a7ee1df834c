/*
 * bi_ctrl.h -- comparators and instruments of libbi.so.
 *
 * The comparators are NOT batch-invariant or NOT deterministic, on purpose.  They exist for
 * two reasons: to measure what invariance costs against the faster schedules it rules out,
 * and to act as positive controls for the invariance harness.  Each one must show
 * violations somewhere, or the harness could not see any.
 *
 * Two instruments sit beside them: bi_ctrl_gemm_split runs bi_gemm's kernel at a split
 * count the plan does not choose (batch-invariant for a fixed count), and
 * bi_ctrl_wait_timeout_probe drives the bounded-wait failure path.
 * Conventions are those of bi.h.
 */
#ifndef BI_CTRL_H
#define BI_CTRL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * bi_ctrl_lora_shrink_atomic -- the shrink of bi_lora_shrink, with the split_k partials
 * added into t by floating-point atomics, in whatever order the CTAs finish.  This is
 * the nondeterministic baseline of "Reproducible LoRA Inference Through Deterministic
 * Split-K Reduction" (abstract).  t is zeroed on `stream` first.
 */
int bi_ctrl_lora_shrink_atomic(const void* x, const void* A, float* t, int64_t M, int64_t K, int32_t r,
                               int32_t split_k, void* stream);

/*
 * bi_ctrl_lora_shrink_tc -- the shrink on tcgen05 at r = 16, 32 or 64: the same K slices and
 * slice-ordered on-chip combine as bi_lora_shrink, with each slice's partial accumulated by
 * tcgen05.mma (M = 128 rows, N = r, K = 16) in its own TMEM accumulator.  A cluster holds
 * split_k CTAs of one slice each while the row tiles fit the GPU's clusters of that size in one
 * round, else split_k / 2 CTAs of two slices each (same bits either way); the partials cross
 * the cluster as bulk shared-memory copies and four warps per CTA combine them.  At r = 64 it
 * is bi_lora_shrink's kernel (bitwise the same call).  At r = 16 and 32 it is the study behind
 * keeping mma.sync there: slower at r = 16, within a few percent at r = 32.  Batch-invariant and
 * deterministic; at r = 16 and 32 its bits differ from bi_lora_shrink's in the last places (a
 * different accumulation inside the 16-deep steps).  Arguments as bi_lora_shrink; r must be 16,
 * 32 or 64.
 */
int bi_ctrl_lora_shrink_tc(const void* x, const void* A, float* t, int64_t M, int64_t K, int32_t r, int32_t split_k,
                           void* stream);

/*
 * bi_ctrl_rmsnorm_split -- RMSNorm whose row reduction is cut across S CTAs of a
 * thread-block cluster, S in {1, 2, 4, 8}, chosen from M (more pieces for smaller batches).
 * It is the small-batch "split reduction" that "Defeating Nondeterminism in LLM
 * Inference" (Spanish summary, section "Diseño de kernels invariantes al batch",
 * RMSNorm) names as the strategy that sacrifices batch invariance.  Arguments as
 * bi_rmsnorm.  The row length H must split into slices of at most 1024 16-byte vectors,
 * and M <= 65535.
 */
int bi_ctrl_rmsnorm_split(const void* x, const void* w, void* y, int64_t M, int64_t H, int64_t ldx, int64_t ldy,
                          float eps, int io_dtype, int w_dtype, void* stream);

/*
 * bi_ctrl_gemm_splitk -- bi_gemm with a split-K chosen from M, the batch-size-dependent
 * strategy of the "Multiplicación de matrices" section of the same page.  When the batch
 * alone yields too few output tiles to fill the GPU, K is cut into S in {2, 4, 8} slices.
 * Each slice runs bi_gemm's tile kernel unsplit into fp32 partials in ws (S = 1: the whole
 * product, straight into C).  The partials are then added in slice order and rounded to
 * c_dtype.  A row's accumulation order therefore depends on M.
 * ws must hold bi_ctrl_gemm_splitk_workspace_size(M, N, K) bytes (0 when S = 1).
 */
size_t bi_ctrl_gemm_splitk_workspace_size(int64_t M, int64_t N, int64_t K);
int bi_ctrl_gemm_splitk(const void* A, const void* W, void* C, int64_t M, int64_t N, int64_t K, int c_dtype,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * bi_ctrl_gemm_split -- bi_gemm with the K split count given by the caller instead of
 * bi_gemm_splits(N, K): the plan study behind that choice.  For a fixed `splits` it is
 * batch-invariant like bi_gemm; it is here to time the plan's candidates against each
 * other at every batch size.  splits in 1 .. 4 and at most ceil(K / 64); a weight too wide
 * for the CTA-pair tiles takes splits = 1 only (BI_ERR_UNSUPPORTED_SHAPE otherwise).
 * splits = 1 runs the CTA-pair kernel; splits > 1 runs the cluster-split kernel (bi.h, bi_gemm).
 * No workspace is needed: bi_ctrl_gemm_split_workspace_size returns 0, and ws may be NULL.
 */
size_t bi_ctrl_gemm_split_workspace_size(int64_t M, int64_t N, int64_t K, int32_t splits);
int bi_ctrl_gemm_split(const void* A, const void* W, void* C, int64_t M, int64_t N, int64_t K, int c_dtype,
                       int32_t splits, void* ws, size_t ws_bytes, void* stream);

/*
 * bi_ctrl_decode_attn_adaptive -- bi_decode_attn with the split size chosen from the
 * batch: 128-token chunks when B < 16, 256 otherwise.  That is the batch-dependent
 * split-KV which the "Attention" section of the same page warns against.  Arguments as
 * bi_decode_attn (head_dim 128).  ws must hold
 * bi_ctrl_decode_attn_adaptive_workspace_size(total_tokens, Hq) bytes.
 */
size_t bi_ctrl_decode_attn_adaptive_workspace_size(int64_t total_tokens, int32_t Hq);
int bi_ctrl_decode_attn_adaptive(const void* q, const void* k, const void* v, const int32_t* kv_indptr,
                                 const int32_t* kv_len, int32_t B, int64_t total_tokens, int32_t Hq, int32_t Hkv,
                                 float scale, void* out, int out_dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * bi_ctrl_wait_timeout_probe -- exercises the failure path that every kernel's bounded waits
 * share, without a fault.  One CTA waits on an mbarrier that nothing arrives on.  After
 * limit_ns (1 us .. 2 s) the wait gives up, bit 0x2 is OR-ed into the device error word
 * (bi_get_device_error), and the kernel returns.  The CUDA context stays usable.  Tests use
 * it to check the path from a device-side timeout to the host-visible status.
 */
int bi_ctrl_wait_timeout_probe(uint64_t limit_ns, void* stream);

/*
 * bi_ctrl_set_pdl -- turn programmatic dependent launch on (enable != 0, the default) or off for
 * the library's later launches; returns the previous setting.  With it on, a kernel may begin
 * its set-up (barriers, tensor memory, descriptor prefetch) while the kernel before it on the
 * stream finishes, and waits for that kernel before it touches global memory.  It changes when
 * work starts, never what is computed: outputs are bitwise the same either way.  Here to
 * measure what the overlap gains.  Process-wide; not synchronised with launches in flight.
 */
int bi_ctrl_set_pdl(int enable);

#ifdef __cplusplus
}
#endif

#endif /* BI_CTRL_H */
