/*
 * bi_ctrl.h -- comparators of libbi.so.  These are NOT batch-invariant or NOT
 * deterministic, on purpose.
 *
 * They exist for two reasons: to measure what invariance costs against the faster
 * schedules it rules out, and to act as positive controls for the invariance harness.
 * Each one must show violations somewhere, or the harness could not see any.
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

#ifdef __cplusplus
}
#endif

#endif /* BI_CTRL_H */
