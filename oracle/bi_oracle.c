/*
 * bi_oracle.c -- plain, slow, fp64 CPU oracle for the batch-invariant forward ops.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this file.  Only the test suite, the smoke check and the bench's
 * CPU-baseline / reference leg use it.  It shares no code, header, table or
 * helper with the CUDA kernels: it decodes bfloat16 itself, rounds to bfloat16
 * itself, and accumulates every reduction in IEEE double, sequentially, in index
 * order.
 *
 * What each function computes, and the passage it follows:
 *
 *  - bio_rmsnorm: "Defeating Nondeterminism in LLM Inference" (Spanish summary,
 *    es.news.hada.io), section "Diseño de kernels invariantes al batch", RMSNorm.
 *    The page gives no formula; the plain Llama-style reading is used:
 *    y_j = x_j / sqrt(mean_j(x_j^2) + eps) * w_j, mean over H (not H-1), eps
 *    inside the square root, weight applied as w (not 1+w).
 *  - bio_gemm: same page, "Multiplicación de matrices": C = A . W, bf16 operands,
 *    accumulated here in fp64 (the page's tiled tensor-core schedule reaches the
 *    same real-number result).
 *  - bio_lora_shrink / bio_lora_shrink_split: "Reproducible LoRA Inference Through
 *    Deterministic Split-K Reduction", abstract: t = x . A with FP32 shrink output;
 *    the split-K=8 variant forms per-slice partials and combines them in slice
 *    order, which in real arithmetic equals the unsplit sum.
 *  - bio_lora_expand: the same abstract ("low-rank LoRA multiplications"): the
 *    low-rank product added to the base output, y += scale * bf16(t) . B.
 *  - bio_decode_attn / bio_decode_attn_split: "Defeating Nondeterminism in LLM
 *    Inference", section "Attention": decode attention; the split-KV (FlashDecoding)
 *    form with a fixed split size merges per-chunk (max, sum, unnormalised output)
 *    triples in chunk order with a log-sum-exp rescale.  The unsplit softmax is the
 *    plain definition; the split form is the method's steps in fp64.
 *
 * dtype codes: 0 = float32, 1 = bfloat16 (raw 16-bit patterns, uint16).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define BIO_F32 0
#define BIO_BF16 1

/* ---- number formats --------------------------------------------------- */

/* bfloat16 -> double: the 16 bits are the top half of an IEEE binary32. */
double bio_bf16_to_f64(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * double -> bfloat16, round to nearest, ties to even, in one rounding step from
 * the double value (8 significand bits kept).  Written from the IEEE definition:
 * scale into [2^7, 2^8) by the binade, round the significand with nearbyint()
 * (default mode = ties-to-even), rebuild.  Subnormal bf16 results use the fixed
 * quantum 2^-133; overflow gives infinity.  NaN maps to the quiet NaN 0x7FC0.
 */
uint16_t bio_f64_to_bf16(double v)
{
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    (void)frexp(a, &e);             /* a = f * 2^e, f in [0.5, 1) */
    int ue = e - 1;                  /* a in [2^ue, 2^(ue+1)) */
    if (ue < -126) ue = -126;        /* subnormal range: fixed quantum */
    double q = ldexp(1.0, ue - 7);   /* spacing of bf16 values in this binade */
    double r = nearbyint(a / q) * q; /* a/q is exact (power-of-two scaling) */
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80; /* overflow to inf */
    /* r is now exactly a bf16 value; encode it through binary32. */
    float f = (float)r;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

/* double -> float32 round to nearest even (the C conversion under the default mode). */
float bio_f64_to_f32(double v) { return (float)v; }

/* Round every element of an fp64 array to bf16 bits / to float32. */
void bio_round_bf16(const double* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = bio_f64_to_bf16(in[i]);
}
void bio_round_f32(const double* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = bio_f64_to_f32(in[i]);
}

static double load(const void* p, int dtype, int64_t i)
{
    if (dtype == BIO_F32) return (double)((const float*)p)[i];
    return bio_bf16_to_f64(((const uint16_t*)p)[i]);
}

/* ---- RMSNorm ----------------------------------------------------------- */

/* y[m, j] = x[m, j] / sqrt(sum_j x[m, j]^2 / H + eps) * w[j], all in fp64.
   x row m starts at element m*ldx; y row m at m*ldy. */
void bio_rmsnorm(const void* x, int x_dtype, const void* w, int w_dtype, double* y,
                 int64_t M, int64_t H, int64_t ldx, int64_t ldy, double eps)
{
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t j = 0; j < H; ++j) {
            double v = load(x, x_dtype, m * ldx + j);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)H + eps);
        for (int64_t j = 0; j < H; ++j)
            y[m * ldy + j] = load(x, x_dtype, m * ldx + j) * inv * load(w, w_dtype, j);
    }
}

/* ---- dense GEMM -------------------------------------------------------- */

/* C[m, n] = sum_k A[m, k] * W[k, n]; A [M,K] and W [K,N] row-major bf16 bits. */
void bio_gemm(const uint16_t* A, const uint16_t* W, double* C, int64_t M, int64_t N, int64_t K)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += bio_bf16_to_f64(A[m * K + k]) * bio_bf16_to_f64(W[k * N + n]);
            C[m * N + n] = acc;
        }
}

/* ---- LoRA -------------------------------------------------------------- */

/* t[m, j] = sum_k x[m, k] * A[k, j]; x [M,K], A [K,r] row-major bf16 bits. */
void bio_lora_shrink(const uint16_t* x, const uint16_t* A, double* t, int64_t M, int64_t K, int64_t r)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += bio_bf16_to_f64(x[m * K + k]) * bio_bf16_to_f64(A[k * r + j]);
            t[m * r + j] = acc;
        }
}

/* Split-K form: K is cut into `split` contiguous slices of K/split; slice s gives
   a partial P_s over its own columns; the partials are then combined in slice
   order s = 0, 1, ..., split-1.  Requires K % split == 0. */
int bio_lora_shrink_split(const uint16_t* x, const uint16_t* A, double* t, int64_t M, int64_t K,
                          int64_t r, int64_t split)
{
    if (split <= 0 || K % split != 0) return 1;
    int64_t ks = K / split;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < r; ++j) {
            double total = 0.0;
            for (int64_t s = 0; s < split; ++s) {
                double part = 0.0;
                for (int64_t k = s * ks; k < (s + 1) * ks; ++k)
                    part += bio_bf16_to_f64(x[m * K + k]) * bio_bf16_to_f64(A[k * r + j]);
                total += part;
            }
            t[m * r + j] = total;
        }
    return 0;
}

/* y_out[m, n] = y_in[m, n] + scale * sum_j bf16(t[m, j]) * B[j, n].
   t is the float32 shrink output; it enters the low-rank product rounded to
   bf16 (round to nearest even), the declared input precision of the expand.
   y_in is float32 or bf16 [M, N]; B [r, N] bf16 bits. */
void bio_lora_expand(const float* t, const uint16_t* B, const void* y_in, int y_dtype, double* y_out,
                     int64_t M, int64_t r, int64_t N, double scale)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < r; ++j) {
                double tb = bio_bf16_to_f64(bio_f64_to_bf16((double)t[m * r + j]));
                acc += tb * bio_bf16_to_f64(B[j * N + n]);
            }
            y_out[m * N + n] = load(y_in, y_dtype, m * N + n) + scale * acc;
        }
}

/* ---- decode attention -------------------------------------------------- */

/*
 * One decode query per sequence b.  q [B, Hq, D] bf16; k, v packed [T, Hkv, D]
 * bf16 with sequence b at tokens kv_indptr[b] .. kv_indptr[b] + kv_len[b] - 1.
 * Query head h reads kv head h / (Hq / Hkv).  out [B, Hq, D] fp64.
 * Plain softmax: s_j = scale * q . k_j ; p = softmax(s) ; out = sum_j p_j v_j.
 */
int bio_decode_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* kv_indptr,
                    const int32_t* kv_len, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, double scale,
                    double* out, double* s_scratch /* at least max kv_len doubles */)
{
    if (Hkv <= 0 || Hq % Hkv != 0) return 1;
    int64_t group = Hq / Hkv;
    for (int64_t b = 0; b < B; ++b) {
        int64_t base = kv_indptr[b], L = kv_len[b];
        if (L <= 0) return 2;
        for (int64_t h = 0; h < Hq; ++h) {
            int64_t g = h / group;
            const uint16_t* qh = q + (b * Hq + h) * D;
            double mx = -INFINITY;
            for (int64_t j = 0; j < L; ++j) {
                const uint16_t* kj = k + ((base + j) * Hkv + g) * D;
                double s = 0.0;
                for (int64_t d = 0; d < D; ++d) s += bio_bf16_to_f64(qh[d]) * bio_bf16_to_f64(kj[d]);
                s *= scale;
                s_scratch[j] = s;
                if (s > mx) mx = s;
            }
            double denom = 0.0;
            for (int64_t j = 0; j < L; ++j) denom += exp(s_scratch[j] - mx);
            double* o = out + (b * Hq + h) * D;
            for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t j = 0; j < L; ++j) {
                double p = exp(s_scratch[j] - mx) / denom;
                const uint16_t* vj = v + ((base + j) * Hkv + g) * D;
                for (int64_t d = 0; d < D; ++d) o[d] += p * bio_bf16_to_f64(vj[d]);
            }
        }
    }
    return 0;
}

/*
 * Split-KV form with a fixed split size `chunk` (tokens [c*chunk, min((c+1)*chunk, L))):
 * per chunk c: m_c = max s_j, l_c = sum e^(s_j - m_c), o_c = sum e^(s_j - m_c) v_j
 * (unnormalised); then for c = 0, 1, ... in order:
 *   m' = max(m, m_c); l = l e^(m - m') + l_c e^(m_c - m'); o = o e^(m - m') + o_c e^(m_c - m')
 * and out = o / l.  Same arguments as bio_decode_attn; o_scratch holds D doubles.
 */
int bio_decode_attn_split(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* kv_indptr,
                          const int32_t* kv_len, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, double scale,
                          int64_t chunk, double* out, double* o_scratch)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || chunk <= 0) return 1;
    int64_t group = Hq / Hkv;
    for (int64_t b = 0; b < B; ++b) {
        int64_t base = kv_indptr[b], L = kv_len[b];
        if (L <= 0) return 2;
        for (int64_t h = 0; h < Hq; ++h) {
            int64_t g = h / group;
            const uint16_t* qh = q + (b * Hq + h) * D;
            double m_run = -INFINITY, l_run = 0.0;
            double* o = out + (b * Hq + h) * D;
            for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t c0 = 0; c0 < L; c0 += chunk) {
                int64_t c1 = c0 + chunk < L ? c0 + chunk : L;
                /* chunk max */
                double mc = -INFINITY;
                for (int64_t j = c0; j < c1; ++j) {
                    const uint16_t* kj = k + ((base + j) * Hkv + g) * D;
                    double s = 0.0;
                    for (int64_t d = 0; d < D; ++d) s += bio_bf16_to_f64(qh[d]) * bio_bf16_to_f64(kj[d]);
                    s *= scale;
                    if (s > mc) mc = s;
                }
                /* chunk sum and unnormalised output */
                double lc = 0.0;
                for (int64_t d = 0; d < D; ++d) o_scratch[d] = 0.0;
                for (int64_t j = c0; j < c1; ++j) {
                    const uint16_t* kj = k + ((base + j) * Hkv + g) * D;
                    const uint16_t* vj = v + ((base + j) * Hkv + g) * D;
                    double s = 0.0;
                    for (int64_t d = 0; d < D; ++d) s += bio_bf16_to_f64(qh[d]) * bio_bf16_to_f64(kj[d]);
                    s *= scale;
                    double e = exp(s - mc);
                    lc += e;
                    for (int64_t d = 0; d < D; ++d) o_scratch[d] += e * bio_bf16_to_f64(vj[d]);
                }
                /* ordered log-sum-exp merge */
                double mn = m_run > mc ? m_run : mc;
                double a = (m_run == -INFINITY) ? 0.0 : exp(m_run - mn);
                double bsc = exp(mc - mn);
                l_run = l_run * a + lc * bsc;
                for (int64_t d = 0; d < D; ++d) o[d] = o[d] * a + o_scratch[d] * bsc;
                m_run = mn;
            }
            for (int64_t d = 0; d < D; ++d) o[d] /= l_run;
        }
    }
    return 0;
}
