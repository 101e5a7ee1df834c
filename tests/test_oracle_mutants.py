"""Each plausible mistake planted in a copy of the oracle must fail at least one pin.

The copy is compiled on the CPU from an edited source text; the oracle file
itself is never changed.  A mutant that every pin still passes would mean the
pins cannot see that kind of error.
"""
import os
import re

import pytest

import oracle
import oracle_pins

# (name, function the edit is confined to, old text, new text)
MUTANTS = [
    ("rms_sum_not_mean", "bio_rmsnorm", "ss / (double)H + eps", "ss + eps"),
    ("rms_eps_outside_sqrt", "bio_rmsnorm", "1.0 / sqrt(ss / (double)H + eps)", "1.0 / (sqrt(ss / (double)H) + eps)"),
    ("rms_one_plus_w", "bio_rmsnorm", "* inv * load(w, w_dtype, j)", "* inv * (1.0 + load(w, w_dtype, j))"),
    ("rms_no_sqrt", "bio_rmsnorm", "1.0 / sqrt(ss / (double)H + eps)", "1.0 / (ss / (double)H + eps)"),
    ("rms_divide_h_minus_1", "bio_rmsnorm", "ss / (double)H", "ss / (double)(H - 1)"),
    ("gemm_transposed_w", "bio_gemm", "W[k * N + n]", "W[n * K + k]"),
    ("gemm_dropped_first_k", "bio_gemm", "for (int64_t k = 0; k < K; ++k)", "for (int64_t k = 1; k < K; ++k)"),
    ("gemm_wrong_a_row", "bio_gemm", "A[m * K + k]", "A[(m * K + k + K) % (M * K)]"),
    ("shrink_transposed_a", "bio_lora_shrink(", "A[k * r + j]", "A[j * K + k]"),
    ("split_keeps_last_partial", "bio_lora_shrink_split", "total += part", "total = part"),
    ("split_wrong_slice", "bio_lora_shrink_split", "k < (s + 1) * ks", "k < (s + 1) * ks - 1"),
    ("expand_no_bf16_round", "bio_lora_expand", "bio_bf16_to_f64(bio_f64_to_bf16((double)t[m * r + j]))",
     "(double)t[m * r + j]"),
    ("expand_no_scale", "bio_lora_expand", "+ scale * acc", "+ acc"),
    ("expand_subtract", "bio_lora_expand", "+ scale * acc", "- scale * acc"),
    ("attn_gqa_modulo", "bio_decode_attn(", "int64_t g = h / group;", "int64_t g = h % Hkv;"),
    ("attn_no_scale", "bio_decode_attn(", "s *= scale;", ""),
    ("attn_no_max_shift_sign", "bio_decode_attn(", "exp(s_scratch[j] - mx) / denom", "exp(mx - s_scratch[j]) / denom"),
    ("attn_base_ignored", "bio_decode_attn(", "int64_t base = kv_indptr[b], L = kv_len[b];",
     "int64_t base = 0, L = kv_len[b];"),
    ("attn_drop_last_token", "bio_decode_attn(", "for (int64_t j = 0; j < L; ++j) denom", "for (int64_t j = 0; j < L - 1; ++j) denom"),
    ("split_no_rescale_old", "bio_decode_attn_split", "o[d] = o[d] * a + o_scratch[d] * bsc", "o[d] = o[d] + o_scratch[d] * bsc"),
    ("split_l_not_rescaled", "bio_decode_attn_split", "l_run = l_run * a + lc * bsc", "l_run = l_run + lc * bsc"),
    ("split_last_chunk_dropped", "bio_decode_attn_split", "int64_t c1 = c0 + chunk < L ? c0 + chunk : L;",
     "int64_t c1 = c0 + chunk < L ? c0 + chunk : (L > c0 + 1 ? L - 1 : L);"),
    ("bf16_truncate", "bio_f64_to_bf16", "nearbyint(a / q)", "floor(a / q)"),
    ("bf16_round_half_up", "bio_f64_to_bf16", "nearbyint(a / q)", "floor(a / q + 0.5)"),
    ("bf16_one_bit_short", "bio_f64_to_bf16", "ue - 7", "ue - 6"),
    ("bf16_no_subnormal_clamp", "bio_f64_to_bf16", "if (ue < -126) ue = -126;", ""),
]


def _function_span(src: str, name: str):
    m = re.search(r"^(?:void|int|double|float|uint16_t)\s+" + re.escape(name.rstrip("(")) + r"\(", src, re.M)
    start = m.start()
    # the body runs from the first "{" after the signature to its matching "}"
    i = src.index("{", start)
    depth = 0
    for j in range(i, len(src)):
        if src[j] == "{":
            depth += 1
        elif src[j] == "}":
            depth -= 1
            if depth == 0:
                return start, j + 1
    raise ValueError(name)


def _mutate(src: str, fn: str, old: str, new: str) -> str:
    a, b = _function_span(src, fn)
    body = src[a:b]
    assert old in body, f"mutation anchor {old!r} not found in {fn}"
    return src[:a] + body.replace(old, new) + src[b:]


@pytest.mark.parametrize("name,fn,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, fn, old, new, tmp_path):
    src = _mutate(oracle.source_text(), fn, old, new)
    handle = oracle.compile_variant(src, str(tmp_path / f"mut_{name}.so"))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(handle)
        except AssertionError:
            failed.append(pin.__name__)
        except (ValueError, FloatingPointError, OverflowError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name!r} passed every pin"
