"""Pins for the fp64 oracle: facts fixed by the pages' definitions and by mathematics.

Every pin takes an oracle handle (the real library, or a copy compiled with a
planted mistake) and raises AssertionError when the oracle disagrees with:
closed forms, exact rational / high-precision brute force on tiny inputs,
invariants (scale, permutation, split-equals-unsplit), and special cases that
reduce to a textbook routine.  No pin calls the CUDA library; no expected value
here comes from anything but arithmetic written in this file or a cited fixture
under tests/golden/.
"""
from __future__ import annotations

import decimal
import json
import math
import os
from fractions import Fraction

import numpy as np

import oracle
from invariant_deterministic_rmsnorm_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(vals) -> np.ndarray:
    return inputs.f32_to_bf16_bits(np.asarray(vals, np.float32))


def _frac_bf16(b) -> Fraction:
    return Fraction(float(oracle.bf16_bits_to_f64(np.array([b], np.uint16))[0]))


# ============================================================ bf16 rounding
def pin_bf16_rounding_cases(h):
    """Hand-worked nearest-even cases at the ties, the subnormal edge and overflow (tests/golden/bf16_rounding.json)."""
    with open(os.path.join(GOLDEN, "bf16_rounding.json")) as f:
        cases = json.load(f)["cases"]
    L = oracle.lib(h)
    for c in cases:
        v = float.fromhex(c["value_hex"])
        got = int(L.bio_f64_to_bf16(v))
        assert got == int(c["bf16"], 16), f"bf16({c['value_hex']}) = {got:#06x}, expected {c['bf16']}"


def pin_bf16_matches_torch(h):
    """On float32 inputs, nearest-even fp64->bf16 equals torch's float32->bfloat16 conversion (a library routine)."""
    import torch
    rng = np.random.default_rng(11)
    f = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        (rng.standard_normal(2000) * 1e-38).astype(np.float32),
                        (rng.standard_normal(2000) * 1e37).astype(np.float32),
                        np.array([3.3895e38, 3.3961e38, -3.39e38, 1.17549435e-38, 9.2e-41], np.float32)])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_bf16(f.astype(np.float64), h)
    assert np.array_equal(got, ref), f"{int((got != ref).sum())} mismatches vs torch bf16"


# ============================================================ RMSNorm
def pin_rmsnorm_constant_row(h):
    """x == c everywhere gives y_j = c / sqrt(c^2 + eps) * w_j (closed form)."""
    H = 64
    eps = 1e-6
    w = inputs.normal(5, (H,), 1.0, 0.1)
    for c in (1.0, -3.5, 1e-3, 0.0009765625):
        x = np.full((1, H), c, np.float32)
        y = oracle.rmsnorm(x, w, eps, h)[0]
        cf = float(np.float32(c))
        expect = cf / math.sqrt(cf * cf + eps) * w.astype(np.float64)
        assert np.allclose(y, expect, rtol=1e-14, atol=0), (c, y[:3], expect[:3])


def pin_rmsnorm_scale_invariance(h):
    """With eps = 0, y(2^k x) == y(x) bit for bit (power-of-two scaling is exact in fp64)."""
    x, w = inputs.rmsnorm_case(3, 96, "f32", seed_x=21, seed_w=22)
    y0 = oracle.rmsnorm(x, w, 0.0, h)
    for k in (-6, 3, 20):
        yk = oracle.rmsnorm((x * np.float32(2.0 ** k)).astype(np.float32), w, 0.0, h)
        assert np.array_equal(y0, yk), k


def pin_rmsnorm_alternating_row(h):
    """A row of +a, -a, +a, ... has the same mean square as the constant row a."""
    H = 32
    w = np.ones(H, np.float32)
    a = 0.75
    alt = np.array([[a if j % 2 == 0 else -a for j in range(H)]], np.float32)
    const = np.full((1, H), a, np.float32)
    ya = oracle.rmsnorm(alt, w, 1e-6, h)[0]
    yc = oracle.rmsnorm(const, w, 1e-6, h)[0]
    assert np.array_equal(np.abs(ya), yc) and np.all(ya[1::2] < 0)


def pin_rmsnorm_brute_force_h4(h):
    """H = 4 against exact rationals and a 50-digit square root."""
    x = np.array([[0.5, -1.25, 2.0, 0.375], [3.0, 0.0, -0.0625, 1.5]], np.float32)
    w = np.array([1.0, 0.5, -2.0, 1.125], np.float32)
    eps = 1e-6
    y = oracle.rmsnorm(x, w, eps, h)
    with decimal.localcontext(decimal.Context(prec=50)):
        for m in range(2):
            ms = sum(Fraction(float(v)) ** 2 for v in x[m]) / 4 + Fraction(eps)
            root = (decimal.Decimal(ms.numerator) / decimal.Decimal(ms.denominator)).sqrt()
            for j in range(4):
                exact = decimal.Decimal(float(x[m, j])) * decimal.Decimal(float(w[j])) / root
                assert abs(float(exact) - y[m, j]) <= 4e-16 * max(1.0, abs(float(exact))), (m, j)


def pin_rmsnorm_unit_rms(h):
    """With w = 1 and eps = 0, every output row has mean square 1."""
    x, _ = inputs.rmsnorm_case(4, 256, "f32", seed_x=31)
    y = oracle.rmsnorm(x, np.ones(256, np.float32), 0.0, h)
    assert np.allclose((y * y).mean(axis=1), 1.0, rtol=1e-13, atol=0)


def pin_rmsnorm_bf16_rows_independent(h):
    """Each output row depends only on its own input row: row i of a batch equals its solo call, bit for bit."""
    x, w = inputs.rmsnorm_case(5, 128, "bf16", seed_x=41)
    yb = oracle.rmsnorm(x, w, 1e-6, h)
    for i in range(5):
        assert np.array_equal(yb[i], oracle.rmsnorm(x[i:i + 1], w, 1e-6, h)[0])


# ============================================================ GEMM
def pin_gemm_identity(h):
    """K = N, W = I gives C = A exactly."""
    A = inputs.normal_bf16(51, (5, 24))
    I = _bits(np.eye(24))
    C = oracle.gemm(A, I, h)
    assert np.array_equal(C, oracle.bf16_bits_to_f64(A))


def pin_gemm_one_hot(h):
    """Row e_k of A picks row k of W (non-square, so a transposed operand cannot pass)."""
    K, N = 12, 20
    W = inputs.normal_bf16(52, (K, N), 0, 0.02)
    A = _bits(np.eye(K)[[3, 0, 11, 7]])
    C = oracle.gemm(A, W, h)
    assert np.array_equal(C, oracle.bf16_bits_to_f64(W)[[3, 0, 11, 7]])


def pin_gemm_small_int_exact(h):
    """Small-integer operands: every product and partial sum is an integer well below 2^53, so the
    result must equal exact integer arithmetic."""
    M, N, K = 7, 9, 40
    A = inputs.small_int_bf16(53, (M, K))
    W = inputs.small_int_bf16(54, (K, N))
    C = oracle.gemm(A, W, h)
    Ai = oracle.bf16_bits_to_f64(A).astype(np.int64)
    Wi = oracle.bf16_bits_to_f64(W).astype(np.int64)
    for m in range(M):
        for n in range(N):
            assert C[m, n] == sum(int(Ai[m, k]) * int(Wi[k, n]) for k in range(K))


def pin_gemm_brute_force_tiny(h):
    """Tiny random bf16 shapes against exact rational sums (error bound K * 2^-53 * sum |a w|)."""
    M, N, K = 3, 5, 7
    A = inputs.normal_bf16(55, (M, K))
    W = inputs.normal_bf16(56, (K, N), 0, 0.02)
    C = oracle.gemm(A, W, h)
    for m in range(M):
        for n in range(N):
            terms = [_frac_bf16(A[m, k]) * _frac_bf16(W[k, n]) for k in range(K)]
            exact = sum(terms)
            bound = K * 2.0 ** -52 * float(sum(abs(t) for t in terms))
            assert abs(C[m, n] - float(exact)) <= bound + 1e-300, (m, n)


# ============================================================ LoRA
def pin_shrink_row_sum(h):
    """r = 1 and A = 1 gives t = the row sum of x (exact rationals)."""
    x = inputs.normal_bf16(61, (3, 64))
    t = oracle.lora_shrink(x, _bits(np.ones((64, 1))), h)
    for m in range(3):
        exact = sum(_frac_bf16(b) for b in x[m])
        assert abs(t[m, 0] - float(exact)) <= 64 * 2.0 ** -52 * float(sum(abs(_frac_bf16(b)) for b in x[m]))


def pin_shrink_split_equals_unsplit(h):
    """The 8-way split with an ordered combine equals the unsplit sum (exact in real arithmetic)."""
    x = inputs.normal_bf16(62, (4, 512))
    A = inputs.normal_bf16(63, (512, 16), 0, 0.02)
    t1 = oracle.lora_shrink(x, A, h)
    t8 = oracle.lora_shrink_split(x, A, 8, h)
    assert np.allclose(t1, t8, rtol=1e-13, atol=1e-15)


def pin_shrink_small_int_exact(h):
    """Small integers: the split shrink equals exact integer arithmetic, column by column."""
    M, K, r = 3, 256, 8
    x = inputs.small_int_bf16(64, (M, K))
    A = inputs.small_int_bf16(65, (K, r))
    xi = oracle.bf16_bits_to_f64(x).astype(np.int64)
    Ai = oracle.bf16_bits_to_f64(A).astype(np.int64)
    for t in (oracle.lora_shrink(x, A, h), oracle.lora_shrink_split(x, A, 8, h)):
        for m in range(M):
            for j in range(r):
                assert t[m, j] == sum(int(xi[m, k]) * int(Ai[k, j]) for k in range(K)), (m, j)


def pin_expand_one_hot(h):
    """B = one-hot row j copies bf16(t[:, j]) (nearest even) scaled into the output."""
    M, r, N = 3, 4, 8
    t = np.array([[1.00390625, 1 + 3 * 2 ** -9, -2.5, 0.1],
                  [3.0, -1.0009765625, 7.0, 1e-3],
                  [0.0, 1.0, 2.0, 3.0]], np.float32)
    Bm = np.zeros((r, N), np.float32)
    Bm[1, :] = 1.0
    y_in = _bits(np.full((M, N), 0.5))
    y = oracle.lora_expand(t, _bits(Bm), y_in, 2.0, h)
    # bf16 of t[:,1]: 1 + 3*2^-9 lies between 1 and 1+2^-7 (bf16 spacing at 1), nearer the latter;
    # -1.0009765625 = -(1 + 2^-10) rounds to -1; 1.0 is exact.
    col = np.array([1 + 2 ** -7, -1.0, 1.0])
    assert np.array_equal(y, 0.5 + 2.0 * np.repeat(col[:, None], N, axis=1))


def pin_expand_brute_force(h):
    """Random expand against exact rationals over the bf16-rounded t."""
    M, r, N = 2, 5, 6
    t = inputs.normal(66, (M, r))
    Bm = inputs.normal_bf16(67, (r, N), 0, 0.02)
    y_in = inputs.normal(68, (M, N))
    y = oracle.lora_expand(t, Bm, y_in, 0.5, h)
    tb = oracle.round_bf16(t.astype(np.float64), h)
    for m in range(M):
        for n in range(N):
            exact = Fraction(float(y_in[m, n])) + Fraction(1, 2) * sum(
                _frac_bf16(tb[m, j]) * _frac_bf16(Bm[j, n]) for j in range(r))
            assert abs(y[m, n] - float(exact)) <= 1e-15 * (1 + abs(float(exact))), (m, n)


# ============================================================ decode attention
def _attn_inputs(kv_len, Hq=8, Hkv=2, D=16, seed=71, chunk=4):
    kv_len = np.asarray(kv_len, np.int32)
    q, k, v, indptr, T = inputs.attn_case(kv_len, Hq, Hkv, D, chunk, seed)
    return q, k, v, indptr, kv_len


def pin_attn_equal_scores(h):
    """q = 0 makes every score equal: out = mean_j v_j (exact rationals)."""
    q, k, v, ip, ln = _attn_inputs([5, 9])
    q[:] = 0
    out = oracle.decode_attn(q, k, v, ip, ln, 2, 0.25, h)
    vf = oracle.bf16_bits_to_f64(v)
    for b in range(2):
        base, L = int(ip[b]), int(ln[b])
        for hh in range(8):
            g = hh // 4
            mean = vf[base:base + L, g, :].mean(axis=0)
            assert np.allclose(out[b, hh], mean, rtol=1e-14, atol=1e-15)


def pin_attn_single_token(h):
    """L = 1 gives out = v_0 whatever q and k are."""
    q, k, v, ip, ln = _attn_inputs([1, 1, 1])
    out = oracle.decode_attn(q, k, v, ip, ln, 2, 0.3, h)
    vf = oracle.bf16_bits_to_f64(v)
    for b in range(3):
        for hh in range(8):
            assert np.allclose(out[b, hh], vf[int(ip[b]), hh // 4], rtol=1e-15, atol=0)


def pin_attn_dominant_score(h):
    """One key aligned with q and a logit gap of about 100 gives out = that key's value to ~e^-100."""
    D = 16
    q, k, v, ip, ln = _attn_inputs([6], Hq=4, Hkv=1, D=D)
    q[:] = _bits(np.ones((1, 4, D)))
    kk = np.zeros((6, 1, D), np.float32)
    kk[4] = 1.0
    k[:6] = _bits(kk)
    out = oracle.decode_attn(q, k, v, ip, ln, 1, 100.0 / D, h)  # gap = 100
    vf = oracle.bf16_bits_to_f64(v)
    for hh in range(4):
        assert np.allclose(out[0, hh], vf[4, 0], rtol=0, atol=1e-40 + 1e-30 * np.abs(vf[:6, 0]).max())


def pin_attn_two_tokens_logistic(h):
    """Two keys: the weight on key 1 is the logistic function of scale * (s1 - s0)."""
    D = 8
    q, k, v, ip, ln = _attn_inputs([2], Hq=1, Hkv=1, D=D)
    qq = np.zeros((1, 1, D), np.float32); qq[0, 0, 0] = 1.0
    kk = np.zeros((2, 1, D), np.float32); kk[0, 0, 0] = 0.5; kk[1, 0, 0] = 2.0
    vv = np.zeros((2, 1, D), np.float32); vv[0, 0, :] = 0.0; vv[1, 0, :] = 1.0
    q[:] = _bits(qq); k[:2] = _bits(kk); v[:2] = _bits(vv)
    for scale in (0.1, 0.7, 3.0):
        out = oracle.decode_attn(q, k, v, ip, ln, 1, scale, h)
        p1 = 1.0 / (1.0 + math.exp(-scale * 1.5))
        assert np.allclose(out[0, 0], p1, rtol=1e-14, atol=0), scale


def pin_attn_gqa_and_offsets(h):
    """Query head h reads kv head h // (Hq/Hkv); sequence b reads only its own tokens.
    v is constant per (sequence, kv head) and q = 0, so out[b, h] = that constant."""
    kv_len = np.array([3, 7, 5], np.int32)
    Hq, Hkv, D = 8, 4, 8
    q, k, v, ip, ln = _attn_inputs(kv_len, Hq, Hkv, D, chunk=4)
    q[:] = 0
    vv = np.zeros(v.shape, np.float32)
    for b in range(3):
        for g in range(Hkv):
            vv[int(ip[b]):int(ip[b]) + int(kv_len[b]), g, :] = 10 * b + g + 1
    v[:] = _bits(vv)
    out = oracle.decode_attn(q, k, v, ip, ln, Hkv, 0.5, h)
    for b in range(3):
        for hh in range(Hq):
            # weights are 1/L (inexact in fp64): equal to the constant up to a few ulps
            assert np.allclose(out[b, hh], 10 * b + hh // (Hq // Hkv) + 1, rtol=4e-16 * 8, atol=0), (b, hh)


def pin_attn_brute_force_tiny(h):
    """L = 3, D = 4 against a 40-digit decimal softmax."""
    q, k, v, ip, ln = _attn_inputs([3], Hq=2, Hkv=1, D=4, seed=77)
    scale = 0.5
    out = oracle.decode_attn(q, k, v, ip, ln, 1, scale, h)
    qf, kf, vf = (oracle.bf16_bits_to_f64(a) for a in (q, k, v))
    with decimal.localcontext(decimal.Context(prec=40)):
        for hh in range(2):
            s = [decimal.Decimal(scale) * sum(decimal.Decimal(qf[0, hh, d]) * decimal.Decimal(kf[j, 0, d])
                                              for d in range(4)) for j in range(3)]
            e = [si.exp() for si in s]
            z = sum(e)
            for d in range(4):
                exact = sum(e[j] * decimal.Decimal(vf[j, 0, d]) for j in range(3)) / z
                assert abs(float(exact) - out[0, hh, d]) <= 1e-14 * (1 + abs(float(exact))), (hh, d)


def pin_attn_split_equals_unsplit(h):
    """The fixed-chunk split with an ordered log-sum-exp merge equals the plain softmax to ~1e-12,
    across chunk boundaries (L = chunk-1, chunk, chunk+1, 2*chunk and ragged)."""
    chunk = 16
    kv_len = np.array([15, 16, 17, 32, 45, 1], np.int32)
    q, k, v, ip, ln = _attn_inputs(kv_len, Hq=4, Hkv=2, D=8, chunk=chunk, seed=79)
    a = oracle.decode_attn(q, k, v, ip, ln, 2, 0.35, h)
    b = oracle.decode_attn_split(q, k, v, ip, ln, 2, 0.35, chunk, h)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)


def pin_attn_split_large_logits(h):
    """Chunks whose maxima differ by hundreds: the merge's rescale must not overflow or drop terms."""
    chunk = 4
    D = 4
    q, k, v, ip, ln = _attn_inputs([12], Hq=1, Hkv=1, D=D, chunk=chunk, seed=81)
    qq = np.zeros((1, 1, D), np.float32); qq[0, 0, 0] = 1.0
    kk = np.zeros((12, 1, D), np.float32)
    kk[:, 0, 0] = [0, 1, 2, 3, 300, 301, 299, 300, -50, -49, 0, 1]
    q[:] = _bits(qq); k[:12] = _bits(kk)
    a = oracle.decode_attn(q, k, v, ip, ln, 1, 1.0, h)
    b = oracle.decode_attn_split(q, k, v, ip, ln, 1, 1.0, chunk, h)
    assert np.all(np.isfinite(b)) and np.allclose(a, b, rtol=1e-12, atol=1e-14)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
