"""Pins of the decoder oracle (oracle/decoder.py) to things other than itself.

  * closed forms: RoPE at position 0 is the identity, a unit vector is turned by the textbook
    angle, the SwiGLU odd part silu(g) - silu(-g) = g, attention over one key returns its value;
  * invariants: RoPE keeps pair norms and depends on relative position only; the oracle
    decoder gives a sequence the same bits alone, batched, and prefilled in chunks;
  * special cases: with every projection into the residual stream zeroed the decoder reduces
    to the final RMSNorm and the vocabulary projection of the embedding;
  * brute force: a scalar pure-Python decoder (complex-number rotation, explicit softmax
    loops, its own bf16 rounding) on tiny dims agrees to 1e-9;
  * planted mistakes: each edit of the oracle source that a plausible slip would make fails
    one of the pins above.
"""
import cmath
import math
import struct
import types

import numpy as np
import pytest

import oracle
from oracle import decoder as od
from invariant_deterministic_rmsnorm_b200 import inputs


def _bits(vals):
    return inputs.f32_to_bf16_bits(np.asarray(vals, np.float32))


# ------------------------------------------------------------------ RoPE
def test_rope_position_zero_is_identity():
    x = inputs.normal_bf16(11, (3, 2 * 8))
    out = od.rope(x, np.zeros(3, np.int32), 2, 8, 500000.0)
    assert np.array_equal(out, oracle.bf16_bits_to_f64(x))


def test_rope_turns_unit_vectors_by_the_textbook_angle():
    # head_dim 4, theta 16: pair 0 (dims 0, 2) turns by p, pair 1 (dims 1, 3) by p * 16^(-1/2) = p / 4
    e0 = _bits([[1, 0, 0, 0]])
    e1 = _bits([[0, 1, 0, 0]])
    p = np.array([4], np.int32)
    assert np.allclose(od.rope(e0, p, 1, 4, 16.0)[0], [math.cos(4), 0, math.sin(4), 0], atol=1e-15)
    assert np.allclose(od.rope(e1, p, 1, 4, 16.0)[0], [0, math.cos(1), 0, math.sin(1)], atol=1e-15)


def test_rope_keeps_pair_norms_and_depends_on_relative_position():
    D = 128
    q = inputs.normal_bf16(12, (1, D))
    k = inputs.normal_bf16(13, (1, D))
    x = oracle.bf16_bits_to_f64(q)[0]
    r = od.rope(q, np.array([777], np.int32), 1, D, 500000.0)[0]
    assert np.allclose(x[:64] ** 2 + x[64:] ** 2, r[:64] ** 2 + r[64:] ** 2, rtol=1e-12)

    def dot(m, n):
        return float(od.rope(q, np.array([m], np.int32), 1, D, 500000.0)[0] @
                     od.rope(k, np.array([n], np.int32), 1, D, 500000.0)[0])
    assert dot(10, 3) == pytest.approx(dot(1010, 1003), rel=1e-9, abs=1e-9)
    assert dot(10, 3) != pytest.approx(dot(10, 4), rel=1e-6)


# ------------------------------------------------------------------ SwiGLU, add, argmax, embed
def test_swiglu_odd_part_and_zero():
    g = np.linspace(-6, 6, 24, dtype=np.float32)
    gu = np.concatenate([_bits(g), np.full(24, 0x3F80, np.uint16)])[None, :]       # u = 1
    gu_neg = np.concatenate([_bits(-g), np.full(24, 0x3F80, np.uint16)])[None, :]
    diff = od.swiglu(gu)[0] - od.swiglu(gu_neg)[0]
    assert np.allclose(diff, oracle.bf16_bits_to_f64(_bits(g)), rtol=1e-14, atol=1e-15)
    assert od.swiglu(np.array([[0, 0x4000]], np.uint16))[0, 0] == 0.0
    # u scales linearly
    gu2 = gu.copy()
    gu2[0, 24:] = 0x4000  # u = 2
    assert np.allclose(od.swiglu(gu2), 2 * od.swiglu(gu), rtol=1e-15)


def test_add_is_exact_in_f64():
    a, b = _bits([[1.5, -2.0]]), _bits([[0.25, 2.0]])
    assert od.add(a, b).tolist() == [[1.75, 0.0]]


def test_argmax_ties_and_nan():
    x = np.array([[1.0, 3.0, 3.0, -1.0], [np.nan, 0.0, np.nan, -5.0], [np.nan] * 4], np.float32)
    assert od.argmax(x).tolist() == [1, 1, 0]


def test_embed_range():
    table = inputs.normal_bf16(14, (5, 8))
    assert np.array_equal(od.embed([4, 0, 4], table), table[[4, 0, 4]])
    with pytest.raises(ValueError):
        od.embed([5], table)


# ------------------------------------------------------------------ causal attention
def test_attention_over_one_key_returns_its_value_per_kv_group():
    # two kv heads with distinct values: q head h must read kv head h // 2
    D = 8
    k = inputs.normal_bf16(15, (3, 2, D))
    v = inputs.normal_bf16(16, (3, 2, D))
    q = inputs.normal_bf16(17, (1, 4 * D))
    out = od.causal_attn(q, k, v, [1], [1], 4, 2, 0.3)
    vv = oracle.bf16_bits_to_f64(v)
    for h in range(4):
        assert np.array_equal(out[0, h * D:(h + 1) * D], vv[1, h // 2])


def test_attention_with_equal_scores_is_the_prefix_mean():
    D = 8
    k = np.tile(inputs.normal_bf16(18, (1, 1, D)), (6, 1, 1))
    v = inputs.normal_bf16(19, (6, 1, D))
    q = inputs.normal_bf16(20, (2, D))
    out = od.causal_attn(q, k, v, [0, 0], [3, 6], 1, 1, 0.5)
    vv = oracle.bf16_bits_to_f64(v)[:, 0]
    assert np.allclose(out[0], vv[:3].mean(0), rtol=1e-14, atol=1e-15)
    assert np.allclose(out[1], vv.mean(0), rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------------ the whole decoder
MINI = inputs.DecoderShape(hidden=8, layers=2, q_heads=2, kv_heads=1, head_dim=4, ffn=6, vocab=11, eps=1e-5,
                           theta=100.0)


def _mini_weights(seed=0):
    # larger spreads than the serving init, so that attention and RoPE are far from uniform
    out = {}
    for i, (name, r, c, mean, std) in enumerate(MINI.matrices()):
        w = inputs.normal_bf16(seed * 1000 + i, (r, c), mean, 0.6 if mean == 0.0 else 0.2)
        out[name] = w[0] if r == 1 else w
    return out


def _f(bits) -> float:
    return struct.unpack("<f", struct.pack("<I", int(bits) << 16))[0]


def _bf(x: float) -> float:
    """Nearest-even bf16 of a Python float (normal range): keep 8 significant bits."""
    if x == 0.0:
        return 0.0
    m, e = math.frexp(x)
    return round(m * 256) * 2.0 ** (e - 8)


class _Brute:
    """A scalar, loop-by-loop decoder written independently of oracle/decoder.py."""

    def __init__(self, shape, w):
        self.s = shape
        self.w = {k: (np.vectorize(_f)(v).tolist()) for k, v in w.items()}
        self.cache = {}  # (seq, layer) -> list of (k heads, v heads)

    def _norm(self, x, w):
        ms = sum(t * t for t in x) / len(x)
        inv = 1.0 / math.sqrt(ms + self.s.eps)
        return [_bf(x[j] * inv * w[j]) for j in range(len(x))]

    def _mat(self, x, W):
        return [_bf(sum(x[k] * W[k][n] for k in range(len(x)))) for n in range(len(W[0]))]

    def _rot(self, vec, p):
        D = self.s.head_dim
        half = D // 2
        out = list(vec)
        for i in range(half):
            z = complex(vec[i], vec[i + half]) * cmath.exp(1j * p * self.s.theta ** (-2.0 * i / D))
            out[i], out[i + half] = _bf(z.real), _bf(z.imag)
        return out

    def token(self, seq, tok, p):
        s, w = self.s, self.w
        D, Hq, Hkv = s.head_dim, s.q_heads, s.kv_heads
        h = list(w["embed"][tok])
        for l in range(s.layers):
            x = self._norm(h, w[f"l{l}.attn_norm"])
            qkv = self._mat(x, w[f"l{l}.wqkv"])
            qs = [self._rot(qkv[j * D:(j + 1) * D], p) for j in range(Hq)]
            ks = [self._rot(qkv[(Hq + j) * D:(Hq + j + 1) * D], p) for j in range(Hkv)]
            vs = [qkv[(Hq + Hkv + j) * D:(Hq + Hkv + j + 1) * D] for j in range(Hkv)]
            self.cache.setdefault((seq, l), []).append((ks, vs))
            att = []
            for hh in range(Hq):
                g = hh // (Hq // Hkv)
                sc = [sum(qs[hh][d] * kk[g][d] for d in range(D)) / math.sqrt(D) for kk, _ in self.cache[(seq, l)]]
                mx = max(sc)
                e = [math.exp(t - mx) for t in sc]
                tot = sum(e)
                for d in range(D):
                    att.append(_bf(sum(e[j] / tot * vv[g][d] for j, (_, vv) in enumerate(self.cache[(seq, l)]))))
            o = self._mat(att, w[f"l{l}.wo"])
            h = [_bf(a + b) for a, b in zip(h, o)]
            x = self._norm(h, w[f"l{l}.mlp_norm"])
            gu = self._mat(x, w[f"l{l}.wgu"])
            F = s.ffn
            a = [_bf(gu[j] / (1.0 + math.exp(-gu[j])) * gu[F + j]) for j in range(F)]
            d = self._mat(a, w[f"l{l}.wdown"])
            h = [_bf(a_ + b_) for a_, b_ in zip(h, d)]
        x = self._norm(h, w["final_norm"])
        return [sum(x[k] * w["lm_head"][k][n] for k in range(len(x))) for n in range(s.vocab)]


def _run_oracle(mod, w, steps, max_seqs=3, cap=32):
    dec = mod.OracleDecoder(MINI, w, max_seqs, cap)
    return [dec.forward(slots, toks) for slots, toks in steps]


STEPS = [([0, 2], [[3, 7, 1, 10, 0], [5, 5]]), ([0, 2], [[4], [9]]), ([2], [[1]])]


def _brute_steps(w, steps):
    br = _Brute(MINI, w)
    length = {}
    out = []
    for slots, toks in steps:
        rows = []
        for sl, tt in zip(slots, toks):
            for t in tt:
                lg = br.token(sl, t, length.get(sl, 0))
                length[sl] = length.get(sl, 0) + 1
            rows.append(lg)
        out.append(np.array(rows))
    return out


def test_decoder_matches_brute_force():
    w = _mini_weights()
    got = _run_oracle(od, w, STEPS)
    ref = _brute_steps(w, STEPS)
    for g, r in zip(got, ref):
        assert np.allclose(g, r, rtol=1e-9, atol=1e-12), np.abs(g - r).max()


def test_decoder_is_batch_and_chunk_invariant():
    w = _mini_weights(1)
    prompt = [3, 7, 1, 10, 0, 2, 8]
    alone = od.OracleDecoder(MINI, w, 3, 32)
    a0 = alone.forward([0], [prompt])
    a1 = alone.forward([0], [[6]])
    batched = od.OracleDecoder(MINI, w, 3, 32)
    b0 = batched.forward([0, 1, 2], [[1, 2], prompt, [9, 9, 9]])
    b1 = batched.forward([0, 1, 2], [[4], [6], [5]])
    assert np.array_equal(a0[0], b0[1]) and np.array_equal(a1[0], b1[1])
    chunked = od.OracleDecoder(MINI, w, 3, 32)
    chunked.forward([2], [prompt[:3]])
    c0 = chunked.forward([2], [prompt[3:]])
    assert np.array_equal(a0[0], c0[0])


def test_decoder_with_zeroed_residual_branches_is_norm_and_head_of_the_embedding():
    w = _mini_weights(2)
    for l in range(MINI.layers):
        w[f"l{l}.wo"] = np.zeros_like(w[f"l{l}.wo"])
        w[f"l{l}.wdown"] = np.zeros_like(w[f"l{l}.wdown"])
    got = od.OracleDecoder(MINI, w, 1, 16).forward([0], [[2, 9, 4]])[0]
    e = [_f(b) for b in w["embed"][4]]
    x = [_bf(t / math.sqrt(sum(u * u for u in e) / len(e) + MINI.eps) * _f(g)) for t, g in zip(e, w["final_norm"])]
    ref = [sum(x[k] * _f(w["lm_head"][k][n]) for k in range(len(x))) for n in range(MINI.vocab)]
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ planted mistakes
MUTANTS = {
    "attention sees one key too few": ("base, pos + 1, Hq", "base, np.maximum(pos, 1), Hq"),
    "q heads read with the wrong layout": ("reshape(T, q_heads, D)", "reshape(T, D, q_heads).transpose(0, 2, 1)"),
    "rope pairs interleaved": ("a, b = x[..., :half], x[..., half:]", "a, b = x[..., 0::2], x[..., 1::2]"),
    "rope frequency exponent": ("-2.0 * np.arange(half", "-1.0 * np.arange(half"),
    "rope rotates the wrong way": ("out[..., :half] = a * c - b * s", "out[..., :half] = a * c + b * s"),
    "rope skips the keys": ("qkv[:, :nqk] = round_bf16(rope(qkv, pos, Hq + Hkv, D, s.theta))",
                            "qkv[:, :Hq * D] = round_bf16(rope(qkv, pos, Hq, D, s.theta))"),
    "swiglu gate and up swapped": ("g / (1.0 + np.exp(-g)) * u", "u / (1.0 + np.exp(-u)) * g"),
    "residual dropped": ("h = round_bf16(add(h, round_bf16(gemm(att", "h = round_bf16((round_bf16(gemm(att"),
    "logits of the first token": ("last = np.cumsum([len(t) for t in tokens]) - 1",
                                  "last = np.cumsum([0] + [len(t) for t in tokens])[:-1]"),
    "mlp norm weight of attention": ('w[f"l{l}.mlp_norm"]', 'w[f"l{l}.attn_norm"]'),
    "positions restart each call": ("pos = np.concatenate([self.length[sl] + np.arange",
                                    "pos = np.concatenate([0 * self.length[sl] + np.arange"),
}


def _mutant_module(old, new):
    src = open(od.__file__).read()
    assert src.count(old) >= 1, old
    mod = types.ModuleType("oracle._decoder_mutant")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), od.__file__ + ":mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    mod = _mutant_module(old, new)
    w = _mini_weights()
    try:
        got = _run_oracle(mod, w, STEPS)
    except Exception:
        return  # a mistake that breaks the run is caught too
    ref = _brute_steps(w, STEPS)
    assert not all(np.allclose(g, r, rtol=1e-9, atol=1e-12) for g, r in zip(got, ref)), name
