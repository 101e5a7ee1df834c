"""The decoder ops of include/bi_model.h against the fp64 oracle, and their batch invariance.

Copies and integer results (embedding gather, KV append, argmax) must be bit-exact.  The
element-wise fp32 ops (RoPE, residual add, SwiGLU) round once to bf16, so they may differ from
the oracle's rounded fp64 result only where the fp32 value sits next to a rounding boundary:
at most 1 bf16 step, and on a small fraction of elements.  Prefill attention follows the
attention tolerance: relative Frobenius error <= 2e-3 per head.  Its output is bitwise
independent of the other sequences in the call and of how the prompt was cut into chunks.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import decoder as od
from gpu_util import bf16_to_f64, bf16_ulp_distance, dev, host, rel_frobenius
from invariant_deterministic_rmsnorm_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def test_embed_is_an_exact_gather():
    table = inputs.normal_bf16(30, (1000, 512))
    toks = np.random.default_rng(31).integers(0, 1000, 77).astype(np.int32)
    out = host(binding.bi_embed(dev(toks), dev(table)))
    assert np.array_equal(out, od.embed(toks, table))


def test_embed_bad_token_sets_the_error_bit():
    table = dev(inputs.normal_bf16(30, (10, 64)))
    binding.bi_clear_device_error()
    out = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    binding.bi_embed(dev(np.array([3, 10], np.int32)), table, out=out)
    assert binding.bi_get_device_error() & 0x200
    binding.bi_clear_device_error()
    assert torch.equal(out[0], table[3]) and not out[1].any()


@pytest.mark.parametrize("heads,ld", [(40, 6144), (2, 256)])
def test_rope_parity(heads, ld):
    T, D = 300, 128
    x = inputs.normal_bf16(32, (T, ld))
    pos = np.random.default_rng(33).integers(0, 2200, T).astype(np.int32)
    pos[:3] = [0, 1, 2111]
    table = binding.bi_rope_table(2200, D, 500000.0)
    got = host(binding.bi_rope(dev(x), dev(pos), heads, table, D))
    exact = od.rope(x, pos, heads, D, 500000.0)
    ref = oracle.round_bf16(exact)
    # one bf16 rounding on each side, plus the fp32 error of a rotation (a few 2^-24 of the
    # pair's norm, which dominates where the two products nearly cancel)
    xx = bf16_to_f64(x[:, :heads * D]).reshape(T, heads, 2, D // 2)
    pair = np.sqrt((xx ** 2).sum(2, keepdims=True))
    norm = np.broadcast_to(pair, xx.shape).reshape(T, heads * D)
    g = bf16_to_f64(got[:, :heads * D])
    assert np.all(np.abs(g - exact) <= 2.0 ** -8 * np.abs(exact) + 2.0 ** -20 * norm)
    d = bf16_ulp_distance(got[:, :heads * D], ref)
    assert (d > 0).mean() < 1e-3, (d > 0).mean()
    assert np.array_equal(got[:, heads * D:], x[:, heads * D:])  # columns past the heads untouched
    assert np.array_equal(got[0], x[0])  # position 0 is the identity


def test_rope_16_byte_and_4_byte_paths_give_the_same_bits():
    """Rows that are 16-byte aligned (row stride a multiple of 8) take the kernel with 16-byte
    accesses; an even row stride that is not a multiple of 8 takes the 4-byte kernel.  Both run
    the same operations on every element."""
    T, D, heads = 257, 128, 40
    x = inputs.normal_bf16(34, (T, heads * D))
    pos = np.random.default_rng(35).integers(0, 2200, T).astype(np.int32)
    table = binding.bi_rope_table(2200, D, 500000.0)
    rows = {}
    for ld in (6144, 6146):
        buf = np.zeros((T, ld), np.uint16)
        buf[:, :heads * D] = x
        rows[ld] = host(binding.bi_rope(dev(buf), dev(pos), heads, table, D))[:, :heads * D]
    assert np.array_equal(rows[6144], rows[6146])
    assert not np.array_equal(rows[6144], x)  # the rotation did run


def test_rope_table_and_bad_position():
    t = host(binding.bi_rope_table(3000, 128, 500000.0)).astype(np.float64)
    i = np.arange(64)
    for p in (0, 1, 2999):
        ang = p * np.power(500000.0, -2.0 * i / 128)
        assert np.allclose(t[p, :, 0], np.cos(ang), rtol=0, atol=2 ** -24)
        assert np.allclose(t[p, :, 1], np.sin(ang), rtol=0, atol=2 ** -24)
    x = dev(inputs.normal_bf16(41, (2, 256)))
    x0 = x.clone()
    binding.bi_clear_device_error()
    binding.bi_rope(x, dev(np.array([5, 3000], np.int32)), 2, binding.bi_rope_table(3000, 128))
    assert binding.bi_get_device_error() & 0x1000
    binding.bi_clear_device_error()
    assert torch.equal(x[1], x0[1]) and not torch.equal(x[0], x0[0])


def test_kv_append_scatters_rows_exactly():
    src = inputs.normal_bf16(34, (50, 6144))
    rows = np.random.default_rng(35).permutation(200)[:50].astype(np.int32)
    cache = torch.zeros((200, 8, 128), dtype=torch.bfloat16, device="cuda")
    binding.bi_kv_append(dev(src)[:, 4096:5120], dev(rows), cache)
    c = host(cache).reshape(200, 1024)
    assert np.array_equal(c[rows], src[:, 4096:5120])
    others = np.setdiff1d(np.arange(200), rows)
    assert not c[others].any()


def test_add_and_swiglu_parity():
    T, N = 129, 14336
    h = inputs.normal_bf16(36, (T, N))
    d = inputs.normal_bf16(37, (T, N), 0, 0.3)
    # the fp32 sum of two bf16 values is exact unless their exponents are 16 or more apart, and
    # then the smaller one is below a quarter step of the larger: one rounding either way
    got = host(binding.bi_add(dev(h), dev(d)))
    assert np.array_equal(got, oracle.round_bf16(od.add(h, d)))
    gu = inputs.normal_bf16(38, (T, 2 * N), 0, 2.0)
    got = host(binding.bi_swiglu(dev(gu)))
    dist = bf16_ulp_distance(got, oracle.round_bf16(od.swiglu(gu)))
    assert dist.max() <= 1 and (dist > 0).mean() < 1e-3, (dist > 0).mean()


def test_argmax_matches_the_oracle_bit_for_bit():
    x = inputs.normal(39, (64, 32000))
    x[1, [5, 17, 31999]] = 100.0           # ties: smallest index wins
    x[2, :] = np.nan
    x[3, 7] = np.nan
    x[3, 9] = 50.0
    x[4, :] = -np.inf
    got = host(binding.bi_argmax(dev(x)))
    assert np.array_equal(got, od.argmax(x))
    assert got[1] == 5 and got[2] == 0 and got[3] == 9 and got[4] == 0


# ------------------------------------------------------------------ prefill attention
HQ, HKV, D = 32, 8, 128


def _prefill_case(q_lens, pos0, seed=40, gap=64, ld=6144):
    """q rows [T, ld] (q heads in the first 4096 columns) and a packed cache in which sequence b
    starts at a gap after the previous one, holding positions 0 .. pos0[b] + q_lens[b] - 1."""
    q_lens = np.asarray(q_lens, np.int64)
    pos0 = np.asarray(pos0, np.int64)
    kv_len = pos0 + q_lens
    kv_base = np.zeros(len(q_lens), np.int64)
    off = 0
    for b, n in enumerate(kv_len):
        kv_base[b] = off
        off += int(n) + gap
    T = int(q_lens.sum())
    q = inputs.normal_bf16(seed, (T, ld))
    k = inputs.normal_bf16(seed + 1, (off, HKV, D))
    v = inputs.normal_bf16(seed + 2, (off, HKV, D))
    return q, k, v, q_lens, pos0, kv_base


def _run_prefill(q, k, v, q_lens, pos0, kv_base):
    q_indptr = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    tiles = binding.prefill_tiles(q_lens)
    out = binding.bi_prefill_attn(dev(q) if isinstance(q, np.ndarray) else q, dev(k), dev(v), dev(q_indptr),
                                  dev(np.array(tiles, np.int32)), tiles[-1], dev(kv_base.astype(np.int32)),
                                  dev(pos0.astype(np.int32)), HQ)
    return host(out)


def _oracle_prefill(q, k, v, q_lens, pos0, kv_base):
    base = np.repeat(kv_base, q_lens)
    pos = np.concatenate([p + np.arange(n) for p, n in zip(pos0, q_lens)])
    return od.causal_attn(q, k, v, base, pos + 1, HQ, HKV, 1.0 / np.sqrt(D))


@pytest.mark.parametrize("q_lens,pos0", [
    ([1, 63, 64, 65, 200, 7], [0, 0, 0, 0, 0, 0]),        # ragged tiles and KV blocks
    ([130, 5, 64], [300, 1, 63]),                          # chunked prefill over a cached prefix
    ([1, 1, 1], [0, 1000, 2047]),                          # single rows (decode through prefill)
    ([300, 129, 128, 127], [0, 0, 5, 700]),                # several 128-row tiles, ragged last tiles
])
def test_prefill_attention_parity(q_lens, pos0):
    q, k, v, ql, p0, kb = _prefill_case(q_lens, pos0)
    got = bf16_to_f64(_run_prefill(q, k, v, ql, p0, kb))
    ref = _oracle_prefill(q, k, v, ql, p0, kb)
    assert np.isfinite(got).all()
    for h in range(HQ):
        sl = slice(h * D, (h + 1) * D)
        assert rel_frobenius(got[:, sl], ref[:, sl]) <= 2e-3


def test_prefill_attention_is_batch_and_chunk_invariant():
    q_lens, pos0 = [200, 77, 333], [0, 0, 0]
    q, k, v, ql, p0, kb = _prefill_case(q_lens, pos0, seed=50)
    full = _run_prefill(q, k, v, ql, p0, kb)
    # sequence 1 alone (rows 200 .. 276 of q)
    alone = _run_prefill(q[200:277], k, v, ql[1:2], p0[1:2], kb[1:2])
    assert np.array_equal(alone, full[200:277])
    # sequence 2 as three chunks: [0, 50), [50, 51), [51, 333) with their cached prefixes
    rows = np.arange(277, 610)
    cuts = [(0, 50), (50, 51), (51, 333)]
    for a, b in cuts:
        part = _run_prefill(q[rows[a:b]], k, v, np.array([b - a]), np.array([a]), kb[2:3])
        assert np.array_equal(part, full[rows[a:b]]), (a, b)
    # the same three chunks in one call, each as its own "sequence" over the shared cache
    qs = np.concatenate([q[rows[a:b]] for a, b in cuts])
    mixed = _run_prefill(qs, k, v, np.array([b - a for a, b in cuts]), np.array([a for a, _ in cuts]),
                         np.repeat(kb[2], 3))
    assert np.array_equal(mixed, full[rows])


def test_prefill_attention_layout_error_sets_bit():
    q, k, v, ql, p0, kb = _prefill_case([10], [0])
    binding.bi_clear_device_error()
    bad_kb = np.array([k.shape[0] - 5], np.int64)  # positions run past the cache
    _run_prefill(q, k, v, ql, p0, bad_kb)
    assert binding.bi_get_device_error() & 0x800
    binding.bi_clear_device_error()


def test_prefill_attention_ignores_non_finite_spare_rows():
    """Cache rows outside every sequence's live positions hold NaN: the masked scores and the
    zeroed value rows keep them out of every output, which must match the zero-filled case bit
    for bit."""
    q_lens, pos0 = [70, 129, 5], [0, 30, 200]
    q, k, v, ql, p0, kb = _prefill_case(q_lens, pos0, seed=60, gap=100)
    live = np.zeros(k.shape[0], bool)
    for base, n in zip(kb, p0 + ql):
        live[base:base + n] = True
    k_nan, v_nan = k.copy(), v.copy()
    k_nan[~live] = 0x7FC0
    v_nan[~live] = 0x7FC0
    k_zero, v_zero = k.copy(), v.copy()
    k_zero[~live] = 0
    v_zero[~live] = 0
    got = _run_prefill(q, k_nan, v_nan, ql, p0, kb)
    ref_bits = _run_prefill(q, k_zero, v_zero, ql, p0, kb)
    assert np.isfinite(bf16_to_f64(got)).all()
    assert np.array_equal(got, ref_bits)
    ref = _oracle_prefill(q, k, v, ql, p0, kb)
    assert rel_frobenius(bf16_to_f64(got), ref) <= 2e-3
