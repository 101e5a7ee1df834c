"""bi_decode_attn on the GPU: parity with the fp64 oracle (plain softmax), chunk boundaries,
GQA groupings, closed forms, bitwise batch invariance, device-side layout checks.

Tolerance: relative Frobenius error <= 2e-3 per request against the unrounded fp64 oracle, for
fp32 output.  The kernel's arithmetic is fp32 with exact bf16 products, so the sanity bound
1e-4 is also enforced.  bf16 output: within one bf16 rounding of the oracle.
Batch invariance: exact bits of each probe request's output, solo vs embedded.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bf16_to_f64, dev, host, rel_frobenius
from invariant_deterministic_rmsnorm_b200 import binding, inputs

pytestmark = pytest.mark.gpu
D = 128
CHUNK = 256


def _run(q, k, v, indptr, kv_len, Hkv, out_dtype=torch.float32, scale=None):
    out = binding.bi_decode_attn(dev(q), dev(k), dev(v), dev(indptr), dev(kv_len.astype(np.int32)),
                                 scale=scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return host(out)


def _check(kv_len, Hq=32, Hkv=8, seed=1, bound=1e-4):
    kv_len = np.asarray(kv_len, np.int32)
    q, k, v, indptr, T = inputs.attn_case(kv_len, Hq, Hkv, D, CHUNK, seed)
    got = _run(q, k, v, indptr, kv_len, Hkv)
    ref = oracle.decode_attn(q, k, v, indptr, kv_len, Hkv, 1.0 / np.sqrt(D))
    for b in range(len(kv_len)):
        err = rel_frobenius(got[b], ref[b])
        assert err <= 2e-3 and err <= bound, (b, int(kv_len[b]), err)
    return got, ref


def test_parity_chunk_boundaries():
    _check([1, 2, 255, 256, 257, 511, 512, 513, 1000])


@pytest.mark.parametrize("Hq,Hkv", [(32, 32), (32, 16), (32, 8), (32, 4)])
def test_parity_gqa_groupings(Hq, Hkv):
    _check([300, 77, 1024], Hq=Hq, Hkv=Hkv, seed=3)


def test_parity_workload_lengths():
    """Lengths drawn as in the decode workload, U[512, 32768]."""
    _check(inputs.kv_lengths(4), seed=5)


def test_bf16_output():
    kv_len = np.array([700, 3000], np.int32)
    q, k, v, indptr, T = inputs.attn_case(kv_len, 32, 8, D, CHUNK, 7)
    got = bf16_to_f64(_run(q, k, v, indptr, kv_len, 8, torch.bfloat16))
    ref = oracle.decode_attn(q, k, v, indptr, kv_len, 8, 1.0 / np.sqrt(D))
    rms = np.sqrt((ref ** 2).mean(axis=-1, keepdims=True))
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * rms)


def test_equal_scores_give_mean_of_values():
    kv_len = np.array([600, 1], np.int32)
    q, k, v, indptr, T = inputs.attn_case(kv_len, 32, 8, D, CHUNK, 9)
    q[:] = 0
    got = _run(q, k, v, indptr, kv_len, 8)
    vf = bf16_to_f64(v)
    for b in range(2):
        base, L = int(indptr[b]), int(kv_len[b])
        for h in range(32):
            mean = vf[base:base + L, h // 4, :].mean(axis=0)
            assert np.allclose(got[b, h], mean, rtol=1e-5, atol=1e-6)


def test_sequences_with_spare_capacity():
    """kv_indptr[b+1] - kv_indptr[b] larger than kv_len[b]: the spare tokens (here NaN) are never read."""
    kv_len = np.array([300, 40], np.int32)
    q, k, v, indptr, T = inputs.attn_case(kv_len, 32, 8, D, CHUNK, 11)
    cap = np.array([0, 1024, 1536], np.int32)
    k2 = np.full((1536, 8, D), 0x7FC0, np.uint16)  # quiet NaN in every spare slot
    v2 = np.full((1536, 8, D), 0x7FC0, np.uint16)
    for b in range(2):
        L = int(kv_len[b])
        k2[cap[b]:cap[b] + L] = k[indptr[b]:indptr[b] + L]
        v2[cap[b]:cap[b] + L] = v[indptr[b]:indptr[b] + L]
    got = _run(q, k2, v2, cap, kv_len, 8)
    ref = oracle.decode_attn(q, k, v, indptr, kv_len, 8, 1.0 / np.sqrt(D))
    assert np.all(np.isfinite(got))
    for b in range(2):
        assert rel_frobenius(got[b], ref[b]) <= 1e-4


def test_workspace_and_layout_errors():
    kv_len = np.array([300], np.int32)
    q, k, v, indptr, T = inputs.attn_case(kv_len, 32, 8, D, CHUNK, 13)
    with pytest.raises(binding.BIError):
        binding.bi_decode_attn(dev(q), dev(k), dev(v), dev(indptr), dev(kv_len), workspace=None, chunk=128)
    lib = binding.library()
    assert lib.bi_decode_attn_workspace_size(T, 32, D, CHUNK) == ((T + 255) // 256) * 32 * (D + 2) * 4
    # a sequence start that is not chunk-aligned is caught on the device, without a fault
    binding.bi_clear_device_error()
    bad = np.array([16, 16 + 512], np.int32)
    k3 = np.zeros((1024, 8, D), np.uint16)
    binding.bi_decode_attn(dev(q), dev(k3), dev(k3), dev(bad), dev(kv_len))
    assert binding.bi_get_device_error() & 0x100
    binding.bi_clear_device_error()
    assert binding.bi_get_device_error() == 0


def _device_seqs(seed, lens, Hkv=8):
    g = torch.Generator(device="cuda").manual_seed(seed)
    out = []
    for L in lens:
        kk = torch.randn((int(L), Hkv, D), generator=g, device="cuda").to(torch.bfloat16)
        vv = torch.randn((int(L), Hkv, D), generator=g, device="cuda").to(torch.bfloat16)
        qq = torch.randn((32, D), generator=g, device="cuda").to(torch.bfloat16)
        out.append((qq, kk, vv))
    return out


def _pack(reqs):
    """Pack requests (q, k, v) into one chunk-aligned cache, in the given order."""
    lens = [r[1].shape[0] for r in reqs]
    padded = [((L + CHUNK - 1) // CHUNK) * CHUNK for L in lens]
    indptr = np.zeros(len(reqs) + 1, np.int64)
    indptr[1:] = np.cumsum(padded)
    T = int(indptr[-1])
    k = torch.zeros((T, 8, D), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    for i, (qq, kk, vv) in enumerate(reqs):
        k[indptr[i]:indptr[i] + kk.shape[0]] = kk
        v[indptr[i]:indptr[i] + vv.shape[0]] = vv
    q = torch.stack([r[0] for r in reqs]).contiguous()
    ip = torch.tensor(indptr, dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return q, k, v, ip, ln


def test_batch_invariance():
    probes = _device_seqs(inputs.SEED_PROBES, [300, 1, 4097, 20000])
    solo = []
    for p in probes:
        q, k, v, ip, ln = _pack([p])
        solo.append(binding.bi_decode_attn(q, k, v, ip, ln, out_dtype=torch.float32)[0].clone())
    rng_len = np.random.default_rng(inputs.SEED_KVLEN)
    bad = 0
    for B in [1, 2, 3, 4, 5, 8, 16, 17, 32, 64, 128, 255, 256]:
        for trial in range(2 if B > 64 else 3):
            lens = rng_len.integers(1, 1025, size=B)
            fill = _device_seqs(1000 + 97 * B + trial, lens)
            rng = np.random.default_rng([inputs.SEED_POSITIONS, B, trial])
            pos = rng.choice(B, size=min(B, len(probes)), replace=False)
            for i, w in enumerate(pos):
                fill[int(w)] = probes[i]
            q, k, v, ip, ln = _pack(fill)
            out = binding.bi_decode_attn(q, k, v, ip, ln, out_dtype=torch.float32)
            for i, w in enumerate(pos):
                bad += int(not torch.equal(out[int(w)].view(torch.int32), solo[i].view(torch.int32)))
            del fill, q, k, v
    assert bad == 0
    # replay
    q, k, v, ip, ln = _pack(probes)
    first = binding.bi_decode_attn(q, k, v, ip, ln, out_dtype=torch.float32).clone()
    for _ in range(9):
        assert torch.equal(binding.bi_decode_attn(q, k, v, ip, ln, out_dtype=torch.float32).view(torch.int32),
                           first.view(torch.int32))
    assert binding.bi_get_device_error() == 0


def test_small_batch_in_a_large_cache():
    """Six requests in scattered 2048-token slots of a 128-slot cache (a serving engine's
    layout: each sequence's capacity runs to the next listed sequence).  The live chunks are
    spread over the CTAs, not the cache's capacity; the outputs are bitwise those of the same
    requests packed tightly, and match the oracle."""
    cap, n_slots = 2048, 128
    slots = [3, 17, 18, 60, 100, 127]
    lens = [1, 2048, 700, 257, 1999, 256]
    reqs = _device_seqs(inputs.SEED_PROBES + 5, lens)
    T = n_slots * cap
    k = torch.zeros((T, 8, D), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    for s, (qq, kk, vv) in zip(slots, reqs):
        k[s * cap:s * cap + kk.shape[0]] = kk
        v[s * cap:s * cap + vv.shape[0]] = vv
    q = torch.stack([r[0] for r in reqs]).contiguous()
    ip = torch.tensor(slots + [slots[-1] + 1], dtype=torch.int32, device="cuda") * cap
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    binding.bi_clear_device_error()
    got = binding.bi_decode_attn(q, k, v, ip, ln, out_dtype=torch.float32)
    packed = binding.bi_decode_attn(*_pack(reqs), out_dtype=torch.float32)
    assert torch.equal(got.view(torch.int32), packed.view(torch.int32))
    assert binding.bi_get_device_error() == 0
    for b, (qq, kk, vv) in enumerate(reqs):
        ref = oracle.decode_attn(host(qq)[None], host(kk), host(vv), np.array([0, kk.shape[0]], np.int64),
                                 np.array([kk.shape[0]], np.int32), 8, 1.0 / np.sqrt(D))
        assert rel_frobenius(host(got[b]), ref[0]) <= 1e-4, b


def test_decreasing_kv_indptr_is_reported():
    """Overlapping sequences (a decreasing kv_indptr) are refused on the device: bit 0x100 and no fault."""
    kv_len = np.array([100, 100], np.int32)
    q, k, v, indptr, T = inputs.attn_case(kv_len, 32, 8, D, CHUNK, 17)
    k3 = np.zeros((1024, 8, D), np.uint16)
    binding.bi_clear_device_error()
    binding.bi_decode_attn(dev(q), dev(k3), dev(k3), dev(np.array([512, 0, 1024], np.int32)), dev(kv_len))
    assert binding.bi_get_device_error() & 0x100
    binding.bi_clear_device_error()
