"""The comparators: correct results (parity with the fp64 oracle) but NOT batch-invariant.

Each comparator is a schedule that the pages name as breaking batch invariance: a split
reduction for small batches (RMSNorm), split-K chosen by batch size (matmul), a split-KV
chunk size chosen by batch size (attention), and the atomic split-K shrink (in the LoRA
tests).  They are the positive controls of the invariance harness: each must show
violations somewhere in the sweep, or the harness could not detect the property it gates.
(cuBLAS, called through torch.matmul, is timed and spot-checked in the benchmark; whether
it varies with the batch size depends on the shape and the library version.)
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bf16_to_f64, dev, host, rel_err_rowscaled, rel_frobenius
from invariant_deterministic_rmsnorm_b200 import binding, harness, inputs

pytestmark = pytest.mark.gpu


def _device_rows(seed, M, cols):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((M, cols), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("M", [1, 100, 300, 1000])
def test_split_rmsnorm_parity(M):
    x, w = inputs.rmsnorm_case(M, 4096, "bf16")
    y = host(binding.bi_ctrl_rmsnorm_split(dev(x), dev(w)))
    ref = oracle.round_bf16(oracle.rmsnorm(x, w, 1e-6))
    from gpu_util import bf16_ulp_distance
    assert bf16_ulp_distance(y, ref).max() <= 1


def test_split_rmsnorm_is_not_batch_invariant():
    """fp32 output: a changed reduction tree moves the sum by an ulp or so, which bf16 output
    would mostly round away (bf16 outputs of the split kernel agree across M for most rows)."""
    w = dev(inputs.normal(0, (4096,), 1.0, 0.1))
    probes = dev(inputs.normal(inputs.SEED_PROBES, (8, 4096)))
    fill = {t: _device_rows(1000 + t, 2048, 4096).float() for t in range(3)}
    run = lambda b: binding.bi_ctrl_rmsnorm_split(b.contiguous(), w)
    rep = harness.bi_check_rows("rmsnorm_split", run, probes, lambda t: fill[t], [1, 8, 200, 400, 1000])
    assert rep.violations > 0, rep.as_dict()


@pytest.mark.parametrize("M", [1, 64, 513])
def test_splitk_gemm_parity(M):
    A, W = inputs.gemm_case(M, 6144, 4096)
    C = host(binding.bi_ctrl_gemm_splitk(dev(A), dev(W)))
    rows = sorted({0, M - 1})
    assert rel_frobenius(C[rows], oracle.gemm(A[rows], W)) <= 1e-4


def test_splitk_gemm_is_not_batch_invariant():
    K, N = 4096, 6144
    W = dev(inputs.normal_bf16(0, (K, N), 0, 0.02))
    probes = dev(inputs.normal_bf16(inputs.SEED_PROBES, (8, K)))
    fill = {t: _device_rows(1000 + t, 4096, K) for t in range(3)}
    run = lambda b: binding.bi_ctrl_gemm_splitk(b.contiguous(), W)
    rep = harness.bi_check_rows("gemm_splitk", run, probes, lambda t: fill[t], [1, 16, 128, 600, 4096])
    assert rep.violations > 0, rep.as_dict()


def test_adaptive_attention_parity_and_not_batch_invariant():
    kv_len = np.array([700, 300, 2000], np.int32)
    q, k, v, ip, T = inputs.attn_case(kv_len, 32, 8, 128, 256, 3)
    out = host(binding.bi_ctrl_decode_attn_adaptive(dev(q), dev(k), dev(v), dev(ip), dev(kv_len),
                                                    out_dtype=torch.float32))
    ref = oracle.decode_attn(q, k, v, ip, kv_len, 8, 1.0 / np.sqrt(128))
    for b in range(3):
        assert rel_frobenius(out[b], ref[b]) <= 1e-4
    # the same first request inside a batch of 20 (256-token chunks) vs alone (128-token chunks)
    lens = np.concatenate([kv_len[:1], np.full(19, 300, np.int32)])
    q2, k2, v2, ip2, T2 = inputs.attn_case(lens, 32, 8, 128, 256, 3)
    q2[0] = q[0]
    k2[:ip2[1]] = 0
    v2[:ip2[1]] = 0
    k2[:700] = k[:700]
    v2[:700] = v[:700]
    big = host(binding.bi_ctrl_decode_attn_adaptive(dev(q2), dev(k2), dev(v2), dev(ip2), dev(lens),
                                                    out_dtype=torch.float32))
    solo = host(binding.bi_ctrl_decode_attn_adaptive(dev(q[:1]), dev(k[:ip[1]]), dev(v[:ip[1]]),
                                                     dev(np.array([0, ip[1]], np.int32)), dev(kv_len[:1]),
                                                     out_dtype=torch.float32))
    assert not np.array_equal(big[0].view(np.uint32), solo[0].view(np.uint32))
    # while the batch-invariant kernel gives the same bits in both
    big_bi = host(binding.bi_decode_attn(dev(q2), dev(k2), dev(v2), dev(ip2), dev(lens), out_dtype=torch.float32))
    solo_bi = host(binding.bi_decode_attn(dev(q[:1]), dev(k[:ip[1]]), dev(v[:ip[1]]),
                                          dev(np.array([0, ip[1]], np.int32)), dev(kv_len[:1]),
                                          out_dtype=torch.float32))
    assert np.array_equal(big_bi[0].view(np.uint32), solo_bi[0].view(np.uint32))
