"""bi_gemm on the GPU: exact layout pins, parity with the fp64 oracle, bitwise batch invariance.

Tolerances:
  * small-integer operands (|a|, |w| <= 8, K * 64 < 2^24): every partial sum is exact in fp32,
    so the fp32 output must equal the oracle bit for bit, whatever the accumulation order.
  * random bf16 operands: relative Frobenius error <= 2e-3 against the unrounded fp64 oracle.
    fp32 accumulation over K terms sits many orders of magnitude below this bound.
  * batch invariance: exact bits, solo vs embedded at random positions, M = 1 .. 8192.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bf16_to_f64, dev, host, oracle_rows, rel_frobenius
from invariant_deterministic_rmsnorm_b200 import binding, harness, inputs

pytestmark = pytest.mark.gpu

LLAMA_SHAPES = [(4096, 6144), (4096, 14336), (14336, 4096)]  # (K, N)
# the decoder's fused gate/up projection and its vocabulary projection: wider than a row of
# 256-wide CTA-pair tiles can cover on one GPU, so they run on the single-CTA plan
WIDE_SHAPES = [(4096, 28672), (4096, 32000)]


def _gemm(A_np, W_np, out=torch.float32):
    C = binding.bi_gemm(dev(A_np), dev(W_np), out_dtype=out)
    torch.cuda.synchronize()
    return host(C)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 520, 264), (1, 16, 8), (300, 1032, 1000), (129, 4096, 72)])
def test_small_int_exact(M, N, K):
    A = inputs.small_int_bf16(53, (M, K))
    W = inputs.small_int_bf16(54, (K, N))
    C = _gemm(A, W)
    ref = oracle.gemm(A, W)
    assert np.array_equal(C.astype(np.float64), ref), int((C != ref).sum())


def test_one_hot_rows_pick_weight_rows():
    M, K, N = 130, 192, 264
    A = inputs.f32_to_bf16_bits(np.eye(K, dtype=np.float32)[np.arange(M) % K])
    W = inputs.normal_bf16(52, (K, N), 0, 0.02)
    C = _gemm(A, W)
    assert np.array_equal(C.astype(np.float64), bf16_to_f64(W)[np.arange(M) % K])


@pytest.mark.parametrize("M", [1, 3, 8, 32])
def test_parity_small_config(M):
    """A = bf16 of the small RMSNorm workload's output, W [256, 512] ~ N(0, 0.02)."""
    x, w = inputs.rmsnorm_case(M, 256, "f32")
    A = oracle.round_bf16(oracle.rmsnorm(x, w, 1e-6))
    W = inputs.normal_bf16(inputs.SEED_WEIGHTS, (256, 512), 0, 0.02)
    C = _gemm(A, W)
    assert rel_frobenius(C, oracle.gemm(A, W)) <= 2e-3


@pytest.mark.parametrize("K,N", LLAMA_SHAPES + WIDE_SHAPES)
@pytest.mark.parametrize("M", [1, 129, 257])
def test_parity_llama_shapes_sampled_rows(K, N, M):
    A, W = inputs.gemm_case(M, N, K)
    C = _gemm(A, W)
    rows = sorted(set([0, M // 2, M - 1]))
    ref = oracle.gemm(A[rows], W)
    err = rel_frobenius(C[rows], ref)
    assert err <= 2e-3, err
    # sanity bound far below the gate: tensor-core fp32 accumulation measures ~1.6e-5 at
    # K = 14336; bf16 accumulation would be ~1e-2
    assert err <= 1e-4, err


def test_parity_ragged_tiles_random():
    M, N, K = 333, 776, 456  # 3 row tiles, 4 column tiles, 8 K-blocks, all ragged
    A, W = inputs.gemm_case(M, N, K, seed_a=91, seed_w=92)
    C = _gemm(A, W)
    assert rel_frobenius(C, oracle.gemm(A, W)) <= 1e-5


def test_bf16_output():
    M, N, K = 257, 6144, 4096
    A, W = inputs.gemm_case(M, N, K)
    Cb = _gemm(A, W, torch.bfloat16)
    C32 = _gemm(A, W, torch.float32)
    rows = [0, 100, 256]
    ref = oracle.gemm(A[rows], W)
    assert rel_frobenius(bf16_to_f64(Cb[rows]), ref) <= 2e-3
    # the bf16 output is the nearest-even rounding of the kernel's own fp32 accumulator
    assert np.array_equal(Cb, inputs.f32_to_bf16_bits(C32))
    # elementwise: bf16 rounding (at most 2^-8 relative to |r|) plus fp32 accumulation error,
    # which scales with the row (bounded here by 2e-4 * rms(row))
    g = bf16_to_f64(Cb[rows])
    rms = np.sqrt((ref ** 2).mean(axis=1, keepdims=True))
    assert np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-4 * rms)


@pytest.mark.parametrize("K,N", LLAMA_SHAPES + WIDE_SHAPES)
def test_full_size_every_row_on_a_column_slice(K, N):
    """The bench's launch configuration, M = 4096, on both plans (CTA pairs for the three
    Llama-shaped projections, single CTAs for the two wide ones).  Every one of the 4096 rows
    is compared with the oracle on 256 columns that straddle a tile boundary, so a slip in any
    row tile, in either CTA of a pair, or across a column-tile edge shows.  The bf16 output the
    bench uses must be the nearest-even rounding of the fp32 accumulator at every element."""
    M = 4096
    A, W = inputs.gemm_case(M, N, K)
    C32 = _gemm(A, W, torch.float32)
    c0 = N - 384
    ref = oracle_rows(oracle.gemm, A, np.ascontiguousarray(W[:, c0:c0 + 256]))
    g = C32[:, c0:c0 + 256].astype(np.float64)
    rms = np.sqrt((ref ** 2).mean(axis=1, keepdims=True))
    row_err = np.linalg.norm(g - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert row_err.max() <= 2e-3 and row_err.max() <= 1e-4, (int(row_err.argmax()), float(row_err.max()))
    assert np.all(np.abs(g - ref) <= 1e-3 * rms)
    Cb = _gemm(A, W, torch.bfloat16)
    assert np.array_equal(Cb, inputs.f32_to_bf16_bits(C32))


@pytest.mark.parametrize("K,N", WIDE_SHAPES)
@pytest.mark.parametrize("M", [1, 129, 300])
def test_small_int_exact_wide_plan(K, N, M):
    """Small-integer operands through the single-CTA plan of the wide weights: every partial sum
    is an exact integer in fp32, so every element must equal the oracle bit for bit.  K = 264
    ends in a ragged K block; M = 129 and 300 end in ragged row tiles; 32000 = 125 x 256 exactly,
    28672 = 112 x 256."""
    Ks = 264
    A = inputs.small_int_bf16(55, (M, Ks))
    W = inputs.small_int_bf16(56, (Ks, N))
    C = _gemm(A, W)
    ref = oracle_rows(oracle.gemm, A, W, block=16)
    assert np.array_equal(C.astype(np.float64), ref), int((C != ref).sum())


def test_empty_and_bad_args():
    A = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((64, 256), dtype=torch.bfloat16, device="cuda")
    assert binding.bi_gemm(A, W).shape == (0, 256)
    with pytest.raises(binding.BIError):
        binding.bi_gemm(torch.zeros((4, 60), dtype=torch.bfloat16, device="cuda"),
                        torch.zeros((60, 256), dtype=torch.bfloat16, device="cuda"))


def _device_rows(seed: int, M: int, K: int) -> torch.Tensor:
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((M, K), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("K,N", LLAMA_SHAPES + [(256, 512)] + WIDE_SHAPES)
def test_batch_invariance(K, N):
    W = dev(inputs.normal_bf16(inputs.SEED_WEIGHTS, (K, N), 0, 0.02))
    probes = dev(inputs.normal_bf16(inputs.SEED_PROBES, (8, K)))
    fill = {}

    def filler(trial):
        if trial not in fill:
            fill[trial] = _device_rows(inputs.SEED_FILLER_BASE + trial, 8192, K)
        return fill[trial]

    run = lambda batch: binding.bi_gemm(batch.contiguous(), W, out_dtype=torch.float32)
    rep = harness.bi_check_rows(f"gemm_{K}x{N}", run, probes, filler, inputs.m_sweep(8192))
    harness.rerun_check_rows(run, filler(0)[:1024], n=10, report=rep)
    assert rep.violations == 0, rep.as_dict()
    assert rep.rerun_violations == 0, rep.as_dict()
    assert binding.bi_get_device_error() == 0
