"""The K split of bi_gemm's CTA-pair plan on the GPU.

"Defeating Nondeterminism in LLM Inference", section "Multiplicación de matrices": a split
of K is batch-invariant when it does not depend on the batch.  bi_ctrl_gemm_split runs
bi_gemm's tiles with a split count given by the caller (S = 1: the CTA-pair kernel; S > 1:
the cluster-split kernel, S CTA pairs whose partials meet in distributed shared memory),
which the tests below use to reach every S.

  * small-integer operands: every partial sum is exact in fp32, so the output equals the
    oracle bit for bit at every S.
  * the slice order: partials 2^24, 1, 1, 0 add to 2^24 only in the order
    ((P0 + P1) + P2) + P3 (any order that adds the two 1s first gives 2^24 + 2).
  * random operands: relative Frobenius error <= 1e-5 against the fp64 oracle.
  * bits of a row do not depend on the batch at a fixed S.
  * no workspace is needed, and two calls in a row give the same bits.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import dev, host, rel_frobenius
from invariant_deterministic_rmsnorm_b200 import binding, inputs

pytestmark = pytest.mark.gpu

# 2 row tiles (the second ragged), 4 column tiles (the last 8 wide), 33 K blocks (the last
# 8 deep): slices of 16/17, 11/11/11 and 8/8/8/9 blocks
RAGGED = (333, 776, 2056)


def _split(A_np, W_np, S, out=torch.float32):
    C = binding.bi_ctrl_gemm_split(dev(A_np), dev(W_np), S, out_dtype=out)
    torch.cuda.synchronize()
    return host(C)


@pytest.mark.parametrize("S", [1, 2, 3, 4])
def test_split_small_int_exact(S):
    M, N, K = RAGGED
    A = inputs.small_int_bf16(61, (M, K))
    W = inputs.small_int_bf16(62, (K, N))
    C = _split(A, W, S)
    ref = oracle.gemm(A, W)
    assert np.array_equal(C.astype(np.float64), ref), int((C != ref).sum())


@pytest.mark.parametrize("S", [2, 3, 4])
def test_split_random_parity(S):
    M, N, K = RAGGED
    A, W = inputs.gemm_case(M, N, K, seed_a=63, seed_w=64)
    C = _split(A, W, S)
    assert rel_frobenius(C, oracle.gemm(A, W)) <= 1e-5


def _order_case(K=4096, N=8):
    """A row of ones; W puts 2^24 in slice 0 (1024 x 2^14), 1 in slice 1, 1 in slice 2 (S = 4)."""
    A = inputs.f32_to_bf16_bits(np.ones((3, K), np.float32))
    Wf = np.zeros((K, N), np.float32)
    Wf[:1024, :] = 2.0 ** 14
    Wf[1024, :] = 1.0
    Wf[2048, :] = 1.0
    return A, inputs.f32_to_bf16_bits(Wf)


def test_split_partials_add_in_slice_order():
    A, W = _order_case()
    exact = oracle.gemm(A, W)[0, 0]
    assert exact == 2.0 ** 24 + 2  # the oracle is exact
    p = [np.float32(2.0 ** 24), np.float32(1), np.float32(1), np.float32(0)]
    ordered = ((p[0] + p[1]) + p[2]) + p[3]
    assert float(ordered) == 2.0 ** 24  # fp32, round to nearest even at each add
    C = _split(A, W, 4)
    assert np.all(C == ordered), C[0, :4]


@pytest.mark.parametrize("K,N", [(4096, 6144), (14336, 4096)])
def test_plan_is_the_ctrl_kernel_at_the_plan_split(K, N):
    """bi_gemm runs the CTA-pair kernel at its plan's split count: the same bits as the control."""
    S = binding.gemm_splits(N, K)
    assert S == 1
    A, W = inputs.gemm_case(300, N, K, seed_a=73, seed_w=74)
    C = host(binding.bi_gemm(dev(A), dev(W)))
    torch.cuda.synchronize()
    assert np.array_equal(C.view(np.uint32), _split(A, W, S).view(np.uint32))


@pytest.mark.parametrize("S", [2, 4])
def test_split_rows_are_batch_invariant(S):
    M, N, K = 300, 776, 2056
    A, W = inputs.gemm_case(M, N, K, seed_a=65, seed_w=66)
    full = _split(A, W, S)
    for r in (0, 149, 255, 256, 299):
        solo = _split(A[r:r + 1], W, S)
        assert np.array_equal(solo[0].view(np.uint32), full[r].view(np.uint32)), r


def test_no_workspace_and_repeatable():
    M, N, K = RAGGED
    lib = binding.library()
    for S in (1, 2, 3, 4):
        assert lib.bi_ctrl_gemm_split_workspace_size(M, N, K, S) == 0
    assert lib.bi_gemm_workspace_size(M, N, K) == 0
    A, W = inputs.gemm_case(M, N, K, seed_a=67, seed_w=68)
    binding.bi_clear_device_error()
    first = _split(A, W, 3)
    again = _split(A, W, 3)
    assert np.array_equal(first.view(np.uint32), again.view(np.uint32))
    assert binding.bi_get_device_error() == 0


@pytest.mark.parametrize("S", [2, 3, 4])
def test_split_bf16_output_is_the_rounded_fp32(S):
    M, N, K = RAGGED
    A, W = inputs.gemm_case(M, N, K, seed_a=75, seed_w=76)
    assert np.array_equal(_split(A, W, S, torch.bfloat16), inputs.f32_to_bf16_bits(_split(A, W, S)))


def test_split_argument_errors():
    A, W = inputs.gemm_case(8, 4096, 4096, seed_a=69, seed_w=70)
    a, w = dev(A), dev(W)
    with pytest.raises(binding.BIError):
        binding.bi_ctrl_gemm_split(a, w, 5)
    with pytest.raises(binding.BIError):
        binding.bi_ctrl_gemm_split(a, w, 0)
    wide = dev(inputs.gemm_case(8, 28672, 64, seed_a=71, seed_w=72)[1])
    with pytest.raises(binding.BIError):
        binding.bi_ctrl_gemm_split(dev(A[:, :64]), wide, 2)
    torch.cuda.synchronize()
