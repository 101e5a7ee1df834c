"""bi_rmsnorm_lora_shrink on the GPU: bitwise the two calls it fuses, parity with the fp64
oracle, batch invariance and replay.

The fused kernel must give exactly the bits of bi_rmsnorm followed by bi_lora_shrink on its
output, because it runs the same operations on every element in the same order.  Those two ops
are pinned to the oracle in their own tests; the parity check here repeats it for the fused
entry point on its own (tolerances of those tests: y within one bf16 rounding, t relative
Frobenius error <= 1e-4 against the oracle's split-8 sum).
"""
import pytest
import torch

import oracle
from gpu_util import bf16_ulp_distance, dev, host, rel_frobenius
from invariant_deterministic_rmsnorm_b200 import binding, harness, inputs

pytestmark = pytest.mark.gpu
H = 4096
EPS = 1e-6


def _case(M, r, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((M, H), generator=g, device="cuda").to(torch.bfloat16)
    w = (1.0 + 0.1 * torch.randn((H,), generator=g, device="cuda")).to(torch.bfloat16)
    A = (0.02 * torch.randn((H, r), generator=g, device="cuda")).to(torch.bfloat16)
    return x, w, A


def _separate(x, w, A):
    y = binding.bi_rmsnorm(x, w, eps=EPS)
    t = binding.bi_lora_shrink(y, A, split_k=8)
    return y, t


@pytest.mark.parametrize("r", [8, 16])
@pytest.mark.parametrize("M", [1, 3, 4, 5, 7, 257, 1000, 4096])
def test_bitwise_equal_to_the_two_calls(r, M):
    """Every tile size that occurs: one row, a partial first tile, exact tiles, a partial last
    tile after many (257, 1000), and the bench's M = 4096 (1024 tiles on 148 CTAs)."""
    x, w, A = _case(M, r, 100 + M + r)
    y_ref, t_ref = _separate(x, w, A)
    y, t = binding.bi_rmsnorm_lora_shrink(x, w, A, eps=EPS)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), int((y != y_ref).sum())
    assert torch.equal(t.view(torch.int32), t_ref.view(torch.int32)), int((t != t_ref).sum())
    assert binding.bi_get_device_error() == 0


def test_strided_rows_and_in_place():
    """x and y as column slices of wider buffers (row strides 6144 and 4608), then y over x."""
    M, r = 300, 16
    x0, w, A = _case(M, r, 7)
    wide_x = torch.zeros((M, 6144), dtype=torch.bfloat16, device="cuda")
    wide_x[:, 1024:1024 + H] = x0
    wide_y = torch.full((M, 4608), 7.0, dtype=torch.bfloat16, device="cuda")
    y_ref, t_ref = _separate(x0, w, A)
    y, t = binding.bi_rmsnorm_lora_shrink(wide_x[:, 1024:1024 + H], w, A, y=wide_y[:, :H], eps=EPS)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(t.view(torch.int32), t_ref.view(torch.int32))
    assert bool((wide_y[:, H:] == 7.0).all()), "a column past H was written"
    xi = x0.clone()
    y2, t2 = binding.bi_rmsnorm_lora_shrink(xi, w, A, y=xi, eps=EPS)
    torch.cuda.synchronize()
    assert y2.data_ptr() == xi.data_ptr()
    assert torch.equal(xi.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(t2.view(torch.int32), t_ref.view(torch.int32))


@pytest.mark.parametrize("r", [8, 16])
def test_parity_with_the_oracle(r):
    """The oracle's RMSNorm (fp64, rounded to bf16 once) and its split-8 shrink of that output."""
    M = 37
    x, w, A = _case(M, r, 55 + r)
    y, t = binding.bi_rmsnorm_lora_shrink(x, w, A, eps=EPS)
    torch.cuda.synchronize()
    x_np, w_np, A_np = host(x), host(w), host(A)
    # y: within one bf16 step of the oracle's own rounding of its fp64 result, as bi_rmsnorm's test
    d = bf16_ulp_distance(host(y), oracle.round_bf16(oracle.rmsnorm(x_np, w_np, EPS)))
    assert d.max() <= 1, int(d.max())
    assert (d == 1).mean() <= 1e-3, float((d == 1).mean())
    t_o = oracle.lora_shrink_split(host(y), A_np, 8)          # the shrink of the kernel's own y
    err = rel_frobenius(host(t), t_o)
    assert err <= 1e-4, err


def test_batch_invariance_and_replay():
    r = 16
    _, w, A = _case(1, r, 3)
    probes = dev(inputs.normal_bf16(inputs.SEED_PROBES, (8, H)))
    fill = {}

    def filler(trial):
        if trial not in fill:
            g = torch.Generator(device="cuda").manual_seed(inputs.SEED_FILLER_BASE + trial)
            fill[trial] = torch.randn((4096, H), generator=g, device="cuda").to(torch.bfloat16)
        return fill[trial]

    def run(batch):
        y, t = binding.bi_rmsnorm_lora_shrink(batch.contiguous(), w, A, eps=EPS)
        return torch.cat([y.float(), t], dim=1)

    rep = harness.bi_check_rows("rmsnorm_lora_shrink", run, probes, filler,
                                [m for m in inputs.m_sweep(4096)])
    harness.rerun_check_rows(run, filler(0)[:1024], n=10, report=rep)
    assert rep.violations == 0, rep.as_dict()
    assert rep.rerun_violations == 0, rep.as_dict()
    assert binding.bi_get_device_error() == 0


def test_unsupported_shapes_are_refused():
    x, w, A = _case(8, 16, 1)
    with pytest.raises(binding.BIError):  # r = 32: the B fragments would not fit in registers
        binding.bi_rmsnorm_lora_shrink(x, w, (0.02 * torch.randn((H, 32), device="cuda")).to(torch.bfloat16))
    with pytest.raises(binding.BIError):  # split_k = 4
        binding.bi_rmsnorm_lora_shrink(x, w, A, split_k=4)
    x2 = torch.randn((8, 2048), device="cuda").to(torch.bfloat16)
    with pytest.raises(binding.BIError):  # H = 2048
        binding.bi_rmsnorm_lora_shrink(x2, w[:2048].contiguous(), A[:2048].contiguous())
    y0, t0 = binding.bi_rmsnorm_lora_shrink(x[:0], w, A)  # an empty batch is a no-op
    assert y0.shape == (0, H) and t0.shape == (0, 16)
    assert binding.bi_get_device_error() == 0
