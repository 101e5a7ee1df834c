"""bi_rmsnorm on the GPU: parity with the fp64 oracle, bitwise batch invariance, edges.

Tolerances:
  * fp32 output: max |g - r| / max(|r|, 1e-3 * rms(row)) <= 1e-5 against the unrounded fp64 oracle.
  * bf16 output: within 1 bf16 step of the oracle's own nearest-even rounding of its fp64 result,
    and at most 0.1 % of elements one step away.  The fp32 kernel result sits within about
    1e-6 relative of the exact value, so it can land on the other side of a bf16 rounding
    boundary only for values within about 1e-6 relative of that boundary.  That is roughly
    2 * 1e-6 / 2^-8 ~ 0.05 % of uniformly placed values.
  * batch invariance: exact bits, solo vs embedded at random positions, M = 1 .. 8192.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bf16_ulp_distance, dev, host, rel_err_rowscaled
from invariant_deterministic_rmsnorm_b200 import binding, harness, inputs

pytestmark = pytest.mark.gpu
EPS = 1e-6


def _run(x_np, w_np, eps=EPS):
    y = binding.bi_rmsnorm(dev(x_np), dev(w_np), eps=eps)
    torch.cuda.synchronize()
    return host(y)


def _check_f32(x, w, y, eps=EPS):
    ref = oracle.rmsnorm(x, w, eps)
    err = rel_err_rowscaled(y.astype(np.float64), ref)
    assert err <= 1e-5, err


def _check_bf16(x, w, y, eps=EPS):
    ref = oracle.round_bf16(oracle.rmsnorm(x, w, eps))
    d = bf16_ulp_distance(y, ref)
    assert d.max() <= 1, int(d.max())
    assert (d == 1).mean() <= 1e-3, float((d == 1).mean())


@pytest.mark.parametrize("M", [1, 3, 8, 32])
def test_parity_f32_h256(M):
    x, w = inputs.rmsnorm_case(M, 256, "f32")
    _check_f32(x, w, _run(x, w))


@pytest.mark.parametrize("M", [1, 7, 129, 1025])
def test_parity_bf16_h4096(M):
    x, w = inputs.rmsnorm_case(M, 4096, "bf16")
    _check_bf16(x, w, _run(x, w))


def test_parity_full_size_bf16():
    """The bench's launch configuration: M = 8192, H = 4096, every row against the oracle."""
    x, w = inputs.rmsnorm_case(8192, 4096, "bf16")
    _check_bf16(x, w, _run(x, w))


@pytest.mark.parametrize("H,dt", [(264, "f32"), (4104, "bf16"), (32768, "bf16"), (16384, "f32"), (8, "bf16"),
                                  (4, "f32"), (1000, "f32")])
def test_parity_ragged_and_max_h(H, dt):
    x, w = inputs.rmsnorm_case(5, H, dt, seed_x=17)
    y = _run(x, w)
    (_check_f32 if dt == "f32" else _check_bf16)(x, w, y)


def test_f32_rows_bf16_weights():
    x = inputs.rows(3, 4, 512, "f32")
    w = inputs.normal_bf16(4, (512,), 1.0, 0.1)
    _check_f32(x, w, _run(x, w))


def test_strided_rows_and_in_place():
    M, H = 6, 256
    x, w = inputs.rmsnorm_case(M, H, "f32")
    big = torch.zeros((M, H + 64), dtype=torch.float32, device="cuda")
    big[:, :H] = dev(x)
    view = big[:, :H]
    yv = binding.bi_rmsnorm(view, dev(w), eps=EPS)
    binding.bi_rmsnorm(view, dev(w), y=view, eps=EPS)  # in place
    torch.cuda.synchronize()
    assert np.array_equal(host(yv), host(view))
    assert torch.all(big[:, H:] == 0)
    _check_f32(x, w, host(yv))


def test_empty_batch_is_noop():
    x = torch.empty((0, 256), dtype=torch.float32, device="cuda")
    w = torch.ones(256, dtype=torch.float32, device="cuda")
    y = binding.bi_rmsnorm(x, w)
    assert y.shape == (0, 256)


def test_bad_args_raise():
    w = torch.ones(256, dtype=torch.float32, device="cuda")
    x = torch.ones((4, 258), dtype=torch.float32, device="cuda")
    with pytest.raises(binding.BIError):
        binding.bi_rmsnorm(x, torch.ones(258, dtype=torch.float32, device="cuda"))
    xo = torch.ones((4, 257), dtype=torch.float32, device="cuda")[:, 1:]
    with pytest.raises(binding.BIError):
        binding.bi_rmsnorm(xo, w)


def _row_runner(dtype_out):
    def run(batch):
        X = np.stack(batch)
        return list(_run(X, run.w))
    return run


@pytest.mark.parametrize("H,dt", [(256, "f32"), (4096, "bf16")])
def test_batch_invariance(H, dt):
    _, w = inputs.rmsnorm_case(1, H, dt)
    probes = list(inputs.rows(inputs.SEED_PROBES, 8 if dt == "bf16" else 4, H, dt))
    cache = {}

    def filler(trial, M):
        if trial not in cache:
            cache[trial] = inputs.rows(inputs.SEED_FILLER_BASE + trial, 8192, H, dt)
        return list(cache[trial][:M])

    run = _row_runner(dt)
    run.w = w
    rep = harness.bi_check(f"rmsnorm_{dt}_{H}", run, probes, filler, inputs.m_sweep(8192))
    harness.rerun_check(run, list(cache[0][:1000]), n=10, report=rep)
    assert rep.violations == 0, rep.as_dict()
    assert rep.rerun_violations == 0, rep.as_dict()
    assert binding.bi_get_device_error() == 0
