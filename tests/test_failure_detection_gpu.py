"""A device-side wait that runs out becomes a host-visible status, and the context survives.

Every kernel's waits are bounded.  When one gives up, the kernel ORs a cause bit into the
library's device error word and returns.  Here a probe kernel waits on an mbarrier that nothing
arrives on (no fault, no trap, no unbounded spin); the wait must give up after its 1 ms limit,
and the next op on the same stream must still run and give correct bits.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_util import dev, host
from invariant_deterministic_rmsnorm_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_and_the_context_survives():
    binding.bi_clear_device_error()
    assert binding.bi_get_device_error() == 0
    t0 = time.perf_counter()
    binding.bi_ctrl_wait_timeout_probe(1_000_000)  # 1 ms
    code = binding.bi_get_device_error()
    elapsed = time.perf_counter() - t0
    assert code & 0x2, hex(code)
    assert elapsed < 1.0  # the wait gave up near its limit, not at the kernels' 2 s default
    binding.bi_clear_device_error()
    # the same context runs an op and the status word is clean again
    x, w = inputs.rmsnorm_case(8, 256, "f32")
    y = host(binding.bi_rmsnorm(dev(x), dev(w), eps=1e-6))
    ref = oracle.rmsnorm(x, w, 1e-6)
    assert np.max(np.abs(y - ref) / np.maximum(np.abs(ref), 1e-6)) <= 1e-5
    assert binding.bi_get_device_error() == 0


def test_probe_rejects_limits_outside_its_range():
    with pytest.raises(binding.BIError):
        binding.bi_ctrl_wait_timeout_probe(10)
    with pytest.raises(binding.BIError):
        binding.bi_ctrl_wait_timeout_probe(5_000_000_000)
