"""The position-invariant scheduling contrast, asserted on the GPU.

Source: the CoRun forum post and its comment thread ("You think you are measuring
intelligence...", thecolony.si): instead of batch-invariant kernels, keep the fast
batch-dependent kernels and fix every shape, prefilling each request alone and decoding a
fixed 128-slot batch replayed from one CUDA graph.  The bench's contrast measurement
(bench.contrast_composition) runs the same synthetic 4-layer Llama-3-8B-shaped decoder three
ways.  Asserted here, bit for bit, over a probe's logits at 8 greedy decode steps after its
prefill:
  - fixed 128-slot shape with the fast kernels: the same alone and among real co-residents,
    and the same in slot 5 and slot 77 (its shapes never change);
  - the fast kernels at the true batch size: alone and in a batch of 37 differ (cuBLAS, the
    split RMSNorm and the batch-adaptive split-KV all change a row's arithmetic with M);
  - the batch-invariant kernels: alone equals in a batch of 37 and in a batched 128-request
    prefill.
Prompts are U[130, 400] tokens (the contrast uses U[16, 2048]; the shorter ones keep 128
isolated prefills quick, and are all longer than the 128-token split the adaptive attention
takes for small batches).
"""
import numpy as np
import pytest

import bench
from invariant_deterministic_rmsnorm_b200 import inputs
from invariant_deterministic_rmsnorm_b200.decoder import Decoder

pytestmark = pytest.mark.gpu


def test_position_invariant_scheduling_contrast():
    shape = inputs.LLAMA3_8B_4L
    w = inputs.decoder_weights_device(shape)
    BF, steps = 128, 8
    lens = np.random.default_rng(inputs.SEED_PROMPT_BASE - 1).integers(130, 401, size=BF)
    prompts = [inputs.prompt(i, int(n), shape.vocab) for i, n in enumerate(lens)]
    filler = inputs.prompt(inputs.SEED_FILLER_BASE, 16, shape.vocab)
    max_len = 400 + steps + 8
    dec_bi = Decoder(shape, w, BF, max_len)
    dec_fast = Decoder(shape, w, BF, max_len, ops=bench.FastOps)
    got = bench.contrast_composition(dec_bi, dec_fast, prompts, filler, BF, steps)
    assert got["fast_fixed128_alone_vs_busy_same_slot"], got
    assert got["fast_fixed128_slot5_vs_slot77"], got
    assert not got["fast_dynamic_alone_vs_batch37"], got
    assert got["fast_dynamic_max_abs_diff"] > 0.0, got
    assert got["bi_alone_vs_batch37"], got
    assert got["bi_alone_vs_batch128_batched_prefill"], got
