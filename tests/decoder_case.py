"""The small decoder workload on which the GPU decoder is compared with the oracle decoder.

Shape: 2 layers, hidden 512, 4 query / 2 kv heads of 128, ffn 768, vocabulary 1000.  Weights:
matrices ~ N(0, 0.05), norm weights ~ N(1, 0.3).  These are wider than the serving init, so
that a wiring mistake (a wrong norm weight, head layout or RoPE pairing) moves the logits by
10 % or more.  Prompts of 1, 37 and 65 tokens in slots 0, 2 and 3, then 3 decode steps of
seeded (teacher-forced) tokens, so that both sides see the same inputs at every step.

Tolerance.  The GPU and the oracle round the same tensors to bf16 at the same points.  Their
pre-rounding values differ by fp32 accumulation error, and a bf16 step flips wherever that
difference straddles a rounding boundary.  Those flips compound through the layers.  The
oracle itself, with its pre-rounding values perturbed by a relative 1e-5, moves its logits by
about 1 % on this workload.  TOL is 3 % per sequence and step (relative Frobenius norm).
tests/test_decoder_tolerance.py pins both sides of that choice: the perturbed oracle stays
under TOL / 2, and every planted wiring mistake exceeds 2 * TOL.
"""
import numpy as np

from invariant_deterministic_rmsnorm_b200 import inputs

SHAPE = inputs.TINY_DECODER
LENS = [1, 37, 65]
SLOTS = [0, 2, 3]
MAX_SEQS = 4
CAP = 256
DECODE = 3
TOL = 3e-2


def weights():
    return inputs.decoder_weights_host(SHAPE, matrix_std=0.05, norm_std=0.3)


def steps():
    prompts = [inputs.prompt(i, n, SHAPE.vocab) for i, n in enumerate(LENS)]
    forced = np.random.default_rng(60).integers(0, SHAPE.vocab, (DECODE, len(LENS))).astype(np.int32)
    return [(prompts, "prefill")] + [([[int(t)] for t in row], "decode") for row in forced]


def rel_errors(got, ref):
    """Relative Frobenius error of each sequence's logits."""
    return [float(np.linalg.norm(np.asarray(g, np.float64) - r) / np.linalg.norm(r)) for g, r in zip(got, ref)]
