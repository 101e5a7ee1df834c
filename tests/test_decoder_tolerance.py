"""Pins the decoder parity tolerance (tests/decoder_case.py) from both sides, on the CPU.

  * Below: the oracle decoder with every inexact pre-rounding value perturbed by a relative
    1e-5 (a stand-in for fp32 accumulation error) stays within TOL / 2 of the unperturbed
    oracle.  The residual adds are exact in both paths, so they are left unperturbed.
  * Above: every planted wiring mistake moves some sequence's logits by more than 2 * TOL,
    so a GPU path that made one would fail the parity test.
"""
import numpy as np
import pytest

import oracle
from oracle import decoder as od
import decoder_case as case
from test_oracle_decoder_pins import MUTANTS, _mutant_module


class _Exact(np.ndarray):
    pass


def _run(mod, w, noise=0.0, seed=0):
    rng = np.random.default_rng(seed)
    plain_round, plain_add = mod.round_bf16, mod.add

    def round_perturbed(v, handle=None):
        exact = isinstance(v, _Exact)
        v = np.asarray(v, np.float64)
        if noise and not exact:
            v = v * (1.0 + noise * rng.standard_normal(v.shape))
        return oracle.round_bf16(v, handle)

    mod.round_bf16 = round_perturbed
    mod.add = lambda a, b: plain_add(a, b).view(_Exact)
    try:
        dec = mod.OracleDecoder(case.SHAPE, w, case.MAX_SEQS, case.CAP)
        return [dec.forward(case.SLOTS, toks) for toks, _ in case.steps()]
    finally:
        mod.round_bf16, mod.add = plain_round, plain_add


@pytest.fixture(scope="module")
def reference():
    w = case.weights()
    return w, _run(od, w)


def test_fp32_scale_perturbations_stay_under_half_the_tolerance(reference):
    w, ref = reference
    worst = max(max(case.rel_errors(g, r)) for seed in (1, 2) for g, r in zip(_run(od, w, 1e-5, seed), ref))
    assert 1e-4 < worst <= case.TOL / 2, worst


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_wiring_mistakes_exceed_twice_the_tolerance(reference, name):
    w, ref = reference
    mod = _mutant_module(*MUTANTS[name])
    got = _run(mod, w)
    worst = max(max(case.rel_errors(g, r)) for g, r in zip(got, ref))
    assert worst > 2 * case.TOL, (name, worst)
