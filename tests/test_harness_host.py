"""Host logic of the batch-invariance harness, checked with CPU stand-in ops (no GPU)."""
import numpy as np

from invariant_deterministic_rmsnorm_b200 import harness, inputs


def _rows(M, H=16, seed=0):
    return list(inputs.normal(seed, (M, H)))


def _filler(trial, M):
    return _rows(M, seed=1000 + trial)


def _rowwise(batch):
    X = np.stack(batch)
    return list(np.tanh(X) * np.float32(0.5))


def _batch_dependent(batch):
    # the row result depends on the batch size: a stand-in for a split chosen by M
    X = np.stack(batch).astype(np.float32)
    return list(X * np.float32(1.0 + 1e-6 * len(batch)))


def test_rowwise_op_has_no_violations():
    rep = harness.bi_check("rowwise", _rowwise, _rows(4, seed=2), _filler, [1, 3, 8, 33, 100])
    assert rep.violations == 0 and rep.comparisons == 1 * 1 * 3 + 3 * 3 + 4 * 3 * 3


def test_batch_dependent_op_is_caught():
    rep = harness.bi_check("dep", _batch_dependent, _rows(4, seed=2), _filler, [1, 2, 8])
    assert rep.violations > 0 and rep.first_failure["M"] in (2, 8)


def test_position_dependent_op_is_caught():
    def posdep(batch):
        X = np.stack(batch)
        return [X[i] + np.float32(i * 1e-3) for i in range(len(batch))]
    rep = harness.bi_check("pos", posdep, _rows(2, seed=2), _filler, [16])
    assert rep.violations > 0


def test_signed_zero_counts_as_violation():
    assert not harness.same_bits(np.array([0.0], np.float32), np.array([-0.0], np.float32))
    assert harness.same_bits(np.array([1.5], np.float32), np.array([1.5], np.float32))


def test_rerun_check():
    rep = harness.rerun_check(_rowwise, _rows(5), n=10)
    assert rep.reruns == 9 and rep.rerun_violations == 0
    rng = np.random.default_rng(0)
    noisy = lambda b: [r + np.float32(rng.standard_normal() * 1e-3) for r in b]
    rep = harness.rerun_check(noisy, _rows(5), n=4)
    assert rep.rerun_violations == 3


def test_positions_are_distinct_and_in_range():
    for M in (1, 5, 8, 9, 8192):
        rep = harness.bi_check("rowwise", _rowwise, _rows(8, seed=2), lambda t, m: _rows(m, seed=1000 + t),
                               [M], trials=1)
        assert rep.comparisons == min(M, 8)


def test_pin_tuple_has_fields():
    d = harness.pin_tuple({"config": "x"})
    for k in ("torch", "git", "utc", "config"):
        assert k in d


def test_bi_check_rows_on_cpu_tensors():
    import torch
    g = torch.Generator().manual_seed(0)
    probes = torch.randn(4, 16, generator=g)
    fill = {t: torch.randn(64, 16, generator=torch.Generator().manual_seed(100 + t)) for t in range(3)}
    rowwise = lambda b: torch.tanh(b) * 0.5
    rep = harness.bi_check_rows("rowwise", rowwise, probes, lambda t: fill[t], [1, 5, 64])
    assert rep.violations == 0 and rep.comparisons == 3 + 4 * 3 + 4 * 3
    dep = lambda b: b * (1.0 + 1e-6 * b.shape[0])
    assert harness.bi_check_rows("dep", dep, probes, lambda t: fill[t], [1, 5]).violations > 0
    # a reduction whose order depends on M: the sum over a row split into M-dependent chunks
    def split_sum(b):
        chunks = 2 if b.shape[0] > 3 else 1
        parts = torch.tensor_split(b, chunks, dim=1)
        s = parts[0].sum(1, keepdim=True)
        for p in parts[1:]:
            s = s + p.sum(1, keepdim=True)
        return s.expand_as(b).contiguous()
    assert harness.bi_check_rows("split", split_sum, probes, lambda t: fill[t], [1, 8]).violations > 0
    rep = harness.rerun_check_rows(rowwise, fill[0], n=5)
    assert rep.reruns == 4 and rep.rerun_violations == 0
