"""bi_lora_shrink / bi_lora_expand on the GPU: exact pins, parity with the fp64 oracle,
bitwise batch invariance and replay determinism, and the atomic comparator as a positive control.

Tolerances:
  * small-integer operands: every partial sum is an integer below 2^24, exact in fp32 in any
    order, so the result must equal the oracle bit for bit (shrink: t; expand: fp32 y).
  * random operands: relative Frobenius error <= 2e-3 against the fp64 oracle (shrink: t;
    expand: the added term y_out - y_in, with fp32 y).
  * bf16 y: elementwise |g - r| <= 2^-8 |r| + 1e-3 * rms(delta row) (one bf16 rounding).
  * batch invariance and replay: exact bits.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bf16_to_f64, dev, host, oracle_rows, rel_frobenius
from invariant_deterministic_rmsnorm_b200 import binding, harness, inputs

pytestmark = pytest.mark.gpu
K = 4096
N = 4096


def _shrink(x_np, A_np, split=8):
    t = binding.bi_lora_shrink(dev(x_np), dev(A_np), split_k=split)
    torch.cuda.synchronize()
    return host(t)


@pytest.mark.parametrize("r", [8, 16, 32, 64])
@pytest.mark.parametrize("split", [8, 1])
def test_shrink_small_int_exact(r, split):
    M = 130
    x = inputs.small_int_bf16(64, (M, K))
    A = inputs.small_int_bf16(65, (K, r))
    t = _shrink(x, A, split)
    assert np.array_equal(t.astype(np.float64), oracle.lora_shrink(x, A))


@pytest.mark.parametrize("r", [8, 16, 64])
@pytest.mark.parametrize("M", [1, 65, 257])
def test_shrink_parity(r, M):
    x, A, _, _ = inputs.lora_case(M, r)
    t = _shrink(x, A)
    ref = oracle.lora_shrink_split(x, A, 8)
    err = rel_frobenius(t, ref)
    assert err <= 2e-3, err
    assert err <= 1e-4, err


@pytest.mark.parametrize("r", [8, 16, 64])
def test_shrink_parity_full_size(r):
    """The bench's launch configuration, M = 4096 (32 tiles of 128 rows, every one a full
    cluster of 8 K slices): every row against the oracle's split-8 sum."""
    M = 4096
    x, A, _, _ = inputs.lora_case(M, r)
    t = _shrink(x, A)
    ref = oracle_rows(oracle.lora_shrink_split, x, A, 8)
    row_err = np.linalg.norm(t - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert rel_frobenius(t, ref) <= 2e-3
    assert row_err.max() <= 1e-4, (int(row_err.argmax()), float(row_err.max()))


def test_shrink_other_k_and_splits():
    M, Kx, r = 100, 14336, 16
    x = inputs.normal_bf16(71, (M, Kx))
    A = inputs.normal_bf16(72, (Kx, r), 0, 0.02)
    ref = oracle.lora_shrink(x, A)
    for split in (1, 2, 4, 8):
        assert rel_frobenius(_shrink(x, A, split), ref) <= 1e-4


@pytest.mark.parametrize("r", [16, 64])
@pytest.mark.parametrize("split", [2, 4, 8])
def test_shrink_persistent_tiles_every_split(r, split):
    """M = 9000 is 71 row tiles, more than the GPU's clusters hold at once, so every cluster walks
    several tiles and its receive buffer turns over (the per-tile byte counts the combiners post
    on their receive barriers).  Rows sampled across the tiles match the oracle's split sum, and a
    second launch gives the same bits."""
    M = 9000
    x, A, _, _ = inputs.lora_case(M, r)
    xd, Ad = dev(x), dev(A)
    t = binding.bi_lora_shrink(xd, Ad, split_k=split)
    again = binding.bi_lora_shrink(xd, Ad, split_k=split)
    torch.cuda.synchronize()
    assert torch.equal(t.view(torch.int32), again.view(torch.int32))
    rows = np.unique(np.concatenate([np.arange(0, M, 257), [M - 1]]))
    ref = oracle.lora_shrink_split(x[rows], A, split)
    got = host(t)[rows]
    row_err = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert row_err.max() <= 1e-4, (row_err.max(), rows[np.argmax(row_err)])
    assert binding.bi_get_device_error() == 0


def test_shrink_rejects_bad_shapes():
    x = torch.zeros((4, 4096), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.BIError):
        binding.bi_lora_shrink(x, torch.zeros((4096, 12), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(binding.BIError):
        binding.bi_lora_shrink(x, torch.zeros((4096, 16), dtype=torch.bfloat16, device="cuda"), split_k=3)
    assert binding.bi_lora_shrink(torch.zeros((0, 4096), dtype=torch.bfloat16, device="cuda"),
                                  torch.zeros((4096, 16), dtype=torch.bfloat16, device="cuda")).shape == (0, 16)


def _device_rows(seed, M, cols, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((M, cols), generator=g, device="cuda", dtype=torch.float32).to(dtype)


@pytest.mark.parametrize("r", [8, 16, 64])
def test_shrink_batch_invariance_and_replay(r):
    A = dev(inputs.normal_bf16(inputs.SEED_WEIGHTS, (K, r), 0, 0.02))
    probes = dev(inputs.normal_bf16(inputs.SEED_PROBES, (8, K)))
    fill = {}

    def filler(trial):
        if trial not in fill:
            fill[trial] = _device_rows(inputs.SEED_FILLER_BASE + trial, 4096, K)
        return fill[trial]

    run = lambda b: binding.bi_lora_shrink(b.contiguous(), A, split_k=8)
    rep = harness.bi_check_rows(f"lora_shrink_r{r}", run, probes, filler, inputs.m_sweep(4096))
    harness.rerun_check_rows(run, filler(0), n=10, report=rep)
    assert rep.violations == 0, rep.as_dict()
    assert rep.rerun_violations == 0, rep.as_dict()
    assert binding.bi_get_device_error() == 0


@pytest.mark.parametrize("r", [8, 16, 32, 64])
def test_shrink_replay_stress(r):
    """Forty launches of one shrink, each into a fresh output, are bit-identical, and the first
    matches the oracle row by row.  M = 5000 makes the persistent CTAs take a second tile.  A
    ring stage handed back without a proxy fence after its ldmatrix reads let the next TMA refill
    land under the slowest warp's last loads: the first rows of a few tiles then came out wrong in
    most launches at r = 64 (three ring stages), so this test fails on that hazard."""
    M = 5000
    x, A, _, _ = inputs.lora_case(M, r)
    xd, Ad = dev(x), dev(A)
    outs = [binding.bi_lora_shrink(xd, Ad, split_k=8) for _ in range(40)]
    torch.cuda.synchronize()
    differ = [i for i, t in enumerate(outs) if not torch.equal(t.view(torch.int32), outs[0].view(torch.int32))]
    assert differ == [], f"{len(differ)} of 39 replays differ from the first"
    exact = oracle_rows(oracle.lora_shrink_split, x, A, 8)
    got = host(outs[0])
    row_err = np.linalg.norm(got - exact, axis=1) / np.linalg.norm(exact, axis=1)
    assert row_err.max() <= 1e-4, (row_err.max(), np.argmax(row_err))
    assert binding.bi_get_device_error() == 0


def test_atomic_comparator_varies_under_replay():
    """Positive control: the same shrink with atomic combination changes bits between identical runs."""
    r, M = 16, 4096
    x = _device_rows(5, M, K)
    A = dev(inputs.normal_bf16(inputs.SEED_WEIGHTS, (K, r), 0, 0.02))
    first = binding.bi_ctrl_lora_shrink_atomic(x, A).clone()
    differ = 0
    for _ in range(20):
        t = binding.bi_ctrl_lora_shrink_atomic(x, A)
        differ += int(not torch.equal(t.view(torch.int32), first.view(torch.int32)))
    det = binding.bi_lora_shrink(x, A)
    # the atomic result is still a correct shrink, within tolerance of the ordered one
    assert rel_frobenius(host(first), host(det)) <= 1e-5
    assert differ > 0, "atomic split-K never varied: the positive control is blind"


# ------------------------------------------------------------------ expand
def _expand(t_np, B_np, y_np, scale=1.0):
    y = dev(y_np)
    binding.bi_lora_expand(dev(t_np), dev(B_np), y, scale=scale)
    torch.cuda.synchronize()
    return host(y)


@pytest.mark.parametrize("r", [8, 16, 32, 64])
def test_expand_small_int_exact_f32(r):
    M = 70
    t = oracle.bf16_bits_to_f64(inputs.small_int_bf16(81, (M, r))).astype(np.float32)
    B = inputs.small_int_bf16(82, (r, N))
    y = oracle.bf16_bits_to_f64(inputs.small_int_bf16(83, (M, N))).astype(np.float32)
    out = _expand(t, B, y, scale=2.0)
    assert np.array_equal(out.astype(np.float64), oracle.lora_expand(t, B, y, 2.0))


@pytest.mark.parametrize("r", [8, 16, 64])
@pytest.mark.parametrize("M", [1, 65, 257])
def test_expand_parity_f32_delta(r, M):
    x, A, B, _ = inputs.lora_case(M, r)
    t = oracle.round_f32(oracle.lora_shrink(x, A))
    y = inputs.normal(9, (M, N))
    out = _expand(t, B, y, scale=0.5)
    ref = oracle.lora_expand(t, B, y, 0.5)
    err = rel_frobenius(out.astype(np.float64) - y, ref - y)
    assert err <= 2e-3, err


@pytest.mark.parametrize("r", [8, 64])
def test_expand_parity_bf16(r):
    M = 129
    x, A, B, y = inputs.lora_case(M, r)
    t = oracle.round_f32(oracle.lora_shrink(x, A))
    out = bf16_to_f64(_expand(t, B, y, scale=2.0))
    ref = oracle.lora_expand(t, B, y, 2.0)
    delta = ref - bf16_to_f64(y)
    rms = np.sqrt((delta ** 2).mean(axis=1, keepdims=True))
    assert np.all(np.abs(out - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3 * rms)


def test_expand_strided_y():
    """y is the first 4096 columns of a wider [M, 6144] buffer (e.g. the q part of a fused qkv)."""
    M, r = 33, 16
    x, A, B, _ = inputs.lora_case(M, r)
    t = oracle.round_f32(oracle.lora_shrink(x, A))
    wide = _device_rows(3, M, 6144, torch.float32)
    before = wide.clone()
    binding.bi_lora_expand(dev(t), dev(B), wide[:, :N], scale=1.0)
    torch.cuda.synchronize()
    assert torch.equal(wide[:, N:], before[:, N:])
    ref = oracle.lora_expand(t, B, host(before[:, :N]).copy(), 1.0)
    assert rel_frobenius(host(wide[:, :N]).astype(np.float64) - host(before[:, :N]),
                         ref - host(before[:, :N])) <= 2e-3


@pytest.mark.parametrize("r", [8, 64])
def test_expand_batch_invariance(r):
    B = dev(inputs.normal_bf16(inputs.SEED_WEIGHTS + 1, (r, N), 0, 0.02))
    P = 8
    t_p = _device_rows(inputs.SEED_PROBES, P, r, torch.float32)
    y_p = _device_rows(inputs.SEED_PROBES + 1, P, N)
    solo = []
    for p in range(P):
        y1 = y_p[p:p + 1].clone()
        binding.bi_lora_expand(t_p[p:p + 1].clone(), B, y1)
        solo.append(y1.view(torch.int16).clone())
    t_f = {tr: _device_rows(1000 + tr, 4096, r, torch.float32) for tr in range(3)}
    y_f = {tr: _device_rows(2000 + tr, 4096, N) for tr in range(3)}
    bad = 0
    for M in inputs.m_sweep(4096):
        for tr in range(3):
            rng = np.random.default_rng([inputs.SEED_POSITIONS, M, tr])
            pos = rng.choice(M, size=min(M, P), replace=False)
            tb, yb = t_f[tr][:M].clone(), y_f[tr][:M].clone()
            for i, w in enumerate(pos):
                tb[int(w)] = t_p[i]
                yb[int(w)] = y_p[i]
            binding.bi_lora_expand(tb, B, yb)
            for i, w in enumerate(pos):
                bad += int(not torch.equal(yb[int(w)].view(torch.int16), solo[i][0]))
    assert bad == 0


# ------------------------------------------------------------------ the tcgen05 shrink
@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("M", [1, 130, 4096])
def test_shrink_tc(M, r):
    """bi_ctrl_lora_shrink_tc: small-integer operands exact (every partial sum is an integer below
    2^24), random operands within the shrink's tolerance of the oracle's split-8 sum, rows
    independent of the batch, and replays identical."""
    xi = inputs.small_int_bf16(66, (M, K))
    Ai = inputs.small_int_bf16(67, (K, r))
    t = host(binding.bi_ctrl_lora_shrink_tc(dev(xi), dev(Ai)))
    assert np.array_equal(t.astype(np.float64), oracle.lora_shrink(xi, Ai))
    x, A, _, _ = inputs.lora_case(M, r)
    xd, Ad = dev(x), dev(A)
    t = binding.bi_ctrl_lora_shrink_tc(xd, Ad)
    ref = oracle_rows(oracle.lora_shrink_split, x, A, 8)
    err = rel_frobenius(host(t), ref)
    assert err <= 2e-3 and err <= 1e-4, err
    for r_ in sorted({0, M // 2, M - 1}):
        solo = binding.bi_ctrl_lora_shrink_tc(xd[r_:r_ + 1].contiguous(), Ad)
        assert torch.equal(solo[0].view(torch.int32), t[r_].view(torch.int32))
    for _ in range(5):
        assert torch.equal(binding.bi_ctrl_lora_shrink_tc(xd, Ad).view(torch.int32), t.view(torch.int32))
