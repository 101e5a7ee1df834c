"""Every op writes exactly its output and nothing else.

Each output is a window inside a larger buffer whose guard bytes (every row's tail, and
whole rows before and after) hold a fixed pattern.  After the call, the window must hold
the expected result and every guard byte must still hold the pattern.
"""
import numpy as np
import pytest
import torch

from gpu_util import dev
from invariant_deterministic_rmsnorm_b200 import binding, inputs

pytestmark = pytest.mark.gpu
GUARD_ROWS = 3
GUARD_COLS = 64
PATTERN = 0x5A


def _guarded(M, N, dtype):
    """A [M + 2g, N + pad] buffer filled with the pattern, and the [M, N] window inside it."""
    es = torch.empty((), dtype=dtype).element_size()
    pad = GUARD_COLS
    big = torch.full(((M + 2 * GUARD_ROWS) * (N + pad) * es,), PATTERN, dtype=torch.uint8, device="cuda")
    view = big.view(dtype).view(M + 2 * GUARD_ROWS, N + pad)
    return big, view, view[GUARD_ROWS:GUARD_ROWS + M, :N]


def _guards_intact(big, view, M, N):
    v = view.view(torch.uint8).view(view.shape[0], -1)
    es = v.shape[1] // view.shape[1]
    top = v[:GUARD_ROWS]
    bottom = v[GUARD_ROWS + M:]
    tails = v[GUARD_ROWS:GUARD_ROWS + M, N * es:]
    return all(bool((t == PATTERN).all()) for t in (top, bottom, tails))


def test_rmsnorm_writes_only_its_rows():
    M, H = 37, 4096
    x, w = inputs.rmsnorm_case(M, H, "bf16")
    big, view, y = _guarded(M, H, torch.bfloat16)
    binding.bi_rmsnorm(dev(x), dev(w), y=y)
    torch.cuda.synchronize()
    assert _guards_intact(big, view, M, H)
    ref = binding.bi_rmsnorm(dev(x), dev(w))
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def test_lora_expand_writes_only_its_window():
    M, r, N = 45, 16, 4096
    t = dev(inputs.normal(3, (M, r)))
    B = dev(inputs.normal_bf16(4, (r, N), 0, 0.02))
    y0 = dev(inputs.normal_bf16(5, (M, N)))
    big, view, y = _guarded(M, N, torch.bfloat16)
    y.copy_(y0)
    binding.bi_lora_expand(t, B, y)
    torch.cuda.synchronize()
    assert _guards_intact(big, view, M, N)
    ref = y0.clone()
    binding.bi_lora_expand(t, B, ref)
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def test_gemm_and_shrink_write_only_their_outputs():
    # contiguous outputs: guard rows before and after (the ABI takes C and t as dense [M, N])
    M, K, N = 130, 4096, 6144
    A = dev(inputs.normal_bf16(6, (M, K)))
    W = dev(inputs.normal_bf16(7, (K, N), 0, 0.02))
    big = torch.full(((M + 2 * GUARD_ROWS) * N * 2,), PATTERN, dtype=torch.uint8, device="cuda")
    C = big.view(torch.bfloat16).view(M + 2 * GUARD_ROWS, N)[GUARD_ROWS:GUARD_ROWS + M]
    binding.bi_gemm(A, W, C=C)
    torch.cuda.synchronize()
    u = big.view(M + 2 * GUARD_ROWS, N * 2)
    assert bool((u[:GUARD_ROWS] == PATTERN).all()) and bool((u[GUARD_ROWS + M:] == PATTERN).all())
    Al = dev(inputs.normal_bf16(8, (K, 16), 0, 0.02))
    bt = torch.full(((M + 2 * GUARD_ROWS) * 16 * 4,), PATTERN, dtype=torch.uint8, device="cuda")
    t = bt.view(torch.float32).view(M + 2 * GUARD_ROWS, 16)[GUARD_ROWS:GUARD_ROWS + M]
    binding.bi_lora_shrink(A, Al, t=t)
    torch.cuda.synchronize()
    ut = bt.view(M + 2 * GUARD_ROWS, 64)
    assert bool((ut[:GUARD_ROWS] == PATTERN).all()) and bool((ut[GUARD_ROWS + M:] == PATTERN).all())


def test_decode_attention_writes_only_its_rows():
    kv_len = np.array([300, 40, 1000], np.int32)
    q, k, v, ip, T = inputs.attn_case(kv_len, 32, 8, 128, 256, 9)
    Bq = len(kv_len)
    big = torch.full(((Bq + 2) * 32 * 128 * 2,), PATTERN, dtype=torch.uint8, device="cuda")
    out = big.view(torch.bfloat16).view(Bq + 2, 32, 128)[1:1 + Bq]
    binding.bi_decode_attn(dev(q), dev(k), dev(v), dev(ip), dev(kv_len), out=out)
    torch.cuda.synchronize()
    u = big.view(Bq + 2, -1)
    assert bool((u[0] == PATTERN).all()) and bool((u[-1] == PATTERN).all())
