"""bi_decode_attn_noalloc: decode attention for callers that cannot allocate device memory.

Some callers hand a kernel only their input and output buffers and have no allocator
to offer (a plugin interface, a serving process whose memory pool owns the GPU's free
memory, a latency-critical loop that cannot afford cudaMalloc's synchronisation).  This
entry point keeps its scratch in a fixed array inside libbi.so.  Here it is called
directly through the C ABI on two calls in a row (the second call runs over whatever the
first left in the array), in fp32 and bf16 output.  It runs the same two kernels as
bi_decode_attn with the same arithmetic, so its output must equal bi_decode_attn's bit for
bit; it is also held to the fp64 oracle at the decode-attention tolerances (fp32: relative
Frobenius error <= 2e-3 and the 1e-4 sanity bound; bf16: within one bf16 rounding).
This file is collected last, so a run that stops at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_util import bf16_to_f64, host, rel_frobenius
from invariant_deterministic_rmsnorm_b200 import binding, inputs

pytestmark = pytest.mark.gpu
D = 128
MAX_SCRATCH = 16 << 20


def _noalloc_fn():
    lib = binding.library()
    fn = lib.bi_decode_attn_noalloc
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    fn.argtypes = [P, P, P, P, P, I32, I64, I32, I32, I32, ctypes.c_float, I32, P, ctypes.c_int, P]
    fn.restype = ctypes.c_int
    return fn


def _case(kv_len, seed):
    kv_len = np.asarray(kv_len, np.int32)
    q, k, v, indptr, T = inputs.attn_case(kv_len, 32, 8, D, 256, seed)

    def dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(a).cuda()
    ref = oracle.decode_attn(q, k, v, indptr, kv_len, 8, 1.0 / np.sqrt(D))
    return dev(q), dev(k), dev(v), dev(indptr), dev(kv_len), T, ref


def _call_noalloc(fn, q, k, v, ip, ln, T, out):
    s = torch.cuda.current_stream().cuda_stream
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    code = 1 if out.dtype == torch.bfloat16 else 0
    return fn(p(q), p(k), p(v), p(ip), p(ln), q.shape[0], T, 32, 8, D, 1.0 / D ** 0.5, 256, p(out),
              code, ctypes.c_void_p(s))


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_matches_workspace_entry_point_on_two_calls_in_a_row(out_dtype):
    fn = _noalloc_fn()
    binding.bi_clear_device_error()
    # the second case is smaller than the first: its call runs over the first call's leftovers
    for kv_len, seed in (([300, 1, 2000, 4097], 21), ([513, 256, 7000], 22)):
        q, k, v, ip, ln, T, exact = _case(kv_len, seed)
        out = torch.full((q.shape[0], 32, D), float("nan"), dtype=out_dtype, device="cuda")
        assert _call_noalloc(fn, q, k, v, ip, ln, T, out) == 0
        ref = binding.bi_decode_attn(q, k, v, ip, ln, out_dtype=out_dtype)
        torch.cuda.synchronize()
        got, exp = host(out), host(ref)
        assert np.array_equal(got.view(np.uint16 if out_dtype == torch.bfloat16 else np.uint32),
                              exp.view(np.uint16 if out_dtype == torch.bfloat16 else np.uint32))
        if out_dtype == torch.bfloat16:  # within one bf16 rounding of the oracle, as the bf16 test asks
            g64 = bf16_to_f64(got)
            rms = np.sqrt((exact ** 2).mean(axis=-1, keepdims=True))
            assert np.all(np.abs(g64 - exact) <= 2.0 ** -8 * np.abs(exact) + 1e-4 * rms)
        else:
            for b in range(q.shape[0]):
                err = rel_frobenius(got[b], exact[b])
                assert err <= 2e-3 and err <= 1e-4, (b, err)
    assert binding.bi_get_device_error() == 0


def test_a_sequence_past_the_cache_is_a_layout_error():
    """kv_indptr[B] > total_tokens: that sequence's row is refused on the device (bit 0x100) and
    left unwritten; the sequences inside the cache still get their exact results."""
    fn = _noalloc_fn()
    q, k, v, ip, ln, T, _ = _case([300, 700], 24)
    good = binding.bi_decode_attn(q[:1].contiguous(), k, v, ip[:2].contiguous(), ln[:1].contiguous(),
                                  out_dtype=torch.float32)
    torch.cuda.synchronize()
    binding.bi_clear_device_error()
    out = torch.zeros((2, 32, D), dtype=torch.float32, device="cuda")
    # claim a cache of 512 tokens: the second sequence (tokens 512 .. 1211) lies past it
    assert _call_noalloc(fn, q, k, v, ip, ln, 512, out) == 0
    torch.cuda.synchronize()
    assert binding.bi_get_device_error() & 0x100
    assert torch.equal(out[0].view(torch.int32), good[0].view(torch.int32))
    assert torch.count_nonzero(out[1]) == 0
    binding.bi_clear_device_error()
    assert binding.bi_get_device_error() == 0


def test_refuses_caches_beyond_the_scratch_limit():
    fn = _noalloc_fn()
    q, k, v, ip, ln, T, _ = _case([300], 23)
    out = torch.empty((1, 32, D), dtype=torch.float32, device="cuda")
    too_many = (MAX_SCRATCH // (32 * (D + 2) * 4) + 1) * 256  # one slot more than fits
    assert binding.bi_decode_attn_workspace_size(too_many, 32) > MAX_SCRATCH
    assert _call_noalloc(fn, q, k, v, ip, ln, too_many, out) == 4  # BI_ERR_WORKSPACE, nothing launched
