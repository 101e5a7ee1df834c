"""bi_decode_attn_noalloc: decode attention for callers that cannot allocate device memory.

Some callers hand a kernel only their input and output buffers and have no allocator
to offer (a plugin interface, a serving process whose memory pool owns the GPU's free
memory, a latency-critical loop that cannot afford cudaMalloc's synchronisation).  This
entry point keeps its scratch in a fixed array inside libbi.so.  Here it is called
directly through the C ABI, and its output is checked against bi_decode_attn's on
two calls in a row (the second call reuses whatever the first left in the array).  The
tolerance is the one the decode-attention tests use: relative Frobenius error <= 2e-3.
This file is collected last, so a run that stops at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import rel_frobenius
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
    return dev(q), dev(k), dev(v), dev(indptr), dev(kv_len), T


def _call_noalloc(fn, q, k, v, ip, ln, T, out):
    s = torch.cuda.current_stream().cuda_stream
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return fn(p(q), p(k), p(v), p(ip), p(ln), q.shape[0], T, 32, 8, D, 1.0 / D ** 0.5, 256, p(out),
              0, ctypes.c_void_p(s))


def test_matches_workspace_entry_point_on_two_calls_in_a_row():
    fn = _noalloc_fn()
    for kv_len, seed in (([300, 1, 2000, 4097], 21), ([513, 256, 7000], 22)):
        q, k, v, ip, ln, T = _case(kv_len, seed)
        out = torch.empty((q.shape[0], 32, D), dtype=torch.float32, device="cuda")
        assert _call_noalloc(fn, q, k, v, ip, ln, T, out) == 0
        ref = binding.bi_decode_attn(q, k, v, ip, ln, out_dtype=torch.float32)
        torch.cuda.synchronize()
        got, exp = out.cpu().numpy(), ref.cpu().numpy()
        for b in range(q.shape[0]):
            assert rel_frobenius(got[b], exp[b]) <= 2e-3
    assert binding.bi_get_device_error() == 0


def test_refuses_caches_beyond_the_scratch_limit():
    fn = _noalloc_fn()
    q, k, v, ip, ln, T = _case([300], 23)
    out = torch.empty((1, 32, D), dtype=torch.float32, device="cuda")
    too_many = (MAX_SCRATCH // (32 * (D + 2) * 4) + 1) * 256  # one slot more than fits
    assert binding.bi_decode_attn_workspace_size(too_many, 32) > MAX_SCRATCH
    assert _call_noalloc(fn, q, k, v, ip, ln, too_many, out) == 4  # BI_ERR_WORKSPACE, nothing launched
