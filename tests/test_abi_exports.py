"""libbi.so loads on a machine without a GPU and exports every entry point include/*.h declares.

Only host-side paths run here: status strings, the ABI version and argument
checks that return before any CUDA call (null pointers, negative sizes, bad
dtypes, misaligned addresses, empty batches).
"""
import ctypes
import glob
import os
import re

import pytest

from invariant_deterministic_rmsnorm_b200 import build as bi_build
from invariant_deterministic_rmsnorm_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names += re.findall(r"^\s*(?:const\s+char\s*\*|int|size_t|void)\s+(bi_\w+)\s*\(", text, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    bi_build.build()
    return binding.library()


def test_headers_declare_entry_points():
    names = _declared()
    for required in ("bi_rmsnorm", "bi_status_str", "bi_get_device_error"):
        assert required in names


@pytest.mark.parametrize("name", _declared())
def test_symbol_exported(lib, name):
    assert hasattr(lib, name), f"{name} declared in include/ but not exported by libbi.so"


def test_status_strings(lib):
    assert lib.bi_abi_version() == 1
    for code, name in binding.STATUS.items():
        assert lib.bi_status_str(code).decode() == name
    assert lib.bi_status_str(99).decode() == "BI_ERR_UNKNOWN"


def _rms(lib, x, w, y, M, H, ldx=None, ldy=None, eps=1e-6, io=0, wd=0):
    P = ctypes.c_void_p
    return lib.bi_rmsnorm(P(x), P(w), P(y), M, H, ldx if ldx is not None else H, ldy if ldy is not None else H,
                          eps, io, wd, None)


def test_rmsnorm_host_checks(lib):
    a = 1 << 20  # a 16-byte aligned fake address; never dereferenced on these paths
    assert _rms(lib, a, a, a, 0, 256) == 0                 # empty batch: no-op
    assert _rms(lib, None, a, a, 4, 256) == 1              # null x
    assert _rms(lib, a, a, a, -1, 256) == 1                # negative M
    assert _rms(lib, a, a, a, 4, 0) == 1                   # H = 0
    assert _rms(lib, a, a, a, 4, 256, io=7) == 1           # unknown dtype
    assert _rms(lib, a, a, a, 4, 256, eps=-1.0) == 1       # negative eps
    assert _rms(lib, a, a, a, 4, 256, ldx=100) == 1        # ldx < H
    assert _rms(lib, a + 4, a, a, 4, 256) == 3             # misaligned x
    assert _rms(lib, a, a, a, 4, 258) == 3                 # H not a multiple of 4 fp32
    assert _rms(lib, a, a, a, 4, 256, ldx=258) == 3        # row stride not 16-byte aligned
    assert _rms(lib, a, a, a, 4, 1 << 16) == 2             # H beyond the in-register plan
    assert _rms(lib, a, a, a, 4, 256, ldy=260) == 1        # in place with a different row stride


def test_model_ops_host_checks(lib):
    P = ctypes.c_void_p
    a = 1 << 20
    s = None
    # embed: empty, bad sizes, misaligned rows
    assert lib.bi_embed(P(a), P(a), P(a), 0, 4096, 32000, s) == 0
    assert lib.bi_embed(P(a), P(a), P(a), 4, 0, 32000, s) == 1
    assert lib.bi_embed(P(a), P(a), P(a), 4, 4100, 32000, s) == 3
    # rope: head_dim not a multiple of 4, theta <= 1, empty, misaligned table
    assert lib.bi_rope_table(P(a), 100, 126, 500000.0, s) == 1
    assert lib.bi_rope_table(P(a), 100, 128, 1.0, s) == 1
    assert lib.bi_rope_table(P(a), 0, 128, 500000.0, s) == 0
    assert lib.bi_rope_table(P(a + 8), 100, 128, 500000.0, s) == 3
    assert lib.bi_rope(P(a), 4, 4096, 32, 126, P(a), P(a), 100, s) == 1
    assert lib.bi_rope(P(a), 0, 4096, 32, 128, P(a), P(a), 100, s) == 0
    assert lib.bi_rope(P(a), 4, 4096, 32, 128, P(a), P(a + 8), 100, s) == 3
    assert lib.bi_rope(P(a), 4, 4095, 32, 128, P(a), P(a), 100, s) == 1
    # kv append: source stride shorter than a row, misaligned row
    assert lib.bi_kv_append(P(a), 512, P(a), P(a), 4, 1024, 100, s) == 1
    assert lib.bi_kv_append(P(a), 1028, P(a), P(a), 4, 1028, 100, s) == 3
    # add / swiglu: strides
    assert lib.bi_add(P(a), 8, P(a), 16, 4, 16, s) == 1
    assert lib.bi_swiglu(P(a), 16, P(a), 16, 4, 16, s) == 1     # ld_gu < 2N
    assert lib.bi_swiglu(P(a), 36, P(a), 18, 4, 18, s) == 3     # N not a multiple of 8
    assert lib.bi_argmax(P(a), 10, 4, 20, P(a), s) == 1         # ld < N
    # prefill attention: head_dim, grouping, empty batch, alignment, strides
    args = lambda **kw: [P(kw.get("q", a)), kw.get("ldq", 4096), 64, P(a), P(a), 1024, P(a), P(a),
                         kw.get("tiles", 1), P(a), P(a), kw.get("B", 1), kw.get("Hq", 32), kw.get("Hkv", 8),
                         kw.get("D", 128), 0.088, P(a), kw.get("ldo", 4096), s]
    assert lib.bi_prefill_attn(*args(D=64)) == 2
    assert lib.bi_prefill_attn(*args(Hkv=5)) == 1
    assert lib.bi_prefill_attn(*args(B=0)) == 0
    assert lib.bi_prefill_attn(*args(tiles=0)) == 0
    assert lib.bi_prefill_attn(*args(q=a + 2)) == 3
    assert lib.bi_prefill_attn(*args(ldq=4100)) == 3
    assert lib.bi_prefill_attn(*args(ldo=2048)) == 1


def test_gemm_split_plan_host(lib):
    """A K split meets on chip, so no GEMM call needs a workspace.  The plan's split counts are
    those bi_gemm_splits reports (a function of N and K only); the argument checks of
    bi_ctrl_gemm_split run before any launch."""
    for N, K in ((6144, 4096), (4096, 4096), (4096, 14336), (14336, 4096), (512, 256), (28672, 4096),
                 (32000, 4096)):
        assert 1 <= lib.bi_gemm_splits(N, K) <= 4, (N, K)
        assert lib.bi_gemm_workspace_size(4096, N, K) == 0
        assert lib.bi_gemm_counter_bytes(4096, N, K) == 0
    for N, K in ((28672, 4096), (32000, 4096), (512, 256)):
        assert lib.bi_gemm_splits(N, K) == 1, (N, K)  # single-CTA plan, or too small to split
    for M in (1, 8, 255, 256, 257, 4096):
        for S in (1, 2, 3, 4):
            assert lib.bi_ctrl_gemm_split_workspace_size(M, 4096, 14336, S) == 0
    a = 1 << 20
    P = ctypes.c_void_p
    assert lib.bi_ctrl_gemm_split(P(a), P(a), P(a), 8, 4096, 4096, 1, 5, None, 0, None) == 1
    assert lib.bi_ctrl_gemm_split(P(a), P(a), P(a), 8, 4096, 4096, 1, 0, None, 0, None) == 1
    assert lib.bi_ctrl_gemm_split(P(a), P(a), P(a), 8, 4096, 64, 1, 2, None, 0, None) == 1  # 1 K block
    assert lib.bi_ctrl_gemm_split(P(a), P(a), P(a), 8, 28672, 4096, 1, 2, None, 0, None) == 2
    assert lib.bi_ctrl_gemm_split(P(a), P(a), P(a), 0, 4096, 4096, 1, 2, None, 0, None) == 0  # empty batch


def test_fused_rmsnorm_shrink_host_checks(lib):
    """bi_rmsnorm_lora_shrink refuses, before any launch, the shapes it does not fuse (they
    take the two separate calls), bad arguments and misaligned rows; an empty batch is a no-op."""
    a = 1 << 20
    P = ctypes.c_void_p
    ok = dict(M=8, H=4096, ldx=4096, ldy=4096, eps=1e-6, r=16, split=8)

    def call(**kw):
        d = dict(ok, **kw)
        return lib.bi_rmsnorm_lora_shrink(P(a), P(a), P(a), P(a), P(a), d["M"], d["H"], d["ldx"], d["ldy"],
                                          d["eps"], d["r"], d["split"], None)
    assert call(M=0) == 0
    assert call(H=2048, ldx=2048, ldy=2048) == 2
    assert call(r=32) == 2 and call(r=64) == 2
    assert call(split=4) == 2
    assert call(ldx=4100) == 3  # a row stride that is not 16 bytes
    assert call(ldx=4000) == 1  # shorter than a row
    assert call(eps=-1.0) == 1 and call(M=-1) == 1
