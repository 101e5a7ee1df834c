"""fp64 CPU oracle for the batch-invariant forward ops -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and it never imports the product path.

This module is argument marshalling for ``bi_oracle.c`` (plain C, fp64, one
sequential sum per output in index order).  The C file names, per function, the
passage of the pages it follows.  Every call releases the GIL (ctypes), so a
caller may run disjoint row ranges on several threads.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bi_oracle.c")
_LIB = os.path.join(_HERE, "libbi_oracle.so")

F32 = 0
BF16 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile bi_oracle.c with gcc into oracle/libbi_oracle.so (strict IEEE: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def compile_variant(src_text: str, out_path: str) -> ctypes.CDLL:
    """Compile an edited copy of the oracle source (used by tests that plant a mistake) and load it."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", src,
                           "-o", out_path, "-lm"])
    lib = ctypes.CDLL(out_path)
    _declare(lib)
    return lib


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _declare(lib: ctypes.CDLL) -> None:
    P = ctypes.c_void_p
    I = ctypes.c_int64
    D = ctypes.c_double
    lib.bio_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.bio_bf16_to_f64.restype = D
    lib.bio_f64_to_bf16.argtypes = [D]
    lib.bio_f64_to_bf16.restype = ctypes.c_uint16
    lib.bio_round_bf16.argtypes = [P, P, I]
    lib.bio_round_f32.argtypes = [P, P, I]
    lib.bio_rmsnorm.argtypes = [P, ctypes.c_int, P, ctypes.c_int, P, I, I, I, I, D]
    lib.bio_gemm.argtypes = [P, P, P, I, I, I]
    lib.bio_lora_shrink.argtypes = [P, P, P, I, I, I]
    lib.bio_lora_shrink_split.argtypes = [P, P, P, I, I, I, I]
    lib.bio_lora_shrink_split.restype = ctypes.c_int
    lib.bio_lora_expand.argtypes = [P, P, P, ctypes.c_int, P, I, I, I, D]
    lib.bio_decode_attn.argtypes = [P, P, P, P, P, I, I, I, I, D, P, P]
    lib.bio_decode_attn.restype = ctypes.c_int
    lib.bio_decode_attn_split.argtypes = [P, P, P, P, P, I, I, I, I, D, I, P, P]
    lib.bio_decode_attn_split.restype = ctypes.c_int


def lib(handle: ctypes.CDLL | None = None) -> ctypes.CDLL:
    global _lib
    if handle is not None:
        return handle
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        _declare(_lib)
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bf16 bits (uint16), got {a.dtype}")


# ---------------------------------------------------------------- conversions
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact decode of bf16 bit patterns (uint16) to float64."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(v: np.ndarray, handle=None) -> np.ndarray:
    """Round fp64 values to bf16 bit patterns with the oracle's own nearest-even routine."""
    L = lib(handle)
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    L.bio_round_bf16(_p(v), _p(out), v.size)
    return out


def round_f32(v: np.ndarray, handle=None) -> np.ndarray:
    L = lib(handle)
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty(v.shape, np.float32)
    L.bio_round_f32(_p(v), _p(out), v.size)
    return out


# ---------------------------------------------------------------- the ops
def rmsnorm(x: np.ndarray, w: np.ndarray, eps: float, handle=None) -> np.ndarray:
    """x [M,H] float32 or bf16 bits, w [H] float32 or bf16 bits -> y [M,H] float64."""
    L = lib(handle)
    x = np.ascontiguousarray(x)
    w = np.ascontiguousarray(w)
    M, H = x.shape
    y = np.empty((M, H), np.float64)
    L.bio_rmsnorm(_p(x), _dtype_code(x), _p(w), _dtype_code(w), _p(y), M, H, H, H, float(eps))
    return y


def gemm(A: np.ndarray, W: np.ndarray, handle=None) -> np.ndarray:
    """A [M,K] bf16 bits, W [K,N] bf16 bits -> C [M,N] float64."""
    L = lib(handle)
    A = np.ascontiguousarray(A, np.uint16)
    W = np.ascontiguousarray(W, np.uint16)
    M, K = A.shape
    K2, N = W.shape
    assert K == K2
    C = np.empty((M, N), np.float64)
    L.bio_gemm(_p(A), _p(W), _p(C), M, N, K)
    return C


def lora_shrink(x: np.ndarray, A: np.ndarray, handle=None) -> np.ndarray:
    """x [M,K] bf16 bits, A [K,r] bf16 bits -> t [M,r] float64."""
    L = lib(handle)
    x = np.ascontiguousarray(x, np.uint16)
    A = np.ascontiguousarray(A, np.uint16)
    M, K = x.shape
    r = A.shape[1]
    t = np.empty((M, r), np.float64)
    L.bio_lora_shrink(_p(x), _p(A), _p(t), M, K, r)
    return t


def lora_shrink_split(x: np.ndarray, A: np.ndarray, split: int, handle=None) -> np.ndarray:
    L = lib(handle)
    x = np.ascontiguousarray(x, np.uint16)
    A = np.ascontiguousarray(A, np.uint16)
    M, K = x.shape
    r = A.shape[1]
    t = np.empty((M, r), np.float64)
    rc = L.bio_lora_shrink_split(_p(x), _p(A), _p(t), M, K, r, split)
    if rc != 0:
        raise ValueError("bio_lora_shrink_split: K must be a multiple of split")
    return t


def lora_expand(t: np.ndarray, B: np.ndarray, y_in: np.ndarray, scale: float, handle=None) -> np.ndarray:
    """t [M,r] float32, B [r,N] bf16 bits, y_in [M,N] float32 or bf16 bits -> y [M,N] float64."""
    L = lib(handle)
    t = np.ascontiguousarray(t, np.float32)
    B = np.ascontiguousarray(B, np.uint16)
    y_in = np.ascontiguousarray(y_in)
    M, r = t.shape
    N = B.shape[1]
    y = np.empty((M, N), np.float64)
    L.bio_lora_expand(_p(t), _p(B), _p(y_in), _dtype_code(y_in), _p(y), M, r, N, float(scale))
    return y


def decode_attn(q, k, v, kv_indptr, kv_len, Hkv: int, scale: float, handle=None) -> np.ndarray:
    """q [B,Hq,D] bf16 bits; k, v [T,Hkv,D] bf16 bits; kv_indptr [B+1] / kv_len [B] int32 -> out [B,Hq,D] float64."""
    L = lib(handle)
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    ip = np.ascontiguousarray(kv_indptr, np.int32)
    ln = np.ascontiguousarray(kv_len, np.int32)
    B, Hq, D = q.shape
    out = np.empty((B, Hq, D), np.float64)
    scratch = np.empty(max(1, int(ln.max()) if ln.size else 1), np.float64)
    rc = L.bio_decode_attn(_p(q), _p(k), _p(v), _p(ip), _p(ln), B, Hq, Hkv, D, float(scale), _p(out), _p(scratch))
    if rc != 0:
        raise ValueError(f"bio_decode_attn: bad arguments (code {rc})")
    return out


def decode_attn_split(q, k, v, kv_indptr, kv_len, Hkv: int, scale: float, chunk: int, handle=None) -> np.ndarray:
    L = lib(handle)
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    ip = np.ascontiguousarray(kv_indptr, np.int32)
    ln = np.ascontiguousarray(kv_len, np.int32)
    B, Hq, D = q.shape
    out = np.empty((B, Hq, D), np.float64)
    scratch = np.empty(D, np.float64)
    rc = L.bio_decode_attn_split(_p(q), _p(k), _p(v), _p(ip), _p(ln), B, Hq, Hkv, D, float(scale), chunk,
                                 _p(out), _p(scratch))
    if rc != 0:
        raise ValueError(f"bio_decode_attn_split: bad arguments (code {rc})")
    return out
