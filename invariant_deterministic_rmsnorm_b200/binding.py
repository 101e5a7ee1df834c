"""Thin ctypes binding over libbi.so, with the same names as the C ABI (include/bi.h, include/bi_model.h).

Argument marshalling only: every step of every op runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors; PyTorch provides device memory and
the stream (the current stream by default).  If libbi.so is missing, loading
raises an error.  There is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbi.so")

BI_F32 = 0
BI_BF16 = 1
STATUS = {0: "BI_OK", 1: "BI_ERR_INVALID_ARG", 2: "BI_ERR_UNSUPPORTED_SHAPE", 3: "BI_ERR_MISALIGNED",
          4: "BI_ERR_WORKSPACE", 5: "BI_ERR_CUDA", 6: "BI_ERR_TIMEOUT"}


class BIError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)} ({status})")
        self.status = status


_lib = None


def library() -> ctypes.CDLL:
    """Load libbi.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libbi.so not found at {LIB_PATH}; build it with "
                               "`python -m invariant_deterministic_rmsnorm_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        _declare(lib)
        _lib = lib
    return _lib


def _declare(lib: ctypes.CDLL) -> None:
    P, I64, I32, F, Z = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    C = ctypes.c_int
    sig = {
        "bi_status_str": ([C], ctypes.c_char_p),
        "bi_abi_version": ([], C),
        "bi_get_device_error": ([P, P], C),
        "bi_clear_device_error": ([P], C),
        "bi_rmsnorm": ([P, P, P, I64, I64, I64, I64, F, C, C, P], C),
        "bi_gemm_workspace_size": ([I64, I64, I64], Z),
        "bi_gemm_splits": ([I64, I64], C),
        "bi_gemm_counter_bytes": ([I64, I64, I64], Z),
        "bi_gemm": ([P, P, P, I64, I64, I64, C, P, Z, P], C),
        "bi_lora_shrink_workspace_size": ([I64, I64, I32, I32], Z),
        "bi_lora_shrink": ([P, P, P, I64, I64, I32, I32, P, Z, P], C),
        "bi_lora_expand": ([P, P, P, I64, I32, I64, I64, F, C, P], C),
        "bi_ctrl_lora_shrink_atomic": ([P, P, P, I64, I64, I32, I32, P], C),
        "bi_ctrl_lora_shrink_tc": ([P, P, P, I64, I64, I32, I32, P], C),
        "bi_decode_attn_workspace_size": ([I64, I32, I32, I32], Z),
        "bi_decode_attn": ([P, P, P, P, P, I32, I64, I32, I32, I32, F, I32, P, C, P, Z, P], C),
        "bi_ctrl_rmsnorm_split": ([P, P, P, I64, I64, I64, I64, F, C, C, P], C),
        "bi_ctrl_gemm_splitk_workspace_size": ([I64, I64, I64], Z),
        "bi_ctrl_gemm_splitk": ([P, P, P, I64, I64, I64, C, P, Z, P], C),
        "bi_ctrl_gemm_split_workspace_size": ([I64, I64, I64, I32], Z),
        "bi_ctrl_gemm_split": ([P, P, P, I64, I64, I64, C, I32, P, Z, P], C),
        "bi_rmsnorm_lora_shrink": ([P, P, P, P, P, I64, I64, I64, I64, F, I32, I32, P], C),
        "bi_ctrl_decode_attn_adaptive_workspace_size": ([I64, I32], Z),
        "bi_ctrl_decode_attn_adaptive": ([P, P, P, P, P, I32, I64, I32, I32, F, P, C, P, Z, P], C),
        "bi_ctrl_wait_timeout_probe": ([ctypes.c_uint64, P], C),
        "bi_ctrl_set_pdl": ([C], C),
        # include/bi_model.h
        "bi_embed": ([P, P, P, I64, I64, I64, P], C),
        "bi_rope_table": ([P, I64, I32, ctypes.c_double, P], C),
        "bi_rope": ([P, I64, I64, I32, I32, P, P, I64, P], C),
        "bi_kv_append": ([P, I64, P, P, I64, I64, I64, P], C),
        "bi_add": ([P, I64, P, I64, I64, I64, P], C),
        "bi_swiglu": ([P, I64, P, I64, I64, I64, P], C),
        "bi_argmax": ([P, I64, I64, I64, P, P], C),
        "bi_advance": ([P, I64, I32, P], C),
        "bi_prefill_attn": ([P, I64, I64, P, P, I64, P, P, I32, P, P, I32, I32, I32, I32, F, P, I64, P], C),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise BIError(fn, status)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BI_F32
    if t.dtype == torch.bfloat16:
        return BI_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _rows(t: torch.Tensor, name: str) -> None:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit stride along the last dimension")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


# ------------------------------------------------------------------ ops
def bi_rmsnorm(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None, eps: float = 1e-6,
               stream=None) -> torch.Tensor:
    """y = x / sqrt(mean(x^2) + eps) * w, row by row.  x, y [M, H] (fp32 or bf16); w [H]."""
    _rows(x, "x")
    if y is None:
        y = torch.empty_like(x, memory_format=torch.contiguous_format)
    _rows(y, "y")
    if w.dim() != 1 or not w.is_contiguous() or not w.is_cuda:
        raise ValueError("w must be a contiguous 1-D CUDA tensor")
    if y.dtype != x.dtype or tuple(y.shape) != tuple(x.shape):
        raise ValueError("y must match x in shape and dtype")
    M, H = x.shape
    st = library().bi_rmsnorm(_ptr(x), _ptr(w), _ptr(y), M, H, max(x.stride(0), H), max(y.stride(0), H),
                              float(eps), _dtype_code(x), _dtype_code(w), _stream(stream))
    _check("bi_rmsnorm", st)
    return y


def gemm_splits(N: int, K: int) -> int:
    """The K split count of bi_gemm's plan for a [K, N] weight on the current device."""
    return int(library().bi_gemm_splits(N, K))


def bi_gemm(A: torch.Tensor, W: torch.Tensor, C: torch.Tensor | None = None, out_dtype=torch.float32,
            stream=None) -> torch.Tensor:
    """C = A @ W with A [M, K] bf16, W [K, N] bf16 (both row-major contiguous); C fp32 or bf16 [M, N].
    The library needs no workspace for any plan (bi_gemm_workspace_size is 0)."""
    for t, n in ((A, "A"), (W, "W")):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 2 or not t.is_cuda:
            raise ValueError(f"{n} must be a contiguous 2-D bf16 CUDA tensor")
    M, K = A.shape
    K2, N = W.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    if C is None:
        C = torch.empty((M, N), dtype=out_dtype, device=A.device)
    if tuple(C.shape) != (M, N) or not C.is_contiguous():
        raise ValueError("C must be a contiguous [M, N] tensor")
    st = library().bi_gemm(_ptr(A), _ptr(W), _ptr(C), M, N, K, _dtype_code(C), ctypes.c_void_p(0), 0,
                           _stream(stream))
    _check("bi_gemm", st)
    return C


def _bf16_2d(t: torch.Tensor, name: str) -> None:
    if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 2 or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous 2-D bf16 CUDA tensor")


def bi_lora_shrink(x: torch.Tensor, A: torch.Tensor, t: torch.Tensor | None = None, split_k: int = 8,
                   stream=None) -> torch.Tensor:
    """t = x @ A (fp32 [M, r]), K cut into split_k slices whose partials are added in slice order."""
    _bf16_2d(x, "x")
    _bf16_2d(A, "A")
    M, K = x.shape
    K2, r = A.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    if t is None:
        t = torch.empty((M, r), dtype=torch.float32, device=x.device)
    if t.dtype != torch.float32 or tuple(t.shape) != (M, r) or not t.is_contiguous():
        raise ValueError("t must be a contiguous fp32 [M, r] tensor")
    st = library().bi_lora_shrink(_ptr(x), _ptr(A), _ptr(t), M, K, r, split_k, ctypes.c_void_p(0), 0,
                                  _stream(stream))
    _check("bi_lora_shrink", st)
    return t


def bi_rmsnorm_lora_shrink(x: torch.Tensor, w: torch.Tensor, A: torch.Tensor, y: torch.Tensor | None = None,
                           t: torch.Tensor | None = None, eps: float = 1e-6, split_k: int = 8,
                           stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """y = RMSNorm(x) * w and t = y @ A in one pass; bitwise bi_rmsnorm then bi_lora_shrink.
    x, y bf16 [M, 4096] (row strides may exceed 4096), w bf16 [4096], A bf16 [4096, r], r 8 or 16."""
    _rows(x, "x")
    _bf16_2d(A, "A")
    if y is None:
        y = torch.empty_like(x, memory_format=torch.contiguous_format)
    _rows(y, "y")
    if x.dtype != torch.bfloat16 or y.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise ValueError("x, y and w must be bf16")
    if w.dim() != 1 or not w.is_contiguous() or not w.is_cuda:
        raise ValueError("w must be a contiguous 1-D CUDA tensor")
    M, H = x.shape
    H2, r = A.shape
    if H != H2 or tuple(y.shape) != (M, H):
        raise ValueError("shape mismatch")
    if t is None:
        t = torch.empty((M, r), dtype=torch.float32, device=x.device)
    if t.dtype != torch.float32 or tuple(t.shape) != (M, r) or not t.is_contiguous():
        raise ValueError("t must be a contiguous fp32 [M, r] tensor")
    st = library().bi_rmsnorm_lora_shrink(_ptr(x), _ptr(w), _ptr(y), _ptr(A), _ptr(t), M, H, max(x.stride(0), H),
                                          max(y.stride(0), H), float(eps), r, split_k, _stream(stream))
    _check("bi_rmsnorm_lora_shrink", st)
    return y, t


def bi_lora_expand(t: torch.Tensor, B: torch.Tensor, y: torch.Tensor, scale: float = 1.0,
                   stream=None) -> torch.Tensor:
    """y += scale * bf16(t) @ B in place; t fp32 [M, r], B bf16 [r, N], y [M, N] (row stride may exceed N)."""
    if t.dtype != torch.float32 or not t.is_contiguous() or t.dim() != 2 or not t.is_cuda:
        raise ValueError("t must be a contiguous fp32 2-D CUDA tensor")
    _bf16_2d(B, "B")
    _rows(y, "y")
    M, r = t.shape
    r2, N = B.shape
    if r != r2 or tuple(y.shape) != (M, N):
        raise ValueError("shape mismatch")
    st = library().bi_lora_expand(_ptr(t), _ptr(B), _ptr(y), M, r, N, max(y.stride(0), N), float(scale),
                                  _dtype_code(y), _stream(stream))
    _check("bi_lora_expand", st)
    return y


def bi_ctrl_lora_shrink_atomic(x: torch.Tensor, A: torch.Tensor, t: torch.Tensor | None = None, split_k: int = 8,
                               stream=None) -> torch.Tensor:
    """Comparator: the same shrink with the partials combined by fp32 atomics (nondeterministic order)."""
    _bf16_2d(x, "x")
    _bf16_2d(A, "A")
    M, K = x.shape
    r = A.shape[1]
    if t is None:
        t = torch.empty((M, r), dtype=torch.float32, device=x.device)
    st = library().bi_ctrl_lora_shrink_atomic(_ptr(x), _ptr(A), _ptr(t), M, K, r, split_k, _stream(stream))
    _check("bi_ctrl_lora_shrink_atomic", st)
    return t


def bi_ctrl_lora_shrink_tc(x: torch.Tensor, A: torch.Tensor, t: torch.Tensor | None = None, split_k: int = 8,
                           stream=None) -> torch.Tensor:
    """The shrink on tcgen05 at r = 16, 32 or 64 (bi_lora_shrink's kernel at r = 64; the study
    behind keeping mma.sync at r = 16 and 32)."""
    _bf16_2d(x, "x")
    _bf16_2d(A, "A")
    M, K = x.shape
    r = A.shape[1]
    if t is None:
        t = torch.empty((M, r), dtype=torch.float32, device=x.device)
    st = library().bi_ctrl_lora_shrink_tc(_ptr(x), _ptr(A), _ptr(t), M, K, r, split_k, _stream(stream))
    _check("bi_ctrl_lora_shrink_tc", st)
    return t


def bi_decode_attn_workspace_size(total_tokens: int, Hq: int, head_dim: int = 128, chunk: int = 256) -> int:
    return int(library().bi_decode_attn_workspace_size(total_tokens, Hq, head_dim, chunk))


def bi_decode_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kv_indptr: torch.Tensor,
                   kv_len: torch.Tensor, out: torch.Tensor | None = None, scale: float | None = None,
                   chunk: int = 256, out_dtype=torch.bfloat16, workspace: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """Decode attention: q [B, Hq, D] against the packed cache k, v [T, Hkv, D] (bf16).

    kv_indptr int32 [B + 1] (chunk-aligned sequence starts), kv_len int32 [B].  A workspace of
    bi_decode_attn_workspace_size(T, Hq) bytes is allocated here when none is passed."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3 or not t.is_cuda:
            raise ValueError(f"{n} must be a contiguous 3-D bf16 CUDA tensor")
    for t, n in ((kv_indptr, "kv_indptr"), (kv_len, "kv_len")):
        if t.dtype != torch.int32 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{n} must be a contiguous int32 CUDA tensor")
    B, Hq, D = q.shape
    T, Hkv, D2 = k.shape
    if tuple(v.shape) != tuple(k.shape) or D2 != D or kv_indptr.numel() != B + 1 or kv_len.numel() != B:
        raise ValueError("shape mismatch")
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty((B, Hq, D), dtype=out_dtype, device=q.device)
    lib = library()
    need = lib.bi_decode_attn_workspace_size(T, Hq, D, chunk)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib.bi_decode_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_indptr), _ptr(kv_len), B, T, Hq, Hkv, D,
                            float(scale), chunk, _ptr(out), _dtype_code(out), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check("bi_decode_attn", st)
    return out


# ------------------------------------------------------------------ decoder ops (include/bi_model.h)
def _i32(t: torch.Tensor, name: str) -> None:
    if t.dtype != torch.int32 or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")


def _bf16_rows(t: torch.Tensor, name: str) -> None:
    _rows(t, name)
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bf16")


def bi_embed(tokens: torch.Tensor, table: torch.Tensor, out: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    """out[t] = table[tokens[t]] (bf16 rows)."""
    _i32(tokens, "tokens")
    _bf16_2d(table, "table")
    vocab, H = table.shape
    T = tokens.numel()
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=table.device)
    if not out.is_contiguous() or tuple(out.shape) != (T, H):
        raise ValueError("out must be a contiguous [T, H] tensor")
    _check("bi_embed", library().bi_embed(_ptr(tokens), _ptr(table), _ptr(out), T, H, vocab, _stream(stream)))
    return out


def bi_rope_table(positions: int, head_dim: int = 128, theta: float = 500000.0, device="cuda",
                  stream=None) -> torch.Tensor:
    """The (cos, sin) table bi_rope reads: fp32 [positions, head_dim / 2, 2]."""
    table = torch.empty((positions, head_dim // 2, 2), dtype=torch.float32, device=device)
    _check("bi_rope_table", library().bi_rope_table(_ptr(table), positions, head_dim, float(theta), _stream(stream)))
    return table


def bi_rope(x: torch.Tensor, pos: torch.Tensor, heads: int, table: torch.Tensor, head_dim: int = 128,
            stream=None) -> torch.Tensor:
    """Rotary embedding in place on the first heads*head_dim columns of each row of x (bf16)."""
    _bf16_rows(x, "x")
    _i32(pos, "pos")
    T = x.shape[0]
    if pos.numel() != T or x.shape[1] < heads * head_dim:
        raise ValueError("shape mismatch")
    if table.dtype != torch.float32 or not table.is_contiguous() or table.dim() != 3 or table.shape[1] * 2 != head_dim:
        raise ValueError("table must be a contiguous fp32 [positions, head_dim / 2, 2] tensor from bi_rope_table")
    _check("bi_rope", library().bi_rope(_ptr(x), T, x.stride(0), heads, head_dim, _ptr(pos), _ptr(table),
                                        table.shape[0], _stream(stream)))
    return x


def bi_kv_append(src: torch.Tensor, dst_row: torch.Tensor, dst: torch.Tensor, stream=None) -> torch.Tensor:
    """dst[dst_row[t], :] = src[t, :dst.shape[1]] (bf16; dst is a contiguous [rows, E] cache view)."""
    _bf16_rows(src, "src")
    _i32(dst_row, "dst_row")
    if dst.dtype != torch.bfloat16 or not dst.is_contiguous():
        raise ValueError("dst must be a contiguous bf16 tensor")
    d2 = dst.view(dst.shape[0], -1)
    T, E = src.shape[0], d2.shape[1]
    if dst_row.numel() != T or src.shape[1] < E:
        raise ValueError("shape mismatch")
    _check("bi_kv_append", library().bi_kv_append(_ptr(src), src.stride(0), _ptr(dst_row), _ptr(dst), T, E,
                                                  d2.shape[0], _stream(stream)))
    return dst


def bi_add(h: torch.Tensor, d: torch.Tensor, stream=None) -> torch.Tensor:
    """h += d in place (bf16 rows, one rounding per element)."""
    _bf16_rows(h, "h")
    _bf16_rows(d, "d")
    if h.shape != d.shape:
        raise ValueError("shape mismatch")
    T, N = h.shape
    _check("bi_add", library().bi_add(_ptr(h), h.stride(0), _ptr(d), d.stride(0), T, N, _stream(stream)))
    return h


def bi_swiglu(gu: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out = silu(gu[:, :N]) * gu[:, N:] with N = gu.shape[1] / 2 (bf16)."""
    _bf16_rows(gu, "gu")
    T, N2 = gu.shape
    if N2 % 2:
        raise ValueError("gu must have an even number of columns")
    N = N2 // 2
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=gu.device)
    _bf16_rows(out, "out")
    _check("bi_swiglu", library().bi_swiglu(_ptr(gu), gu.stride(0), _ptr(out), out.stride(0), T, N,
                                            _stream(stream)))
    return out


def bi_argmax(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Row-wise argmax of fp32 x (smallest index on ties) -> int32 [T]."""
    _rows(x, "x")
    if x.dtype != torch.float32:
        raise ValueError("x must be fp32")
    T, N = x.shape
    if out is None:
        out = torch.empty((T,), dtype=torch.int32, device=x.device)
    _i32(out, "out")
    _check("bi_argmax", library().bi_argmax(_ptr(x), x.stride(0), T, N, _ptr(out), _stream(stream)))
    return out


def bi_advance(v: torch.Tensor, step: int = 1, stream=None) -> torch.Tensor:
    """v += step, in place (int32, on the device)."""
    _i32(v, "v")
    _check("bi_advance", library().bi_advance(_ptr(v), v.numel(), int(step), _stream(stream)))
    return v


PREFILL_TILE_ROWS = 128


def prefill_tiles(q_lens) -> list:
    """q_tile_indptr for query lengths q_lens: prefix sums of ceil(len / 128)."""
    out = [0]
    for n in q_lens:
        out.append(out[-1] + (int(n) + PREFILL_TILE_ROWS - 1) // PREFILL_TILE_ROWS)
    return out


def bi_prefill_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, q_indptr: torch.Tensor,
                    q_tile_indptr: torch.Tensor, n_tiles: int, kv_indptr: torch.Tensor, q_pos0: torch.Tensor,
                    Hq: int, out: torch.Tensor | None = None, scale: float | None = None,
                    stream=None) -> torch.Tensor:
    """Causal prefill attention.  q: bf16 rows [q_rows, >= Hq*128] (any row stride); k_cache, v_cache:
    bf16 [T, Hkv, 128] packed; int32 index arrays as include/bi_model.h describes; out: bf16
    [q_rows, >= Hq*128] (allocated when None)."""
    _bf16_rows(q, "q")
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{n} must be a contiguous 3-D bf16 tensor")
    for t, n in ((q_indptr, "q_indptr"), (q_tile_indptr, "q_tile_indptr"), (kv_indptr, "kv_indptr"),
                 (q_pos0, "q_pos0")):
        _i32(t, n)
    B = q_pos0.numel()
    if q_indptr.numel() != B + 1 or q_tile_indptr.numel() != B + 1 or kv_indptr.numel() < B:
        raise ValueError("index arrays do not match the number of sequences")
    T, Hkv, D = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache and v_cache differ in shape")
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty((q.shape[0], Hq * D), dtype=torch.bfloat16, device=q.device)
    _bf16_rows(out, "out")
    st = library().bi_prefill_attn(_ptr(q), q.stride(0), q.shape[0], _ptr(k_cache), _ptr(v_cache), T,
                                   _ptr(q_indptr), _ptr(q_tile_indptr), int(n_tiles), _ptr(kv_indptr),
                                   _ptr(q_pos0), B, Hq, Hkv, D, float(scale), _ptr(out), out.stride(0),
                                   _stream(stream))
    _check("bi_prefill_attn", st)
    return out


# ------------------------------------------------------------------ comparators (not batch-invariant)
def bi_ctrl_rmsnorm_split(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None, eps: float = 1e-6,
                          stream=None) -> torch.Tensor:
    """Comparator: RMSNorm with the row reduction split across a cluster, split count chosen from M."""
    _rows(x, "x")
    if y is None:
        y = torch.empty_like(x, memory_format=torch.contiguous_format)
    M, H = x.shape
    st = library().bi_ctrl_rmsnorm_split(_ptr(x), _ptr(w), _ptr(y), M, H, max(x.stride(0), H),
                                         max(y.stride(0), H), float(eps), _dtype_code(x), _dtype_code(w),
                                         _stream(stream))
    _check("bi_ctrl_rmsnorm_split", st)
    return y


def bi_ctrl_gemm_splitk(A: torch.Tensor, W: torch.Tensor, C: torch.Tensor | None = None, out_dtype=torch.float32,
                        stream=None) -> torch.Tensor:
    """Comparator: GEMM with a split-K chosen from M (fp32 partials, ordered sum)."""
    _bf16_2d(A, "A")
    _bf16_2d(W, "W")
    M, K = A.shape
    N = W.shape[1]
    if C is None:
        C = torch.empty((M, N), dtype=out_dtype, device=A.device)
    lib = library()
    need = lib.bi_ctrl_gemm_splitk_workspace_size(M, N, K)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=A.device)
    st = lib.bi_ctrl_gemm_splitk(_ptr(A), _ptr(W), _ptr(C), M, N, K, _dtype_code(C), _ptr(ws), ws.numel(),
                                 _stream(stream))
    _check("bi_ctrl_gemm_splitk", st)
    return C


def bi_ctrl_gemm_split(A: torch.Tensor, W: torch.Tensor, splits: int, C: torch.Tensor | None = None,
                       out_dtype=torch.float32, stream=None) -> torch.Tensor:
    """bi_gemm with the K split count given (the plan study): S > 1 runs the cluster-split kernel,
    whose partials meet on chip."""
    _bf16_2d(A, "A")
    _bf16_2d(W, "W")
    M, K = A.shape
    N = W.shape[1]
    if C is None:
        C = torch.empty((M, N), dtype=out_dtype, device=A.device)
    st = library().bi_ctrl_gemm_split(_ptr(A), _ptr(W), _ptr(C), M, N, K, _dtype_code(C), int(splits),
                                      ctypes.c_void_p(0), 0, _stream(stream))
    _check("bi_ctrl_gemm_split", st)
    return C


def bi_ctrl_decode_attn_adaptive(q, k, v, kv_indptr, kv_len, out=None, scale=None, out_dtype=torch.bfloat16,
                                 workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Comparator: decode attention with 128-token chunks for batches under 16, 256 otherwise."""
    B, Hq, D = q.shape
    T, Hkv, _ = k.shape
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty((B, Hq, D), dtype=out_dtype, device=q.device)
    lib = library()
    need = lib.bi_ctrl_decode_attn_adaptive_workspace_size(T, Hq)
    ws = workspace
    if ws is None or ws.numel() * ws.element_size() < need:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib.bi_ctrl_decode_attn_adaptive(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_indptr), _ptr(kv_len), B, T, Hq, Hkv,
                                          float(scale), _ptr(out), _dtype_code(out), _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(stream))
    _check("bi_ctrl_decode_attn_adaptive", st)
    return out


def bi_ctrl_wait_timeout_probe(limit_ns: int = 1_000_000, stream=None) -> None:
    """Launch the one-CTA probe whose bounded wait must run out after limit_ns (sets bit 0x2)."""
    _check("bi_ctrl_wait_timeout_probe", library().bi_ctrl_wait_timeout_probe(int(limit_ns), _stream(stream)))


def bi_get_device_error(stream=None) -> int:
    code = ctypes.c_uint32(0)
    st = library().bi_get_device_error(ctypes.byref(code), _stream(stream))
    if st not in (0, 6):
        raise BIError("bi_get_device_error", st)
    return int(code.value)


def bi_clear_device_error(stream=None) -> None:
    _check("bi_clear_device_error", library().bi_clear_device_error(_stream(stream)))
