"""Helpers shared by the GPU tests: host <-> device transfer of raw bits and tolerance checks."""
from __future__ import annotations

import numpy as np
import torch


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy float32 / int32 / bf16 bits (uint16) -> CUDA tensor with the same bits."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy with the same bits (bf16 comes back as uint16)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 steps between two arrays of bf16 bits (+0 and -0 are 0 apart)."""
    def key(x):
        x = np.asarray(x, np.uint16).astype(np.int64)
        mag = x & 0x7FFF
        return np.where(x & 0x8000, -mag, mag)
    return np.abs(key(a) - key(b))


def rel_err_rowscaled(got: np.ndarray, ref: np.ndarray, floor_frac: float = 1e-3) -> float:
    """max |g - r| / max(|r|, floor_frac * rms(row of r)) over all elements."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    den = np.maximum(np.abs(ref), floor_frac * rms)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(got - ref) / den)) if got.size else 0.0


def rel_frobenius(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (n if n > 0 else 1.0))


def oracle_rows(fn, rows: np.ndarray, *args, block: int = 64) -> np.ndarray:
    """fn(rows[i:j], *args) over row blocks on all host cores, stacked in row order.

    The oracle's ctypes calls release the GIL, and every output row of its ops depends only on
    the same input row, so splitting the rows changes nothing in the result; it only lets the
    full-size parity cases finish in seconds."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    starts = list(range(0, rows.shape[0], block))
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        parts = list(ex.map(lambda i: fn(np.ascontiguousarray(rows[i:i + block]), *args), starts))
    return np.concatenate(parts, axis=0)
