"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the ops themselves: it draws seeded normals
and uniform integers with numpy, quantises them to the storage dtype
(bfloat16 bit patterns, round to nearest even) and lays them out.  The same
bits are handed to the CUDA library and to the CPU oracle.

Recipes (dims are the Llama-3-8B-shaped ones the workloads name):
  * RMSNorm, small:  x fp32 [M,256] ~ N(0,1), w fp32 [256] ~ N(1,0.1), eps 1e-6.
  * RMSNorm, 8B:     x bf16 [M,4096] ~ N(0,1), w bf16 [4096] ~ N(1,0.1).
  * GEMM:            A bf16 [M,K] ~ N(0,1), W bf16 [K,N] ~ N(0,0.02).
  * LoRA:            x bf16 [M,4096] ~ N(0,1); A [4096,r], B [r,4096] ~ N(0,0.02);
                     base output y bf16 [M,4096] ~ N(0,1).
  * Decode attention: q [B,32,128], k/v packed [T,8,128] bf16 ~ N(0,1); kv lengths
                     uniform integers in [512, 32768]; each sequence starts at a
                     multiple of the 256-token chunk.
Seeds: weights 0, activations 1, probes 2, kv lengths 3, positions 7, fillers 1000+trial.
"""
from __future__ import annotations

import numpy as np

SEED_WEIGHTS = 0
SEED_X = 1
SEED_PROBES = 2
SEED_KVLEN = 3
SEED_POSITIONS = 7
SEED_FILLER_BASE = 1000


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Quantise float32 samples to bfloat16 bit patterns (nearest, ties to even; inputs are finite)."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def normal(seed: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(size=shape, dtype=np.float64) * std + mean).astype(np.float32)


def normal_bf16(seed: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    return f32_to_bf16_bits(normal(seed, shape, mean, std))


def rows(seed: int, M: int, H: int, dtype: str, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """M rows of H values, float32 ('f32') or bf16 bits ('bf16')."""
    return normal(seed, (M, H), mean, std) if dtype == "f32" else normal_bf16(seed, (M, H), mean, std)


# ------------------------------------------------------------------ RMSNorm
def rmsnorm_case(M: int, H: int, dtype: str, seed_x: int = SEED_X, seed_w: int = SEED_WEIGHTS):
    x = rows(seed_x, M, H, dtype)
    w = normal(seed_w, (H,), 1.0, 0.1) if dtype == "f32" else normal_bf16(seed_w, (H,), 1.0, 0.1)
    return x, w


# ------------------------------------------------------------------ GEMM
def gemm_case(M: int, N: int, K: int, seed_a: int = SEED_X, seed_w: int = SEED_WEIGHTS):
    A = normal_bf16(seed_a, (M, K))
    W = normal_bf16(seed_w, (K, N), 0.0, 0.02)
    return A, W


def small_int_bf16(seed: int, shape, lo: int = -8, hi: int = 8) -> np.ndarray:
    """Small integers (exact in bf16) so that every partial sum is exact in fp32."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.integers(lo, hi + 1, size=shape).astype(np.float32))


# ------------------------------------------------------------------ LoRA
def lora_case(M: int, r: int, K: int = 4096, N: int = 4096, seed_x: int = SEED_X, seed_w: int = SEED_WEIGHTS):
    x = normal_bf16(seed_x, (M, K))
    A = normal_bf16(seed_w, (K, r), 0.0, 0.02)
    B = normal_bf16(seed_w + 1, (r, N), 0.0, 0.02)
    y = normal_bf16(seed_x + 100, (M, N))
    return x, A, B, y


# ------------------------------------------------------------------ decode attention
def kv_lengths(B: int, lo: int = 512, hi: int = 32768, seed: int = SEED_KVLEN) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=B).astype(np.int32)


def kv_layout(kv_len: np.ndarray, chunk: int = 256):
    """Packed KV layout: sequence b starts at a multiple of `chunk`; returns (kv_indptr[B+1], total_tokens)."""
    padded = ((kv_len.astype(np.int64) + chunk - 1) // chunk) * chunk
    indptr = np.zeros(len(kv_len) + 1, np.int64)
    indptr[1:] = np.cumsum(padded)
    assert indptr[-1] < 2**31, "packed KV exceeds int32 token offsets"
    return indptr.astype(np.int32), int(indptr[-1])


def attn_case(kv_len: np.ndarray, Hq: int = 32, Hkv: int = 8, D: int = 128, chunk: int = 256,
              seed: int = SEED_X):
    """q [B,Hq,D], k/v [T,Hkv,D] bf16 bits; padding tokens between sequences are zero."""
    B = len(kv_len)
    indptr, T = kv_layout(kv_len, chunk)
    q = normal_bf16(seed, (B, Hq, D))
    k = np.zeros((T, Hkv, D), np.uint16)
    v = np.zeros((T, Hkv, D), np.uint16)
    for b in range(B):
        L = int(kv_len[b])
        base = int(indptr[b])
        k[base:base + L] = normal_bf16(seed * 7919 + 2 * b + 1, (L, Hkv, D))
        v[base:base + L] = normal_bf16(seed * 7919 + 2 * b + 2, (L, Hkv, D))
    return q, k, v, indptr, T


# ------------------------------------------------------------------ invariance probes
def probe_positions(M: int, n_positions: int, seed: int) -> np.ndarray:
    """Distinct random row positions in [0, M) (all of them when M <= n_positions)."""
    if M <= n_positions:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(M, size=n_positions, replace=False))


M_SWEEP_POW2 = [1 << i for i in range(14)]  # 1 .. 8192
M_SWEEP_ODD = [3, 5, 7, 15, 17, 31, 33, 63, 65, 127, 129, 255, 257, 511, 513, 1023, 1025, 2047, 2049,
               4095, 4097, 8191]


def m_sweep(max_m: int = 8192):
    return sorted(m for m in set(M_SWEEP_POW2 + M_SWEEP_ODD) if m <= max_m)


# ------------------------------------------------------------------ decoder
# A Llama-shaped decoder: RMSNorm -> fused QKV projection -> RoPE -> attention -> output
# projection -> residual; RMSNorm -> fused gate/up projection -> SwiGLU -> down projection ->
# residual; a final RMSNorm and the vocabulary projection.  Matrices ~ N(0, 0.02) (random
# init: no trained weights are used); norm weights ~ N(1, 0.02); prompts are uniform token
# ids, prompt lengths uniform integers in [16, 2048].
SEED_PROMPT_LEN = 4
SEED_PROMPT_BASE = 5000


class DecoderShape:
    """Dimensions of the decoder (defaults: 4 layers of Llama-3-8B, vocabulary 32000)."""

    def __init__(self, hidden=4096, layers=4, q_heads=32, kv_heads=8, head_dim=128, ffn=14336, vocab=32000,
                 eps=1e-5, theta=500000.0):
        self.hidden, self.layers, self.q_heads, self.kv_heads = hidden, layers, q_heads, kv_heads
        self.head_dim, self.ffn, self.vocab, self.eps, self.theta = head_dim, ffn, vocab, eps, theta

    @property
    def qkv_cols(self) -> int:
        return (self.q_heads + 2 * self.kv_heads) * self.head_dim

    def matrices(self):
        """(name, rows, cols, mean, std) of every weight, in generation order."""
        H, F, V = self.hidden, self.ffn, self.vocab
        out = [("embed", V, H, 0.0, 0.02)]
        for l in range(self.layers):
            out += [(f"l{l}.attn_norm", 1, H, 1.0, 0.02), (f"l{l}.wqkv", H, self.qkv_cols, 0.0, 0.02),
                    (f"l{l}.wo", self.q_heads * self.head_dim, H, 0.0, 0.02), (f"l{l}.mlp_norm", 1, H, 1.0, 0.02),
                    (f"l{l}.wgu", H, 2 * F, 0.0, 0.02), (f"l{l}.wdown", F, H, 0.0, 0.02)]
        out += [("final_norm", 1, H, 1.0, 0.02), ("lm_head", H, V, 0.0, 0.02)]
        return out


LLAMA3_8B_4L = DecoderShape()
TINY_DECODER = DecoderShape(hidden=512, layers=2, q_heads=4, kv_heads=2, ffn=768, vocab=1000)


def decoder_weights_host(shape: DecoderShape, seed: int = SEED_WEIGHTS, matrix_std: float | None = None,
                         norm_std: float | None = None) -> dict:
    """Every weight as bf16 bits (numpy uint16), norm weights 1-D.  For small shapes (host numpy draws).
    matrix_std / norm_std override the spreads of the matrices / the norm weights."""
    out = {}
    for i, (name, r, c, mean, std) in enumerate(shape.matrices()):
        if mean == 0.0 and matrix_std is not None:
            std = matrix_std
        if mean != 0.0 and norm_std is not None:
            std = norm_std
        w = normal_bf16(seed * 1000 + i, (r, c), mean, std)
        out[name] = w[0] if r == 1 else w
    return out


def decoder_weights_device(shape: DecoderShape, seed: int = SEED_WEIGHTS, device="cuda") -> dict:
    """Every weight as a bf16 torch tensor drawn on the device (seeded torch generator): the fast
    route for full-size shapes, whose 1.1e9 draws would take minutes with numpy."""
    import torch

    g = torch.Generator(device=device).manual_seed(seed)
    out = {}
    for name, r, c, mean, std in shape.matrices():
        w = (torch.randn((r, c), generator=g, device=device, dtype=torch.float32) * std + mean).to(torch.bfloat16)
        out[name] = w[0].contiguous() if r == 1 else w
    return out


def prompt_lengths(n: int, lo: int = 16, hi: int = 2048, seed: int = SEED_PROMPT_LEN) -> np.ndarray:
    return np.random.default_rng(seed).integers(lo, hi + 1, size=n).astype(np.int32)


def prompt(index: int, length: int, vocab: int) -> np.ndarray:
    """Token ids of prompt number `index` (uniform in [0, vocab))."""
    return np.random.default_rng(SEED_PROMPT_BASE + index).integers(0, vocab, size=length).astype(np.int32)
