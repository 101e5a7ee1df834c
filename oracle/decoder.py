"""fp64 CPU oracle of the decoder ops and of a whole decoder -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg may
import this module.  It shares no code with the CUDA path.  It builds on the fp64 primitives
of ``bi_oracle.c``: RMSNorm, matmul, bf16 rounding, and the plain unchunked softmax attention
of one query over a key range.  The rest is written out here in numpy, in float64.

What the pages fix, and what is read into them:
  * "Defeating Nondeterminism in LLM Inference" (Spanish summary), section "La verdadera causa
    clave".  Every op must give a token row the same bits at any batch size.  This oracle
    processes row by row, so it is batch-invariant by construction.  A pin checks that.
  * Same page, section "Attention".  Each query attends to its own sequence's keys in one
    consistent layout, and cached keys and new keys are alike.  Here causal attention is,
    for query row i at position p, the plain softmax over the keys at positions 0..p.
  * The pages give no model.  The decoder is read as Llama-3 shaped:
      - pre-norm RMSNorm, eps inside the root;
      - a fused QKV projection;
      - RoPE with rotate-half pairing, theta 500000;
      - grouped-query attention, q head h using kv head h // (Hq / Hkv);
      - an output projection and a residual add;
      - RMSNorm, a fused gate/up projection, SwiGLU (silu(gate) * up), a down projection
        and a residual add;
      - a final RMSNorm and the vocabulary projection.
  * Declared roundings.  Every tensor the GPU path stores in bf16 is rounded to bf16 here at
    the same point, with the oracle's own nearest-even routine: the norm outputs, the
    projections, q and k after RoPE, the attention output, both residual sums and the SwiGLU
    output.  Logits stay fp64.  The GPU's are fp32.
"""
from __future__ import annotations

import numpy as np

from . import bf16_bits_to_f64, decode_attn, gemm, rmsnorm, round_bf16

__all__ = ["embed", "rope", "add", "swiglu", "argmax", "causal_attn", "OracleDecoder"]


def embed(tokens: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Rows of the embedding table (bf16 bits) picked by token id."""
    tokens = np.asarray(tokens, np.int64)
    if tokens.size and (tokens.min() < 0 or tokens.max() >= table.shape[0]):
        raise ValueError("token id out of range")
    return table[tokens]


def rope(x_bits: np.ndarray, pos: np.ndarray, heads: int, head_dim: int, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half pairing, in float64.

    Pair i < head_dim/2 of a head holds dims (i, i + head_dim/2).  It is turned by the angle
    pos * theta^(-2i/head_dim).  x_bits [T, >= heads*head_dim] bf16 bits; returns
    float64 [T, heads*head_dim].
    """
    T = x_bits.shape[0]
    half = head_dim // 2
    x = bf16_bits_to_f64(x_bits[:, :heads * head_dim]).reshape(T, heads, head_dim)
    freq = np.power(float(theta), -2.0 * np.arange(half, dtype=np.float64) / head_dim)
    ang = np.asarray(pos, np.float64)[:, None] * freq[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    out = np.empty_like(x)
    out[..., :half] = a * c - b * s
    out[..., half:] = b * c + a * s
    return out.reshape(T, heads * head_dim)


def add(h_bits: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    """The residual sum h + d of two bf16 tensors, float64."""
    return bf16_bits_to_f64(h_bits) + bf16_bits_to_f64(d_bits)


def swiglu(gu_bits: np.ndarray) -> np.ndarray:
    """silu(g) * u for gu = [g | u] (bf16 bits [T, 2N]) -> float64 [T, N]; silu(g) = g / (1 + e^-g)."""
    n = gu_bits.shape[1] // 2
    g = bf16_bits_to_f64(gu_bits[:, :n])
    u = bf16_bits_to_f64(gu_bits[:, n:2 * n])
    return g / (1.0 + np.exp(-g)) * u


def argmax(x: np.ndarray) -> np.ndarray:
    """Index of the largest value of each row; the smallest index among equals; NaN never wins."""
    x = np.where(np.isnan(x), -np.inf, np.asarray(x, np.float64))
    return np.argmax(x, axis=1).astype(np.int32)


def causal_attn(q_bits, k_cache, v_cache, base, length, q_heads: int, kv_heads: int, scale: float) -> np.ndarray:
    """Attention of each query row over its own key range.

    q_bits [T, >= Hq*D] bf16 bits.  k_cache, v_cache [rows, Hkv, D] bf16 bits.  Row t attends
    to cache rows base[t] .. base[t] + length[t] - 1 with the plain softmax.  Returns
    float64 [T, Hq*D].
    """
    T = q_bits.shape[0]
    D = k_cache.shape[2]
    q = np.ascontiguousarray(q_bits[:, :q_heads * D]).reshape(T, q_heads, D)
    ip = np.append(np.asarray(base, np.int32), np.int32(0))
    out = decode_attn(q, k_cache, v_cache, ip, np.asarray(length, np.int32), kv_heads, scale)
    return out.reshape(T, q_heads * D)


class OracleDecoder:
    """The decoder in float64 with the declared bf16 roundings, over a slotted KV cache.

    Sequence slot s owns cache rows s*cap .. s*cap + cap - 1.  Position p is row s*cap + p.
    ``forward(slots, tokens)`` appends each listed sequence's new tokens at its next
    positions.  It returns the logits of each sequence's last new token, float64
    [len(slots), vocab].
    """

    def __init__(self, shape, weights: dict, max_seqs: int, cap: int):
        self.s, self.w, self.cap = shape, weights, cap
        rows = max_seqs * cap
        self.k = [np.zeros((rows, shape.kv_heads, shape.head_dim), np.uint16) for _ in range(shape.layers)]
        self.v = [np.zeros((rows, shape.kv_heads, shape.head_dim), np.uint16) for _ in range(shape.layers)]
        self.length = np.zeros(max_seqs, np.int64)

    def forward(self, slots, tokens) -> np.ndarray:
        s, w = self.s, self.w
        Hq, Hkv, D = s.q_heads, s.kv_heads, s.head_dim
        toks = np.concatenate([np.asarray(t, np.int32) for t in tokens])
        pos = np.concatenate([self.length[sl] + np.arange(len(t)) for sl, t in zip(slots, tokens)])
        row = np.concatenate([sl * self.cap + self.length[sl] + np.arange(len(t)) for sl, t in zip(slots, tokens)])
        base = np.concatenate([np.full(len(t), sl * self.cap) for sl, t in zip(slots, tokens)])
        if np.any(pos >= self.cap):
            raise ValueError("sequence longer than its cache slot")
        scale = 1.0 / np.sqrt(D)
        h = embed(toks, w["embed"])
        for l in range(s.layers):
            x = round_bf16(rmsnorm(h, w[f"l{l}.attn_norm"], s.eps))
            qkv = round_bf16(gemm(x, w[f"l{l}.wqkv"]))
            nqk = (Hq + Hkv) * D
            qkv[:, :nqk] = round_bf16(rope(qkv, pos, Hq + Hkv, D, s.theta))
            self.k[l][row] = qkv[:, Hq * D:nqk].reshape(-1, Hkv, D)
            self.v[l][row] = qkv[:, nqk:].reshape(-1, Hkv, D)
            att = round_bf16(causal_attn(qkv, self.k[l], self.v[l], base, pos + 1, Hq, Hkv, scale))
            h = round_bf16(add(h, round_bf16(gemm(att, w[f"l{l}.wo"]))))
            x = round_bf16(rmsnorm(h, w[f"l{l}.mlp_norm"], s.eps))
            a = round_bf16(swiglu(round_bf16(gemm(x, w[f"l{l}.wgu"]))))
            h = round_bf16(add(h, round_bf16(gemm(a, w[f"l{l}.wdown"]))))
        for sl, t in zip(slots, tokens):
            self.length[sl] += len(t)
        last = np.cumsum([len(t) for t in tokens]) - 1
        xf = round_bf16(rmsnorm(np.ascontiguousarray(h[last]), w["final_norm"], s.eps))
        return gemm(xf, w["lm_head"])
