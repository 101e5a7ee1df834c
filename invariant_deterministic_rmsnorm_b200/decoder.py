"""A batch-invariant Llama-shaped decoder built only from the library's kernels.

Source: "Defeating Nondeterminism in LLM Inference" (Spanish summary), sections "La verdadera
causa clave" and "Attention".  A request's output changes with the batch it shares unless
every op gives a token row the same bits at any batch size.  Attention must also reduce each
query's keys in one fixed order over one layout that cached and new tokens share.  This
engine strings the batch-invariant ops together, so a request's logits come out bitwise
the same whether it runs alone or among up to max_seqs others.

Each op of a step runs in a libbi.so kernel (see binding.py).  PyTorch supplies device memory,
the stream, and the few small int32 index arrays that this module builds on the host.  Per
layer:

    x   = bi_rmsnorm(h)                   qkv = bi_gemm(x, Wqkv)            (bf16)
    bi_rope(q and k heads of qkv, positions)
    bi_kv_append(k, v -> the layer's packed caches at each token's slot row)
    att = bi_prefill_attn(q, caches)     or, for one new token per sequence,
          bi_decode_attn(q, caches)       (256-token split-KV, fixed split size)
    h  += bi_gemm(att, Wo)               (bi_add)
    x   = bi_rmsnorm(h)                   gu = bi_gemm(x, Wgu)
    h  += bi_gemm(bi_swiglu(gu), Wdown)  (bi_add)

then the last row of each sequence is gathered (bi_embed on h), normalised, and projected to
fp32 logits with bi_gemm.  bi_argmax picks greedy tokens.

KV cache: sequence slot s owns rows s*cap .. s*cap + cap - 1 of each layer's K and V caches
[max_seqs*cap, Hkv, 128] (cap a multiple of the 256-token decode chunk).  Position p of the
sequence is row s*cap + p.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as bi
from .inputs import DecoderShape

CHUNK = 256


def _dev_i32(a, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(device, non_blocking=False)


class Decoder:
    """A decoder with weights `weights` (bf16 device tensors named as DecoderShape.matrices())."""

    def __init__(self, shape: DecoderShape, weights: dict, max_seqs: int, max_len: int, device="cuda",
                 decode_attention: str = "split"):
        if shape.head_dim != 128:
            raise ValueError("the attention kernels take head_dim 128")
        if decode_attention not in ("split", "prefill"):
            raise ValueError("decode_attention is 'split' (bi_decode_attn) or 'prefill' (bi_prefill_attn)")
        self.s, self.w, self.device = shape, weights, torch.device(device)
        self.max_seqs = max_seqs
        self.cap = (max_len + CHUNK - 1) // CHUNK * CHUNK
        self.decode_attention = decode_attention
        rows = max_seqs * self.cap
        kv = (rows, shape.kv_heads, shape.head_dim)
        self.k_cache = [torch.zeros(kv, dtype=torch.bfloat16, device=self.device) for _ in range(shape.layers)]
        self.v_cache = [torch.zeros(kv, dtype=torch.bfloat16, device=self.device) for _ in range(shape.layers)]
        self.length = np.zeros(max_seqs, np.int64)
        ws = bi.bi_decode_attn_workspace_size(rows, shape.q_heads, shape.head_dim, CHUNK)
        self.attn_ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=self.device)

    def reset(self, slots=None) -> None:
        """Forget the cached tokens of `slots` (all when None); cache contents are simply overwritten later."""
        if slots is None:
            self.length[:] = 0
        else:
            self.length[np.asarray(slots)] = 0

    # ------------------------------------------------------------------ one step
    def forward(self, slots, tokens, phase: str = "prefill") -> torch.Tensor:
        """Append tokens[i] (a list of ids) to sequence slots[i], for all i, and run the model over them.

        slots must be strictly increasing.  phase "prefill" runs causal prefill attention over any
        number of new tokens per sequence; "decode" takes exactly one new token per sequence.
        Returns fp32 logits [len(slots), vocab] of each sequence's last new token."""
        s, w, dev = self.s, self.w, self.device
        slots = [int(x) for x in slots]
        if not slots or any(b <= a for a, b in zip(slots, slots[1:])) or slots[0] < 0 or slots[-1] >= self.max_seqs:
            raise ValueError("slots must be strictly increasing and inside [0, max_seqs)")
        lens = np.array([len(t) for t in tokens], np.int64)
        if len(lens) != len(slots) or np.any(lens <= 0):
            raise ValueError("every listed sequence needs at least one new token")
        if phase == "decode" and np.any(lens != 1):
            raise ValueError("a decode step takes exactly one new token per sequence")
        if phase not in ("prefill", "decode"):
            raise ValueError("phase is 'prefill' or 'decode'")
        start = self.length[slots]
        if np.any(start + lens > self.cap):
            raise ValueError("a sequence outgrows its cache slot")
        Hq, Hkv, D, H = s.q_heads, s.kv_heads, s.head_dim, s.hidden
        T, B = int(lens.sum()), len(slots)
        slot_arr = np.asarray(slots, np.int64)

        # host-built index arrays (positions, cache rows, sequence boundaries)
        pos = np.concatenate([st + np.arange(n) for st, n in zip(start, lens)])
        rows = np.repeat(slot_arr * self.cap, lens) + pos
        q_indptr = np.concatenate([[0], np.cumsum(lens)])
        toks = np.concatenate([np.asarray(t, np.int32) for t in tokens])
        d_tok, d_pos, d_rows = _dev_i32(toks, dev), _dev_i32(pos, dev), _dev_i32(rows, dev)
        d_last = _dev_i32(q_indptr[1:] - 1, dev)
        use_split = phase == "decode" and self.decode_attention == "split"
        if use_split:
            kv_indptr = np.concatenate([slot_arr * self.cap, [(slot_arr[-1] + 1) * self.cap]])
            d_kv_indptr, d_kv_len = _dev_i32(kv_indptr, dev), _dev_i32(start + 1, dev)
            d_seq = _dev_i32(np.arange(B), dev)
        else:
            tiles = bi.prefill_tiles(lens)
            d_q_indptr, d_tiles = _dev_i32(q_indptr, dev), _dev_i32(tiles, dev)
            d_kv_base, d_pos0 = _dev_i32(slot_arr * self.cap, dev), _dev_i32(start, dev)

        bf = torch.bfloat16
        h = bi.bi_embed(d_tok, w["embed"])
        x = torch.empty((T, H), dtype=bf, device=dev)
        qkv = torch.empty((T, s.qkv_cols), dtype=bf, device=dev)
        att = torch.empty((T, Hq * D), dtype=bf, device=dev)
        o = torch.empty((T, H), dtype=bf, device=dev)
        gu = torch.empty((T, 2 * s.ffn), dtype=bf, device=dev)
        a = torch.empty((T, s.ffn), dtype=bf, device=dev)
        qbuf = torch.empty((T, Hq, D), dtype=bf, device=dev) if use_split else None
        for l in range(s.layers):
            bi.bi_rmsnorm(h, w[f"l{l}.attn_norm"], y=x, eps=s.eps)
            bi.bi_gemm(x, w[f"l{l}.wqkv"], C=qkv)
            bi.bi_rope(qkv, d_pos, Hq + Hkv, D, s.theta)
            kc, vc = self.k_cache[l], self.v_cache[l]
            bi.bi_kv_append(qkv[:, Hq * D:(Hq + Hkv) * D], d_rows, kc)
            bi.bi_kv_append(qkv[:, (Hq + Hkv) * D:], d_rows, vc)
            if use_split:
                bi.bi_kv_append(qkv, d_seq, qbuf)  # pack the query heads: [B, Hq, D]
                bi.bi_decode_attn(qbuf, kc, vc, d_kv_indptr, d_kv_len, out=att.view(T, Hq, D),
                                  workspace=self.attn_ws)
            else:
                bi.bi_prefill_attn(qkv, kc, vc, d_q_indptr, d_tiles, tiles[-1], d_kv_base, d_pos0, Hq, out=att)
            bi.bi_gemm(att, w[f"l{l}.wo"], C=o)
            bi.bi_add(h, o)
            bi.bi_rmsnorm(h, w[f"l{l}.mlp_norm"], y=x, eps=s.eps)
            bi.bi_gemm(x, w[f"l{l}.wgu"], C=gu)
            bi.bi_swiglu(gu, out=a)
            bi.bi_gemm(a, w[f"l{l}.wdown"], C=o)
            bi.bi_add(h, o)
        self.length[slots] = start + lens
        last = bi.bi_embed(d_last, h)  # row gather: the last new token of each sequence
        xf = bi.bi_rmsnorm(last, w["final_norm"], eps=s.eps)
        return bi.bi_gemm(xf, w["lm_head"], out_dtype=torch.float32)

    # ------------------------------------------------------------------ greedy generation
    def generate(self, slots, prompts, steps: int, keep=None):
        """Prefill `prompts` into `slots`, then run `steps` greedy decode steps.

        Returns (logits, tokens).  logits[i] is a list of fp32 host arrays, one per step
        (prefill included), for each sequence i in `keep` (all when None).  tokens [len(slots),
        steps + 1] holds the greedy tokens."""
        keep = list(range(len(slots))) if keep is None else list(keep)
        out = {i: [] for i in keep}
        toks = []
        logits = self.forward(slots, prompts, "prefill")
        for it in range(steps + 1):
            nxt = bi.bi_argmax(logits)
            for i in keep:
                out[i].append(logits[i].cpu().numpy())
            toks.append(nxt.cpu().numpy())
            if it == steps:
                break
            logits = self.forward(slots, [[int(t)] for t in toks[-1]], "decode")
        return [out[i] for i in keep], np.stack(toks, 1)
