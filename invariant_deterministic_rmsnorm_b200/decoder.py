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
    bi_rope(q and k heads of qkv, positions, the cos/sin table built once per engine)
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


class BIOps:
    """The three batch-dependent-in-general ops of a step, on the library's batch-invariant kernels.

    A Decoder takes another table with the same three calls only to measure an alternative
    (see bench.py --contrast).  The default is always this one."""

    @staticmethod
    def gemm(A, W, C=None, out_dtype=torch.bfloat16):
        return bi.bi_gemm(A, W, C=C, out_dtype=out_dtype)

    @staticmethod
    def rmsnorm(x, w, y=None, eps=1e-6):
        return bi.bi_rmsnorm(x, w, y=y, eps=eps)

    @staticmethod
    def decode_attn(q, k, v, kv_indptr, kv_len, out, workspace):
        return bi.bi_decode_attn(q, k, v, kv_indptr, kv_len, out=out, workspace=workspace)


def _dev_i32(a, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(device, non_blocking=False)


class Decoder:
    """A decoder with weights `weights` (bf16 device tensors named as DecoderShape.matrices())."""

    def __init__(self, shape: DecoderShape, weights: dict, max_seqs: int, max_len: int, device="cuda",
                 decode_attention: str = "split", ops=BIOps):
        if shape.head_dim != 128:
            raise ValueError("the attention kernels take head_dim 128")
        if decode_attention not in ("split", "prefill"):
            raise ValueError("decode_attention is 'split' (bi_decode_attn) or 'prefill' (bi_prefill_attn)")
        self.s, self.w, self.device = shape, weights, torch.device(device)
        self.max_seqs = max_seqs
        self.cap = (max_len + CHUNK - 1) // CHUNK * CHUNK
        self.decode_attention = decode_attention
        self.ops = ops
        rows = max_seqs * self.cap
        kv = (rows, shape.kv_heads, shape.head_dim)
        self.k_cache = [torch.zeros(kv, dtype=torch.bfloat16, device=self.device) for _ in range(shape.layers)]
        self.v_cache = [torch.zeros(kv, dtype=torch.bfloat16, device=self.device) for _ in range(shape.layers)]
        self.length = np.zeros(max_seqs, np.int64)
        self.rope_table = bi.bi_rope_table(self.cap, shape.head_dim, shape.theta, device=self.device)
        ws = bi.bi_decode_attn_workspace_size(rows, shape.q_heads, shape.head_dim, CHUNK)
        self.attn_ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=self.device)

    def reset(self, slots=None) -> None:
        """Forget the cached tokens of `slots` (all when None); cache contents are simply overwritten later."""
        if slots is None:
            self.length[:] = 0
        else:
            self.length[np.asarray(slots)] = 0

    def share_prefix(self, src: int, dst: int, n: int) -> None:
        """A prefix-cache hit: sequence `dst` starts from the first n cached tokens of sequence `src`.

        The K and V rows of positions 0 .. n-1 are copied from src's cache slot into dst's in every
        layer (bi_kv_append, a row scatter), and dst's length becomes n.  Its next prefill then
        appends after them.  Because a cached row depends only on the tokens up to its position,
        dst's logits are bitwise those of prefilling its whole prompt from scratch."""
        src, dst, n = int(src), int(dst), int(n)
        if not (0 <= src < self.max_seqs and 0 <= dst < self.max_seqs) or src == dst:
            raise ValueError("src and dst must be two different slots")
        if not 0 < n <= self.length[src]:
            raise ValueError("the shared prefix must be cached in src")
        rows = _dev_i32(dst * self.cap + np.arange(n), self.device)
        width = self.s.kv_heads * self.s.head_dim
        for cache in self.k_cache + self.v_cache:
            rows_src = cache[src * self.cap:src * self.cap + n].view(n, width)
            bi.bi_kv_append(rows_src, rows, cache)
        self.length[dst] = n

    # ------------------------------------------------------------------ one step
    def _plan(self, slots, tokens, phase):
        """Check a step and build its host-side index arrays."""
        slots = [int(x) for x in slots]
        if not slots or any(b <= a for a, b in zip(slots, slots[1:])) or slots[0] < 0 or slots[-1] >= self.max_seqs:
            raise ValueError("slots must be strictly increasing and inside [0, max_seqs)")
        lens = np.array([len(t) for t in tokens], np.int64)
        if len(lens) != len(slots) or np.any(lens <= 0):
            raise ValueError("every listed sequence needs at least one new token")
        if phase not in ("prefill", "decode"):
            raise ValueError("phase is 'prefill' or 'decode'")
        if phase == "decode" and np.any(lens != 1):
            raise ValueError("a decode step takes exactly one new token per sequence")
        start = self.length[slots]
        if np.any(start + lens > self.cap):
            raise ValueError("a sequence outgrows its cache slot")
        slot_arr = np.asarray(slots, np.int64)
        pos = np.concatenate([st + np.arange(n) for st, n in zip(start, lens)])
        q_indptr = np.concatenate([[0], np.cumsum(lens)])
        split = phase == "decode" and self.decode_attention == "split"
        plan = {"T": int(lens.sum()), "B": len(slots), "split": split, "slots": slots, "lens": lens,
                "tok": np.concatenate([np.asarray(t, np.int32) for t in tokens]), "pos": pos,
                "rows": np.repeat(slot_arr * self.cap, lens) + pos, "last": q_indptr[1:] - 1}
        if split:
            plan["kv_indptr"] = np.concatenate([slot_arr * self.cap, [(slot_arr[-1] + 1) * self.cap]])
            plan["kv_len"] = start + 1
            plan["seq"] = np.arange(len(slots))
        else:
            plan["tiles"] = bi.prefill_tiles(lens)
            plan["q_indptr"], plan["kv_base"], plan["pos0"] = q_indptr, slot_arr * self.cap, start
        return plan

    _INDEX_KEYS = ("tok", "pos", "rows", "last", "kv_indptr", "kv_len", "seq", "tiles", "q_indptr", "kv_base", "pos0")

    def _upload(self, plan) -> dict:
        return {k: _dev_i32(plan[k], self.device) for k in self._INDEX_KEYS if k in plan}

    def _run(self, T: int, split: bool, n_tiles: int, d: dict) -> torch.Tensor:
        """The device part of a step: every launch reads its indices from the int32 tensors in d."""
        s, w, dev, ops = self.s, self.w, self.device, self.ops
        Hq, Hkv, D, H = s.q_heads, s.kv_heads, s.head_dim, s.hidden
        bf = torch.bfloat16
        h = bi.bi_embed(d["tok"], w["embed"])
        x = torch.empty((T, H), dtype=bf, device=dev)
        qkv = torch.empty((T, s.qkv_cols), dtype=bf, device=dev)
        att = torch.empty((T, Hq * D), dtype=bf, device=dev)
        o = torch.empty((T, H), dtype=bf, device=dev)
        gu = torch.empty((T, 2 * s.ffn), dtype=bf, device=dev)
        a = torch.empty((T, s.ffn), dtype=bf, device=dev)
        qbuf = torch.empty((T, Hq, D), dtype=bf, device=dev) if split else None
        for l in range(s.layers):
            ops.rmsnorm(h, w[f"l{l}.attn_norm"], y=x, eps=s.eps)
            ops.gemm(x, w[f"l{l}.wqkv"], C=qkv)
            bi.bi_rope(qkv, d["pos"], Hq + Hkv, self.rope_table, D)
            kc, vc = self.k_cache[l], self.v_cache[l]
            bi.bi_kv_append(qkv[:, Hq * D:(Hq + Hkv) * D], d["rows"], kc)
            bi.bi_kv_append(qkv[:, (Hq + Hkv) * D:], d["rows"], vc)
            if split:
                bi.bi_kv_append(qkv, d["seq"], qbuf)  # pack the query heads: [B, Hq, D]
                ops.decode_attn(qbuf, kc, vc, d["kv_indptr"], d["kv_len"], att.view(T, Hq, D), self.attn_ws)
            else:
                bi.bi_prefill_attn(qkv, kc, vc, d["q_indptr"], d["tiles"], n_tiles, d["kv_base"], d["pos0"], Hq,
                                   out=att)
            ops.gemm(att, w[f"l{l}.wo"], C=o)
            bi.bi_add(h, o)
            ops.rmsnorm(h, w[f"l{l}.mlp_norm"], y=x, eps=s.eps)
            ops.gemm(x, w[f"l{l}.wgu"], C=gu)
            bi.bi_swiglu(gu, out=a)
            ops.gemm(a, w[f"l{l}.wdown"], C=o)
            bi.bi_add(h, o)
        last = bi.bi_embed(d["last"], h)  # row gather: the last new token of each sequence
        xf = ops.rmsnorm(last, w["final_norm"], eps=s.eps)
        return ops.gemm(xf, w["lm_head"], out_dtype=torch.float32)

    def forward(self, slots, tokens, phase: str = "prefill") -> torch.Tensor:
        """Append tokens[i] (a list of ids) to sequence slots[i], for all i, and run the model over them.

        slots must be strictly increasing.  phase "prefill" runs causal prefill attention over any
        number of new tokens per sequence; "decode" takes exactly one new token per sequence.
        Returns fp32 logits [len(slots), vocab] of each sequence's last new token."""
        plan = self._plan(slots, tokens, phase)
        logits = self._run(plan["T"], plan["split"], plan.get("tiles", [0])[-1], self._upload(plan))
        self.length[plan["slots"]] += plan["lens"]
        return logits

    def decode_graph(self, slots) -> "DecodeGraph":
        """A CUDA graph of one greedy decode step over `slots` (see DecodeGraph)."""
        return DecodeGraph(self, slots)

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


class DecodeGraph:
    """One greedy decode step over a fixed set of slots, captured once in a CUDA graph.

    The graph reads the current tokens from a device buffer, appends them at each sequence's
    next position, writes the logits to a static fp32 buffer, and writes the greedy next tokens
    back into the token buffer.  It then advances the device copies of the positions, cache
    rows and KV lengths (or, with prefill attention, the first query positions) by one, with a
    library launch like every other step of the graph.  Consecutive replays thus decode greedily with no host work.
    The host mirrors the lengths in Decoder.length.

    Every launch in the graph is the same launch as in Decoder.forward(..., "decode").  The graph
    changes when work is issued, not what is computed, so a replayed step gives bitwise the
    logits of the eager step.
    """

    def __init__(self, dec: Decoder, slots):
        self.dec = dec
        self.slots = [int(x) for x in slots]
        B = len(self.slots)
        plan = dec._plan(self.slots, [[0]] * B, "decode")
        self.d = dec._upload(plan)
        # positions, cache rows and KV lengths move together; keep them in one buffer so that one
        # library launch (bi_advance) advances them all
        adv = np.stack([np.asarray(plan[k], np.int32) for k in (["pos", "rows", "kv_len"] if plan["split"]
                                                                   else ["pos", "rows"])])
        self.adv = _dev_i32(adv, dec.device)
        self.d["pos"], self.d["rows"] = self.adv[0], self.adv[1]
        if plan["split"]:
            self.d["kv_len"] = self.adv[2]
        else:
            self.d["pos0"] = self.adv[0]  # one query row per sequence: its first row is its only row
        self.split, self.B = plan["split"], B
        n_tiles = plan.get("tiles", [0])[-1]
        stream = torch.cuda.Stream(dec.device)
        stream.wait_stream(torch.cuda.current_stream(dec.device))
        with torch.cuda.stream(stream):
            dec._run(B, self.split, n_tiles, self.d)  # warm-up: per-device set-up happens outside the capture
        torch.cuda.current_stream(dec.device).wait_stream(stream)
        torch.cuda.synchronize(dec.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=stream):
            self.logits = dec._run(B, self.split, n_tiles, self.d)
            bi.bi_argmax(self.logits, out=self.d["tok"])
            bi.bi_advance(self.adv, 1)

    def set_tokens(self, tokens) -> None:
        """Tokens for the next replay (otherwise the previous replay's greedy tokens are used)."""
        t = tokens if isinstance(tokens, torch.Tensor) else torch.as_tensor(np.asarray(tokens, np.int32))
        self.d["tok"].copy_(t.to(self.dec.device, torch.int32))

    def replay(self) -> torch.Tensor:
        """One decode step; returns the static logits buffer (valid until the next replay)."""
        if np.any(self.dec.length[self.slots] + 1 > self.dec.cap):
            raise ValueError("a sequence outgrows its cache slot")
        self.graph.replay()
        self.dec.length[self.slots] += 1
        return self.logits

    def tokens(self) -> torch.Tensor:
        return self.d["tok"]
