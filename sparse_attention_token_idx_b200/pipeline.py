"""One indexer call on the GPU, in the order the reference forward takes:
append this call's keys to the cache, quantise the queries and fold the head
weights, then score every query row against the cache and select its top-k.

``Indexer`` owns the cache buffers (kept between calls) and the per-call
scratch tensors; every step runs in libidx.so through ``binding``.
"""
from __future__ import annotations

import torch

from . import binding as X


class Indexer:
    """scale_storage "f32": key scales as float32 (either fmt); "e8m0": as one
    e8m0 byte per key (fmt must be ue8m0, T_cap a multiple of 16)."""

    def __init__(self, B: int, T_cap: int, fmt: int, k: int, device="cuda", scale_storage: str = "f32"):
        if scale_storage not in ("f32", "e8m0"):
            raise ValueError("scale_storage must be 'f32' or 'e8m0'")
        if scale_storage == "e8m0" and (fmt != X.FMT_UE8M0 or T_cap % 16):
            raise ValueError("e8m0 scale storage needs fmt = ue8m0 and T_cap a multiple of 16")
        self.B, self.T_cap, self.fmt, self.k = B, T_cap, fmt, k
        self.e8m0 = scale_storage == "e8m0"
        self.device = torch.device(device)
        self.k_cache = torch.zeros((B, T_cap, X.DIM), dtype=torch.uint8, device=self.device)
        self.k_scale_cache = torch.zeros((B, T_cap), dtype=torch.uint8 if self.e8m0 else torch.float32,
                                         device=self.device)
        self._bufs = {}

    def _buf(self, name, shape, dtype):
        t = self._bufs.get(name)
        if t is None or t.shape != shape or t.dtype != dtype:
            t = torch.empty(shape, dtype=dtype, device=self.device)
            self._bufs[name] = t
        return t

    def append(self, k_new: torch.Tensor, positions: torch.Tensor, stream=None):
        """Rotate, quantise and store k_new [B, n, 128] bf16 at slots positions[b] …"""
        if self.e8m0:
            X.quant_append_e8(k_new, positions, self.k_cache, self.k_scale_cache, stream=stream)
        else:
            X.quant_append(k_new, positions, self.k_cache, self.k_scale_cache, self.fmt, stream=stream)

    def step(self, k_new, q, w_raw, positions, lengths, *, causal: bool, max_len: int, out=None, stream=None):
        """k_new [B, n, 128] bf16, q [B, n, 64, 128] bf16, w_raw [B, n, 64] fp32,
        positions [B] int32 (first new slot), lengths [B] int32 (= positions + n),
        max_len ≥ max(lengths) on the host.  Returns top-k positions [B, n, k] int32.
        Launches: rotate + quantise queries and new keys (keys appended to the
        cache; e8m0 storage quantises the two sets apart), then score + top-k
        (fused, or scorer + top-k through the workspace for prefill shapes)."""
        B, n = q.shape[0], q.shape[1]
        q_fp8 = self._buf("q_fp8", tuple(q.shape), torch.uint8)
        w = self._buf("w", tuple(w_raw.shape), torch.float32)
        if self.e8m0:   # queries, then keys with byte scales: two launches
            X.quant_queries(q, w_raw, self.fmt, q_fp8, w, stream=stream)
            X.quant_append_e8(k_new, positions, self.k_cache, self.k_scale_cache, stream=stream)
        else:
            X.quant_queries_append(q, w_raw, k_new, positions, self.k_cache, self.k_scale_cache, self.fmt, q_fp8, w,
                                   stream=stream)
        out = out if out is not None else self._buf("idx", (B, n, self.k), torch.int32)
        ws_bytes = X.workspace_size(B, n, max_len, self.k)
        ws = self._buf("ws", (ws_bytes,), torch.uint8) if ws_bytes else None
        return X.score_topk_ex(q_fp8, w, self.k_cache, self.k_scale_cache, lengths, causal, self.k, max_len,
                               out=out, ws=ws, stream=stream)

    def step_front(self, q_proj, w_raw, k_proj, rope_cos, rope_sin, ln_gain, ln_bias, positions, lengths, *,
                   causal: bool, max_len: int, ln_eps: float = 1e-6, out=None, stream=None):
        """One indexer call from the projections on (the caller's GEMMs: q_proj =
        wq_b(qr) [B, n, 64, 128] bf16, k_proj = wk(x) [B, n, 128] bf16, w_raw =
        weights_proj(x) [B, n, 64] fp32): query RoPE, key LayerNorm + RoPE,
        rotation, quantisation and append in one launch, then score + top-k.
        fp32 scale storage only."""
        if self.e8m0:
            raise ValueError("step_front writes fp32 key scales")
        B, n = k_proj.shape[0], k_proj.shape[1]
        q_fp8 = self._buf("q_fp8", tuple(q_proj.shape), torch.uint8)
        w = self._buf("w", tuple(w_raw.shape), torch.float32)
        X.front_quant_append(q_proj, w_raw, k_proj, rope_cos, rope_sin, ln_gain, ln_bias, ln_eps, positions,
                             self.k_cache, self.k_scale_cache, self.fmt, q_fp8, w, stream=stream)
        out = out if out is not None else self._buf("idx", (B, n, self.k), torch.int32)
        ws_bytes = X.workspace_size(B, n, max_len, self.k)
        ws = self._buf("ws", (ws_bytes,), torch.uint8) if ws_bytes else None
        return X.score_topk_ex(q_fp8, w, self.k_cache, self.k_scale_cache, lengths, causal, self.k, max_len,
                               out=out, ws=ws, stream=stream)

    def capture(self, k_new, q, w_raw, positions, lengths, *, causal: bool, max_len: int):
        """Record one step on static input tensors into a CUDA graph; returns
        (graph, out) — replay the graph after refilling the inputs in place."""
        out = self._buf("idx_graph", (q.shape[0], q.shape[1], self.k), torch.int32)
        s = torch.cuda.Stream(device=self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):                      # warm-up outside the capture
            self.step(k_new, q, w_raw, positions, lengths, causal=causal, max_len=max_len, out=out)
        torch.cuda.current_stream(self.device).wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step(k_new, q, w_raw, positions, lengths, causal=causal, max_len=max_len, out=out)
        return g, out
