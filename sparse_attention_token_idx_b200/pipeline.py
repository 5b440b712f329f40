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

    def step_hidden(self, x, qr, wq_b, wk, w_proj, rope_cos, rope_sin, ln_gain, ln_bias, positions, lengths, *,
                    causal: bool, max_len: int, ln_eps: float = 1e-6, out=None, stream=None):
        """One indexer call from the hidden state: x [B, n, hidden] bf16 and qr
        [B, n, q_lora] bf16 through the projections (wq_b [8192, q_lora], wk
        [128, hidden] bf16, w_proj [64, hidden] fp32), then as step_front.  The
        projection outputs stay in this object's buffers (projections())."""
        B, n = x.shape[0], x.shape[1]
        T = B * n
        hidden, q_lora = x.shape[2], qr.shape[2]
        q_proj = self._buf("q_proj", (B, n, X.HEADS, X.DIM), torch.bfloat16)
        k_proj = self._buf("k_proj", (B, n, X.DIM), torch.bfloat16)
        w_raw = self._buf("w_raw", (B, n, X.HEADS), torch.float32)
        need = X.project_workspace_size(T, hidden, q_lora)
        ws = self._buf("proj_ws", (need,), torch.uint8)
        X.project(x.reshape(T, hidden), qr.reshape(T, q_lora), wq_b, wk, w_proj, q_out=q_proj.view(T, X.HEADS, X.DIM),
                  k_out=k_proj.view(T, X.DIM), w_out=w_raw.view(T, X.HEADS), ws=ws, stream=stream)
        return self.step_front(q_proj, w_raw, k_proj, rope_cos, rope_sin, ln_gain, ln_bias, positions, lengths,
                               causal=causal, max_len=max_len, ln_eps=ln_eps, out=out, stream=stream)

    def projections(self):
        """(q_proj, k_proj, w_raw) of the last step_hidden."""
        return self._bufs["q_proj"], self._bufs["k_proj"], self._bufs["w_raw"]

    def capture(self, k_new, q, w_raw, positions, lengths, *, causal: bool, max_len: int, out=None):
        """Record one step on static input tensors into a CUDA graph; returns
        (graph, out) — replay the graph after refilling the inputs in place.
        The step also runs once, for real, before the capture (warm-up)."""
        if out is None:
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


class HostPipeline:
    """Indexer steps fed from pinned host memory with the copies overlapped.

    A submitted step copies its inputs host → device on an upload stream,
    replays its CUDA graph on the compute stream once they have landed, and
    copies the top-k indices device → host on a download stream.  Two slots of
    device buffers (each with its own graph) let step i+1's upload and step
    i−1's download run while step i computes.  Steps compute in submission
    order on one stream, so each sees the cache as the steps before it left it.
    A slot's graph is captured at its first use; that capture's warm-up run is
    the step itself.
    """

    # the step's inputs, in the order they are packed: name, shape (B, n), dtype
    FIELDS = (("k", lambda B, n: (B, n, X.DIM), torch.bfloat16),
              ("q", lambda B, n: (B, n, X.HEADS, X.DIM), torch.bfloat16),
              ("w", lambda B, n: (B, n, X.HEADS), torch.float32),
              ("p", lambda B, n: (B,), torch.int32),
              ("l", lambda B, n: (B,), torch.int32))

    def _layout(self):
        """(name, shape, dtype, byte offset) of each input in a packed buffer
        (offsets rounded up to 256 bytes), and the buffer's size."""
        out, off = [], 0
        for name, shape_of, dt in self.FIELDS:
            shape = shape_of(self.B, self.n)
            nbytes = torch.Size(shape).numel() * torch.empty((), dtype=dt).element_size()
            out.append((name, shape, dt, off))
            off = (off + nbytes + 255) // 256 * 256
        return out, off

    def _views(self, buf):
        return {name: buf[off:off + torch.Size(shape).numel() * torch.empty((), dtype=dt).element_size()]
                .view(dt).view(shape) for name, shape, dt, off in self.layout}

    def __init__(self, indexer: Indexer, B: int, n: int, *, causal: bool, max_len: int, slots: int = 2):
        if slots < 1:
            raise ValueError("slots must be ≥ 1")
        dev = indexer.device
        self.ix, self.causal, self.max_len = indexer, causal, max_len
        self.B, self.n = B, n
        self.layout, self.packed_bytes = self._layout()
        self.packed_hosts = {}      # data_ptr of a host_inputs() buffer → that buffer
        self.up = torch.cuda.Stream(device=dev)
        self.comp = torch.cuda.Stream(device=dev)
        self.down = torch.cuda.Stream(device=dev)
        self.slots = []
        for _ in range(slots):
            packed = torch.empty((self.packed_bytes,), dtype=torch.uint8, device=dev)
            v = self._views(packed)
            self.slots.append({
                "packed": packed,
                "k": v["k"], "q": v["q"], "w": v["w"], "p": v["p"], "l": v["l"],
                "out": torch.empty((B, n, indexer.k), dtype=torch.int32, device=dev),
                "graph": None,
                "uploaded": torch.cuda.Event(),
                "computed": torch.cuda.Event(),
                "downloaded": torch.cuda.Event(),
                "used": False,
            })
        self.count = 0

    def wait(self, event: torch.cuda.Event):
        """Make the next uploads, computes and downloads start after `event`."""
        for st in (self.up, self.comp, self.down):
            st.wait_event(event)

    def join(self, stream=None):
        """Make `stream` (default: the current one) wait for everything submitted."""
        stream = stream if stream is not None else torch.cuda.current_stream(self.ix.device)
        stream.wait_stream(self.comp)
        stream.wait_stream(self.down)

    def host_inputs(self):
        """Pinned host tensors (k_new, q, w_raw, positions, lengths) packed in one
        buffer with the device slots' layout: a step submitted with exactly these
        views is uploaded by a single copy.  Allocate several for rotation."""
        buf = torch.empty((self.packed_bytes,), dtype=torch.uint8).pin_memory()
        self.packed_hosts[buf.data_ptr()] = buf
        v = self._views(buf)
        return v["k"], v["q"], v["w"], v["p"], v["l"]

    def _packed_of(self, hs):
        """The host_inputs() buffer that the five tensors are the views of, or None."""
        buf = self.packed_hosts.get(hs[0].data_ptr())
        if buf is None:
            return None
        base = buf.data_ptr()
        for h, (name, shape, dt, off) in zip(hs, self.layout):
            if h.data_ptr() != base + off or tuple(h.shape) != tuple(shape) or h.dtype != dt:
                return None
        return buf

    def submit(self, h_k, h_q, h_w, h_p, h_l, h_out) -> torch.cuda.Event:
        """One step: pinned host inputs k_new [B, n, 128] bf16, q [B, n, 64, 128]
        bf16, w_raw [B, n, 64] fp32, positions [B], lengths [B] int32 (the views
        of one host_inputs() buffer: a single upload); the indices land in
        pinned h_out [B, n, k] int32 once the returned event has completed.
        Refill the host inputs (or reuse h_out) only after that event, or
        rotate several host buffers."""
        s = self.slots[self.count % len(self.slots)]
        self.count += 1
        if s["used"]:
            self.up.wait_event(s["computed"])        # the slot's inputs are free once its last step computed
        packed = self._packed_of((h_k, h_q, h_w, h_p, h_l))
        with torch.cuda.stream(self.up):
            if packed is not None:            # one copy for the whole step
                s["packed"].copy_(packed, non_blocking=True)
            else:
                for name, h in (("k", h_k), ("q", h_q), ("w", h_w), ("p", h_p), ("l", h_l)):
                    s[name].copy_(h, non_blocking=True)
        s["uploaded"].record(self.up)
        self.comp.wait_event(s["uploaded"])
        if s["used"]:
            self.comp.wait_event(s["downloaded"])    # the slot's output is free once it was read back
        with torch.cuda.stream(self.comp):
            if s["graph"] is None:
                s["graph"], _ = self.ix.capture(s["k"], s["q"], s["w"], s["p"], s["l"], causal=self.causal,
                                                max_len=self.max_len, out=s["out"])
            else:
                s["graph"].replay()
        s["computed"].record(self.comp)
        self.down.wait_event(s["computed"])
        with torch.cuda.stream(self.down):
            h_out.copy_(s["out"], non_blocking=True)
        s["downloaded"].record(self.down)
        s["used"] = True
        return s["downloaded"]
