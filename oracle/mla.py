"""CPU oracle for the sparse latent attention that consumes the indexer's
selection — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and
reference legs) may import this module; the product path never imports it, and
it imports nothing of the product path.

What it computes ("Join query parts" page, the MQA decode excerpt): one decode
token per sequence attends, head by head, over the cached latent rows the
indexer selected.  Each cached position holds 576 features, the 512-wide latent
c_t followed by the 64-wide rotary key r_t; each head's query is the absorbed
content query followed by its rotary query, 576 features (joining the two
parts gives the same product as adding their two scores, as the page says).

    s[h, t] = softmax_scale · Σ_d q[h, d] · kv[t, d]     (t among the selected)
    p[h, ·] = softmax over the selected t of s[h, ·]     (every other t is −inf)
    o[h, j] = Σ_t p[h, t] · kv[t, j],  j < 512           (the latent output,
                                                          before the value
                                                          up-projection)

Readings taken where the pages are silent:
* queries and the cache are bf16 values; everything here is float64;
* a selection entry of −1 (the indexer's padding) selects nothing; a row with
  no selected position has output 0;
* the value up-projection (wkv_b) after the latent output needs trained
  weights and is not part of this step.
"""
from __future__ import annotations

import numpy as np

LAT = 512      # latent width (kv_lora_rank)
ROPE = 64      # rotary width
DIM = LAT + ROPE


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def sparse_mla_decode(q_bits, kv_bits, indices, softmax_scale):
    """q_bits [B, H, 576] bf16 bits, kv_bits [B, T, 576] bf16 bits, indices
    [B, k] int (−1 = none).  Returns (o [B, H, 512] float64, and the weights
    p [B, H, k] float64 aligned with ``indices``, 0 where nothing is selected)."""
    q = bf16_bits_to_f64(q_bits)
    B, H, _ = q.shape
    k = np.asarray(indices).shape[1]
    o = np.zeros((B, H, LAT))
    P = np.zeros((B, H, k))
    for b in range(B):
        sel = np.asarray(indices[b], np.int64)
        ok = sel >= 0
        if not ok.any():
            continue
        kv = bf16_bits_to_f64(kv_bits[b, sel[ok]])           # [n_sel, 576]
        s = float(softmax_scale) * (q[b] @ kv.T)              # [H, n_sel]
        e = np.exp(s - s.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)
        o[b] = p @ kv[:, :LAT]
        P[b][:, ok] = p
    return o, P
