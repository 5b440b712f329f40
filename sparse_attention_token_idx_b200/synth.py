"""Seeded synthetic inputs for the lightning indexer.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds no step of the method: it only draws raw bf16 keys
and queries and raw fp32 head weights, and lays out which cache slots a call
fills.  The recipe follows the workload text of the indexer pages: queries
and keys N(0, 1) with two of the 128 channels scaled ×20 (outliers shared by
q and k), weights N(0, 1), then round-to-nearest-even to bf16.

Random stream (NumPy PCG64, seed = 1000 + workload number for the five
workloads): lengths (variable-length decode only), the two outlier channels,
raw keys [B, rows, 128], raw queries [B, n, 64, 128], raw weights [B, n, 64].
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

D = 128
H = 64
T_CAP = 16384          # cache slots per sequence ("Index key cache" page)
TOPK = 2048


@dataclass
class Case:
    name: str
    B: int
    n: int                     # new rows per sequence in this call (queries = keys)
    T_cap: int
    positions: np.ndarray      # int32 [B]: first slot written by this call
    causal: bool
    k: int
    fmt: int                   # 0 = fp32 scale, 1 = ue8m0 (power-of-two) scale
    k_prior: np.ndarray        # uint16 bf16 bits [B, P, 128]: keys already cached (rows < positions[b])
    k_new: np.ndarray          # uint16 bf16 bits [B, n, 128]
    q: np.ndarray              # uint16 bf16 bits [B, n, 64, 128]
    w_raw: np.ndarray          # float32 [B, n, 64]

    @property
    def lengths(self) -> np.ndarray:
        return (self.positions.astype(np.int64) + self.n).astype(np.int32)


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 → bf16 bits, nearest-even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return u.astype(np.uint16)


def make_case(name, seed, B, n, positions, *, T_cap=T_CAP, causal=False, k=TOPK, fmt=0,
              lengths_draw=None, outlier_scale=20.0) -> Case:
    """Draw one call's inputs.  ``positions`` is an int array [B] or, when
    ``lengths_draw`` = (lo, hi) is given, drawn first as integers in [lo, hi)
    minus n (so that lengths = positions + n)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if lengths_draw is not None:
        lo, hi = lengths_draw
        lengths = rng.integers(lo, hi, B)
        positions = lengths - n
    positions = np.asarray(positions, np.int64).reshape(B)
    if np.any(positions < 0) or np.any(positions + n > T_cap):
        raise ValueError("positions out of the cache")
    outliers = rng.choice(D, 2, replace=False)
    rows = int((positions + n).max()) if B else 0
    k_raw = rng.standard_normal((B, rows, D), dtype=np.float32)
    q_raw = rng.standard_normal((B, n, H, D), dtype=np.float32)
    w_raw = rng.standard_normal((B, n, H), dtype=np.float32)
    k_raw[..., outliers] *= np.float32(outlier_scale)
    q_raw[..., outliers] *= np.float32(outlier_scale)
    k_bits = _to_bf16_bits(k_raw)
    P = int(positions.max()) if B else 0
    k_prior = np.zeros((B, P, D), np.uint16)
    k_new = np.zeros((B, n, D), np.uint16)
    for b in range(B):
        p = int(positions[b])
        k_prior[b, :p] = k_bits[b, :p]
        k_new[b] = k_bits[b, p:p + n]
    return Case(name, B, n, T_cap, positions.astype(np.int32), causal, k, fmt,
                k_prior, k_new, _to_bf16_bits(q_raw), w_raw)


WORKLOADS = {
    0: "decode B=1 T=4096 fp32-scale",
    1: "decode B=16 len~U[1,16384] fp32-scale",
    2: "decode B=128 T=16384 ue8m0-scale",
    3: "prefill B=1 seqlen=4096 causal fp32-scale",
    4: "chunked prefill B=2 2048@14336 causal ue8m0-scale",
}


def workload(idx: int) -> Case:
    """The five benchmark workloads (seed = 1000 + idx)."""
    seed = 1000 + idx
    name = WORKLOADS[idx]
    if idx == 0:
        return make_case(name, seed, 1, 1, [4095], fmt=0)
    if idx == 1:
        return make_case(name, seed, 16, 1, None, fmt=0, lengths_draw=(1, T_CAP + 1))
    if idx == 2:
        return make_case(name, seed, 128, 1, [T_CAP - 1] * 128, fmt=1)
    if idx == 3:
        return make_case(name, seed, 1, 4096, [0], causal=True, fmt=0)
    if idx == 4:
        return make_case(name, seed, 2, 2048, [14336, 14336], causal=True, fmt=1)
    raise KeyError(idx)


# --------------------------------------------------------------------------- projections
HIDDEN = 7168          # hidden width of the synthetic projections (a multiple of 128)
Q_LORA = 1536          # low-rank query width (a multiple of 512, the NKI page's MX K-tile)


@dataclass
class ProjCase:
    x: np.ndarray          # uint16 bf16 bits [T, hidden]
    qr: np.ndarray         # uint16 bf16 bits [T, q_lora]
    wq_b: np.ndarray       # uint16 bf16 bits [64·128, q_lora]  (Linear layout [out, in])
    wk: np.ndarray         # uint16 bf16 bits [128, hidden]
    w_proj: np.ndarray     # float32 [64, hidden]


def make_proj_case(seed, tokens, hidden=HIDDEN, q_lora=Q_LORA) -> ProjCase:
    """Random projection inputs and weights: x, qr ~ N(0, 1); each weight
    matrix ~ N(0, 1 / fan_in) so that the outputs are O(1).  Drawn in this
    order with NumPy PCG64(seed): x, qr, wq_b, wk, w_proj."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((tokens, hidden), dtype=np.float32)
    qr = rng.standard_normal((tokens, q_lora), dtype=np.float32)
    wq = rng.standard_normal((H * D, q_lora), dtype=np.float32) / np.float32(np.sqrt(q_lora))
    wk = rng.standard_normal((D, hidden), dtype=np.float32) / np.float32(np.sqrt(hidden))
    wp = rng.standard_normal((H, hidden), dtype=np.float32) / np.float32(np.sqrt(hidden))
    return ProjCase(_to_bf16_bits(x), _to_bf16_bits(qr), _to_bf16_bits(wq), _to_bf16_bits(wk), wp.astype(np.float32))
