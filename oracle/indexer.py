"""CPU oracle for the DeepSeek-V3.2 lightning indexer — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and
reference legs) may import this module.  The product path (the CUDA library and
its Python binding) never imports, calls or links it, and the oracle never
imports the product path: the two share no code.  The only module both sides
use is the seeded input generator, which holds none of the method's arithmetic.

What it computes, step by step, with the passage each step follows:

* ``hadamard128``      — "Hadamard rotation" page, rotation equation
  (k̄ = k̃ · H_128 / √128) and its note that the transform is orthonormal.
* ``quant_rows``       — the block-FP8 quantisation that follows the rotation
  on the same page ("FP8 quantization of queries and keys in groups of 128
  features"), with one float32 scale per 128 features ("Index key cache" page,
  cache buffer excerpt); the ue8m0 option is the power-of-two scale named in
  the ``fp8_index`` docstring on the "Index scores" page ("e8m0 here").
* ``quant_append``     — "Index key cache" page: the new FP8 keys and scales are
  stored at positions start_pos … end_pos−1 of the per-sequence cache before
  any scoring.
* ``fold_weights``     — "Index scores" page, text under the score equation:
  1/√64 is folded into the head weights, and 1/√128 together with each query's
  FP8 scale.
* ``index_scores``     — "Index scores" page, score equation S^I and the
  ``fp8_index`` docstring (FP8 logits → ReLU → × weight → sum over heads →
  × key scale), plus the causal mask added in prefill (``Indexer.forward``
  excerpt).  ``index_scores_rows`` computes the same for many rows of one
  sequence with matrix products as its steps (full-size checks).
* ``topk``             — ``Indexer.forward`` excerpt (top min(index_topk, ·)
  positions per row) and the NKI "DeepSeek-V3.2 Sparse Indexer Kernel API
  Reference" page, Notes and return types (int32, an unordered set).
* ``project`` — the three projections that open the ``Indexer.forward``
  excerpt (wq_b of the low-rank query, wk of the hidden state, weights_proj
  of the hidden state in fp32).
* ``layer_norm_bf16``, ``rope_bf16``, ``front`` — the steps before the
  rotation in the ``Indexer.forward`` excerpt: the key LayerNorm (k_norm), and
  the rotary embedding, not interleaved, of the queries and keys (gain and
  bias in fp32, cos / sin tables per token: NKI page, parameters).
* ``e8m0_encode`` / ``e8m0_decode`` — the power-of-two key scale stored as one
  byte, the "e8m0" of the ``fp8_index`` docstring ("Index scores" page).
* ``MASK_BOUND_BF16``, ``scores_bf16`` — the NKI page's Notes: masked slots
  hold a finite bound instead of −inf for consumers that read bfloat16.

Readings taken where the pages are silent:

* H_128 is the Sylvester matrix in natural order, H[i, j] = (−1)^popcount(i & j).
* The rotation runs on the bf16 inputs in float64 as a butterfly with strides
  1, 2, 4, …, 64 (pair (a, b) → (a + b, a − b)), then one float64 multiply by
  the correctly rounded float64 value of 128^(−1/2), then one
  round-to-nearest-even to bf16.  The rotated activation is bf16, as the input.
* amax is floored at fl32(1e-4) so that an all-zero block has a finite scale.
* scale = fl32(amax / 448) (IEEE division); ue8m0 rounds that scale up to the
  next power of two (unchanged when it already is one) and stores it as fp32.
* code = e4m3fn(fl32(x / scale)), round to nearest even, saturating to ±448,
  keeping the sign of zero.
* Query row i of a call with n rows sits at position lengths[b] − n + i; key s
  is visible to it iff s < lengths[b] and, when causal, s ≤ that position.
* The row keeps k_t = min(k, number of visible keys) positions; the oracle
  orders by score descending, then position ascending, and pads with −1.
* e8m0 is the OCP MX scale format: an unsigned biased exponent, value
  2^(byte − 127), no sign or mantissa (0xFF not used).
* The finite mask bound, whose value the NKI page does not give, is the most
  negative finite bfloat16, −(2 − 2^−7) · 2^127 — exact in bf16 and fp32, so
  a bf16 consumer reads it unchanged.
* A bf16 score is the round-to-nearest-even of the fp32 score.
* RoPE turns the leading 64 features ("64 rotary" features of the query
  heads, "Join query parts" page); not interleaved means feature i pairs with
  i + 32.  The angles come in as cos / sin tables (NKI page), so the YaRN
  frequency schedule is outside this step.
* The projections' weights: wq_b and wk bf16 in the Linear layout [out, in]
  (the excerpt calls them as Linear layers and gives no dtype; the NKI page's
  MX-fp8 wq_b is a Trainium packing), weights_proj fp32 (the excerpt casts
  x to fp32 before it).  Outputs rounded once, to bf16 (q, k) and fp32 (w).
* LayerNorm: biased variance, eps added under the square root, all in float64
  with sums taken from feature 0 to 127; its output is bf16 (the activations'
  type), and so is the RoPE output.  eps is an argument (fp32).

Precision: the FP8 dot products are computed exactly in float64 (every product
of two e4m3 values is a multiple of 2^-18 below 2^17.7, so a 128-term sum needs
at most 43 significant bits); the head-weighted sum and key scale are float64.
"""
from __future__ import annotations

import math

import numpy as np

D = 128            # index head dimension (d_h)
H = 64             # index heads
E4M3_MAX = 448.0   # largest finite e4m3fn value
# correctly rounded float64 value of 128^(-1/2) = 2^(-3.5): sqrt is IEEE-exact-rounded
INV_SQRT_D_F64 = math.sqrt(2.0 ** -7)
AMAX_FLOOR_F32 = np.float32(1e-4)

FMT_FP32 = 0
FMT_UE8M0 = 1


# --------------------------------------------------------------------------- e4m3fn
def e4m3_values() -> np.ndarray:
    """The 256 e4m3fn code points as float64 (NaN for 0x7F / 0xFF).

    Format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent
    field 0 holds subnormals m·2^-9; no infinities; S.1111.111 is NaN.
    """
    out = np.empty(256, np.float64)
    for c in range(256):
        sign = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            out[c] = np.nan
        elif e == 0:
            out[c] = sign * m * 2.0 ** -9
        else:
            out[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


_E4M3 = e4m3_values()
_E4M3_POS = _E4M3[:0x7F]          # codes 0x00 … 0x7E, strictly increasing


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return _E4M3[np.asarray(codes, np.uint8)]


def _round_to_quantum(a: np.ndarray, min_normal_exp: int, mant_bits: int) -> np.ndarray:
    """Round non-negative float64 ``a`` to nearest-even on a binary grid with
    ``mant_bits`` fraction bits for normals and a fixed subnormal quantum.
    Scaling by a power of two is exact, so np.rint sees the exact quotient."""
    _, e = np.frexp(a)
    q = np.where(a >= 2.0 ** min_normal_exp, (e - 1) - mant_bits, min_normal_exp - mant_bits)
    return np.ldexp(np.rint(np.ldexp(a, -q)), q)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 → e4m3fn code: round to nearest even, saturate to ±448, keep the
    sign of zero.  Finite inputs only."""
    x = np.asarray(x, np.float32).astype(np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode: finite inputs only")
    mag = np.minimum(_round_to_quantum(np.abs(x), -6, 3), E4M3_MAX)
    code = np.searchsorted(_E4M3_POS, mag).astype(np.uint8)
    if not np.array_equal(_E4M3_POS[code], mag):
        raise AssertionError("e4m3_encode: rounded value is not a code point")
    return code | np.where(np.signbit(x), np.uint8(0x80), np.uint8(0))


# --------------------------------------------------------------------------- bf16
def bf16_round(v: np.ndarray) -> np.ndarray:
    """float64 → nearest-even bf16 value (returned as float64; ±inf on overflow).
    bf16: 8 significant bits, normals down to 2^-126, subnormal quantum 2^-133."""
    v = np.asarray(v, np.float64)
    mag = _round_to_quantum(np.abs(v), -126, 7)
    mag = np.where(mag >= 2.0 ** 128, np.inf, mag)
    return np.copysign(mag, v)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Bits of a float64 array whose values are already bf16-representable."""
    f = np.asarray(v, np.float64).astype(np.float32)
    if not np.array_equal(f.astype(np.float64), np.asarray(v, np.float64), equal_nan=True):
        raise AssertionError("value is not bf16-representable")
    return (f.view(np.uint32) >> 16).astype(np.uint16)


# --------------------------------------------------------------------------- rotation
def hadamard128(x: np.ndarray) -> np.ndarray:
    """y = H_128 · x over the last axis, float64 butterfly with strides 1…64.

    At stride h, element j (bit h clear) pairs with j + h: (a, b) → (a + b, a − b).
    The composition of the seven stages is the Sylvester matrix in natural order.
    """
    y = np.array(x, dtype=np.float64, copy=True)
    lead = y.shape[:-1]
    h = 1
    while h < D:
        y = y.reshape(lead + (D // (2 * h), 2, h))
        a = y[..., 0, :]
        b = y[..., 1, :]
        y = np.stack((a + b, a - b), axis=-2).reshape(lead + (D,))
        h *= 2
    return y


def rotate(x_bf16_bits: np.ndarray) -> np.ndarray:
    """Scaled Hadamard rotation of bf16 rows; returns bf16 bits."""
    x = bf16_bits_to_f64(x_bf16_bits)
    y = hadamard128(x) * INV_SQRT_D_F64
    return f64_to_bf16_bits(bf16_round(y))


# --------------------------------------------------------------------------- quant
def scale_from_amax(amax_f32: np.ndarray, fmt: int) -> np.ndarray:
    amax = np.maximum(np.asarray(amax_f32, np.float32), AMAX_FLOOR_F32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    if fmt == FMT_FP32:
        return s
    if fmt != FMT_UE8M0:
        raise ValueError("fmt must be 0 (fp32) or 1 (ue8m0)")
    bits = s.view(np.uint32)
    up = (bits & np.uint32(0x007FFFFF)) != 0
    rounded = np.where(up, (bits & np.uint32(0xFF800000)) + np.uint32(0x00800000), bits)
    return rounded.astype(np.uint32).view(np.float32)


def quant_rows(x_bf16_bits: np.ndarray, fmt: int):
    """Block-FP8 quantisation of already-rotated bf16 rows (block = 128).
    Returns (codes uint8 [..., 128], scale float32 [...])."""
    x = bf16_bits_to_f64(x_bf16_bits).astype(np.float32)      # exact
    amax = np.max(np.abs(x), axis=-1)
    s = scale_from_amax(amax, fmt)
    y = (x / s[..., None]).astype(np.float32)                  # IEEE fp32 division
    return e4m3_encode(y), s


def rotate_quant(x_bf16_bits: np.ndarray, fmt: int):
    return quant_rows(rotate(x_bf16_bits), fmt)


def quant_append(k_bf16_bits, positions, k_cache, k_scale_cache, fmt):
    """Rotate, quantise and store n new keys per sequence at slots
    positions[b] … positions[b]+n−1 (in place)."""
    k_bf16_bits = np.asarray(k_bf16_bits, np.uint16)
    B, n, _ = k_bf16_bits.shape
    codes, scales = rotate_quant(k_bf16_bits, fmt)
    for b in range(B):
        p = int(positions[b])
        if p < 0 or p + n > k_cache.shape[1]:
            raise ValueError("append past the cache capacity")
        k_cache[b, p:p + n] = codes[b]
        k_scale_cache[b, p:p + n] = scales[b]


# --------------------------------------------------------------------------- weights
INV_SQRT_H_F32 = np.float32(0.125)                 # 64^(-1/2), exact
INV_SQRT_D_F32 = np.float32(INV_SQRT_D_F64)         # fl32(128^(-1/2))


def fold_weights(w_raw: np.ndarray, q_scale: np.ndarray) -> np.ndarray:
    """w = fl32(fl32(fl32(w_raw · 64^-1/2) · q_scale) · fl32(128^-1/2)), elementwise."""
    w = (np.asarray(w_raw, np.float32) * INV_SQRT_H_F32).astype(np.float32)
    w = (w * np.asarray(q_scale, np.float32)).astype(np.float32)
    return (w * INV_SQRT_D_F32).astype(np.float32)


def quant_queries(q_bf16_bits, w_raw, fmt):
    """Queries [.., 64, 128] bf16 → (codes, per-head scale, folded weights)."""
    codes, q_scale = rotate_quant(q_bf16_bits, fmt)
    return codes, q_scale, fold_weights(w_raw, q_scale)


# --------------------------------------------------------------------------- front end
ROPE_DIM = 64      # leading features the rotary embedding turns (the 64 rotary features)


def layer_norm_bf16(k_bf16_bits, gain, bias, eps):
    """Key LayerNorm over the 128 features (Indexer.forward excerpt: the key
    projection goes through k_norm before RoPE; NKI page: fp32 gain and bias).
    float64 throughout: mean = (Σ x, summed from feature 0 to 127) / 128,
    var = (Σ (x − mean)², same order) / 128, y = ((x − mean) / sqrt(var + eps))
    · gain + bias, one rounding per operation, then round to bf16."""
    x = bf16_bits_to_f64(k_bf16_bits)
    mean = np.add.accumulate(x, axis=-1)[..., -1] / D
    d = x - mean[..., None]
    var = np.add.accumulate(d * d, axis=-1)[..., -1] / D
    sd = np.sqrt(var + float(np.float32(eps)))
    g = np.asarray(gain, np.float32).astype(np.float64)
    b = np.asarray(bias, np.float32).astype(np.float64)
    y = (d / sd[..., None]) * g + b
    return f64_to_bf16_bits(bf16_round(y))


def rope_bf16(x_bf16_bits, cos, sin):
    """Rotary embedding of the leading 64 features, not interleaved
    (Indexer.forward excerpt): feature i and feature i + 32 (i < 32) are the
    two coordinates turned by angle θ_i, (a, b) → (a·cos θ_i − b·sin θ_i,
    b·cos θ_i + a·sin θ_i); features 64 … 127 pass unchanged.  cos / sin
    [..., 32] float32 (the NKI page's cos / sin tables, per token, broadcast
    over leading axes).  float64 (the products are exact), then bf16."""
    x = bf16_bits_to_f64(x_bf16_bits)
    c = np.asarray(cos, np.float32).astype(np.float64)
    s = np.asarray(sin, np.float32).astype(np.float64)
    half = ROPE_DIM // 2
    a, b = x[..., :half], x[..., half:ROPE_DIM]
    y = x.copy()
    y[..., :half] = a * c - b * s
    y[..., half:ROPE_DIM] = b * c + a * s
    return f64_to_bf16_bits(bf16_round(y))


def project(x_bits, qr_bits, wq_b_bits, wk_bits, w_proj):
    """The indexer's three projections, the first steps of the Indexer.forward
    excerpt ("Index scores" page): q = wq_b(qr) viewed as [tokens, 64, 128]
    (head-major), k = wk(x), and the head weights weights_proj(x.float()).

    x [T, hidden] and qr [T, q_lora] bf16 bits; wq_b [64·128, q_lora] and
    wk [128, hidden] bf16 bits (Linear layout: [out, in]); w_proj [64, hidden]
    float32.  Each product is a float64 matrix product of the exact inputs
    (every bf16 × bf16 or bf16 × fp32 product is exact in float64, and the
    sums stay within one float64 rounding per term), then ONE rounding: to
    bf16 for q and k (the activations' type), to fp32 for the weights (the
    excerpt's x.float()).  Returns (q [T, 64, 128] bf16 bits, k [T, 128] bf16
    bits, w_raw [T, 64] float32)."""
    x = bf16_bits_to_f64(x_bits)
    qr = bf16_bits_to_f64(qr_bits)
    wq = bf16_bits_to_f64(wq_b_bits)
    wk = bf16_bits_to_f64(wk_bits)
    wp = np.asarray(w_proj, np.float32).astype(np.float64)
    T = x.shape[0]
    q = f64_to_bf16_bits(bf16_round(qr @ wq.T)).reshape(T, H, D)
    k = f64_to_bf16_bits(bf16_round(x @ wk.T))
    w = (x @ wp.T).astype(np.float32)
    return q, k, w


def front(q_proj_bits, k_proj_bits, cos, sin, gain, bias, eps):
    """Query and key rows after the projections, ready for the rotation
    (Indexer.forward excerpt, in its order): q [..., 64, 128] gets RoPE; k
    [..., 128] gets the LayerNorm, then RoPE.  cos / sin [..., 32] per token.
    Returns bf16 bits (q, k)."""
    cos = np.asarray(cos, np.float32)
    sin = np.asarray(sin, np.float32)
    q = rope_bf16(q_proj_bits, cos[..., None, :], sin[..., None, :])
    k = rope_bf16(layer_norm_bf16(k_proj_bits, gain, bias, eps), cos, sin)
    return q, k


# --------------------------------------------------------------------------- scores
def visible_count(length: int, n: int, i: int, causal: bool) -> int:
    """Number of keys query row i (of n) of a sequence with ``length`` keys sees."""
    if not causal:
        return int(length)
    return int(length) - int(n) + int(i) + 1


def index_scores(q_codes, w, k_cache, k_scale_cache, lengths, causal, ncols=None,
                 with_bound=True, rows=None, seqs=None):
    """S[b, i, s] = k_scale[s] · Σ_h w[b,i,h] · max(L, 0),  L = Σ_d q·k exact.

    q_codes [B, n, 64, 128] uint8; w [B, n, 64] float32; k_cache [B, T, 128]
    uint8; k_scale_cache [B, T] float32.  Returns float64 arrays S and E (the
    per-entry bound |k_scale| · Σ_h |w·L|) of shape [B, n, ncols]; masked
    entries of S are −inf and of E are 0.  ``rows`` / ``seqs`` restrict the
    computation to some query rows / sequences (the others stay −inf).
    """
    q_codes = np.asarray(q_codes, np.uint8)
    B, n = q_codes.shape[:2]
    lengths = np.asarray(lengths, np.int64)
    if ncols is None:
        ncols = int(lengths.max()) if B else 0
    S = np.full((B, n, ncols), -np.inf)
    E = np.zeros((B, n, ncols))
    for b in (range(B) if seqs is None else seqs):
        L_b = int(lengths[b])
        if L_b == 0:
            continue
        kd = e4m3_decode(k_cache[b, :L_b])                       # [L_b, 128]
        ks = np.asarray(k_scale_cache[b, :L_b], np.float64)
        for i in (range(n) if rows is None else rows):
            v = min(visible_count(L_b, n, i, causal), ncols)
            if v <= 0:
                continue
            qd = e4m3_decode(q_codes[b, i])                      # [64, 128]
            logits = qd @ kd[:v].T                               # [64, v], exact
            wi = np.asarray(w[b, i], np.float64)[:, None]
            S[b, i, :v] = ks[:v] * np.sum(wi * np.maximum(logits, 0.0), axis=0)
            if with_bound:
                E[b, i, :v] = np.abs(ks[:v]) * np.sum(np.abs(wi * logits), axis=0)
    return S, E


def index_scores_rows(q_codes, w, k_codes, k_scale, vis):
    """S and E of several query rows of one sequence, as ``index_scores``
    defines them, with library matrix products as the steps: the logits of all
    rows against the first max(vis) keys as one product (exact: every FP8
    product and partial sum is a multiple of 2^-18 below 2^53), then the
    head-weighted ReLU sum and the bound as batched products over the heads
    (float64; only the summation order over the 64 heads differs from
    ``index_scores``).

    q_codes [R, 64, 128] uint8; w [R, 64] float32; k_codes [>= max(vis), 128]
    uint8 and k_scale [>= max(vis)] float32 of the sequence; vis [R] visible key
    counts.  Returns S, E [R, max(vis)] float64, −inf / 0 from each row's
    visible count on."""
    vis = np.asarray(vis, np.int64)
    R, V = len(vis), int(vis.max()) if len(vis) else 0
    S = np.full((R, V), -np.inf)
    E = np.zeros((R, V))
    if V == 0:
        return S, E
    kd = e4m3_decode(k_codes[:V])                                   # [V, 128]
    ks = np.asarray(k_scale[:V], np.float64)
    qd = e4m3_decode(np.asarray(q_codes, np.uint8)).reshape(R * H, D)
    logits = (qd @ kd.T).reshape(R, H, V)                           # exact
    wi = np.asarray(w, np.float64)[:, None, :]                      # [R, 1, 64]
    S[:] = (wi @ np.maximum(logits, 0.0))[:, 0, :] * ks
    E[:] = (np.abs(wi) @ np.abs(logits))[:, 0, :] * np.abs(ks)
    cols = np.arange(V)[None, :]
    past = cols >= vis[:, None]
    S[past] = -np.inf
    E[past] = 0.0
    return S, E


# --------------------------------------------------------------------------- variants
# e8m0 (OCP MX scale format): one byte, value 2^(byte − 127).
def e8m0_encode(scale: np.ndarray) -> np.ndarray:
    """Byte of a positive power-of-two scale in [2^-127, 2^127]; raises otherwise."""
    s = np.asarray(scale, np.float64)
    m, e = np.frexp(s)                 # s = m · 2^e with m in [0.5, 1)
    if np.any(s <= 0) or np.any(m != 0.5):
        raise AssertionError("e8m0 holds positive powers of two only")
    k = e - 1                          # s = 2^k
    if np.any(k < -127) or np.any(k > 127):
        raise AssertionError("exponent out of the e8m0 range")
    return (k + 127).astype(np.uint8)


def e8m0_decode(byte: np.ndarray) -> np.ndarray:
    return np.ldexp(1.0, np.asarray(byte, np.int64) - 127)


# The finite mask bound: the most negative finite bfloat16.
MASK_BOUND_BF16 = -(2.0 - 2.0 ** -7) * 2.0 ** 127


def masked(S: np.ndarray, bound: float) -> np.ndarray:
    """S with its masked (−inf) entries replaced by a finite bound."""
    return np.where(np.isneginf(S), bound, S)


def scores_bf16(S_f32: np.ndarray) -> np.ndarray:
    """bf16 output of fp32 scores: round to nearest even (values as float64)."""
    return bf16_round(np.asarray(S_f32, np.float32).astype(np.float64))


# --------------------------------------------------------------------------- top-k
def topk_row(scores_row: np.ndarray, visible: int, k: int) -> np.ndarray:
    """The min(k, visible) best positions of one row (score desc, then position
    asc), padded with −1 to length k; int32."""
    out = np.full(k, -1, np.int32)
    kt = min(k, visible)
    if kt <= 0:
        return out
    s = np.asarray(scores_row[:visible], np.float64)
    pos = np.arange(visible)
    order = np.lexsort((pos, -s))
    out[:kt] = order[:kt]
    return out


def topk(S: np.ndarray, lengths, causal: bool, k: int) -> np.ndarray:
    B, n = S.shape[:2]
    out = np.full((B, n, k), -1, np.int32)
    for b in range(B):
        for i in range(n):
            v = min(visible_count(int(lengths[b]), n, i, causal), S.shape[2])
            out[b, i] = topk_row(S[b, i], v, k)
    return out


# --------------------------------------------------------------------------- one step
def indexer_step(state, k_new_bf16, q_bf16, w_raw, positions, causal, k, fmt):
    """One indexer call as the reference forward orders it: append the new keys,
    then score every query against all cached keys so far, then select.

    ``state`` = dict(k_cache=[B,T,128] uint8, k_scale_cache=[B,T] float32),
    modified in place.  Returns (indices, S, E, q_codes, w)."""
    k_new_bf16 = np.asarray(k_new_bf16, np.uint16)
    B, n = k_new_bf16.shape[:2]
    quant_append(k_new_bf16, positions, state["k_cache"], state["k_scale_cache"], fmt)
    lengths = np.asarray(positions, np.int64) + n
    q_codes, _, w = quant_queries(q_bf16, w_raw, fmt)
    S, E = index_scores(q_codes, w, state["k_cache"], state["k_scale_cache"], lengths, causal)
    return topk(S, lengths, causal, k), S, E, q_codes, w
