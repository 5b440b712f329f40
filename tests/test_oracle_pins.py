"""Pins for the CPU oracle: each check ties it to something other than itself —
the FP8/bf16 format definitions worked out in exact rationals, library routines
(scipy's Hadamard matrix, torch's float8 codec, numpy sorting), closed forms,
invariants the pages state (orthonormal rotation, ReLU / weight linearity),
and brute force on tiny inputs.  CPU only."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- helpers
def frac_round(x: Fraction, mant_bits: int, min_exp: int, max_finite: Fraction | None,
               satfinite: bool) -> Fraction | float:
    """Exact round-to-nearest-even of a rational onto a binary float grid."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix floating log error
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = (e - mant_bits) if e >= min_exp else (min_exp - mant_bits)
    quantum = Fraction(2) ** q
    t = a / quantum
    fl = t.numerator // t.denominator
    rem = t - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    if max_finite is not None and r > max_finite:
        if satfinite:
            r = max_finite
        else:
            return sign * math.inf
    return sign * r


def bf16_exact(x: Fraction):
    return frac_round(x, 7, -126, Fraction(2) ** 128 - Fraction(2) ** 119, satfinite=False)


def fp32_exact(x: Fraction):
    return frac_round(x, 23, -126, Fraction(2) ** 128 - Fraction(2) ** 104, satfinite=False)


def e4m3_exact(x: Fraction):
    return frac_round(x, 3, -6, Fraction(448), satfinite=True)


# --------------------------------------------------------------------------- e4m3 codec
def test_e4m3_table_format_points():
    v = O.e4m3_values()
    assert v[0x00] == 0.0 and not np.signbit(v[0x00])
    assert v[0x80] == 0.0 and np.signbit(v[0x80])
    assert v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x08] == 2.0 ** -6
    assert v[0x38] == 1.0 and v[0xB8] == -1.0
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.count_nonzero(np.isfinite(v)) == 254
    assert np.all(np.diff(v[:0x7F]) > 0)


def test_e4m3_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    v = O.e4m3_values()
    fin = np.isfinite(v)
    assert np.array_equal(np.isnan(ref), ~fin)
    assert np.array_equal(ref[fin], v[fin])
    assert np.array_equal(np.signbit(ref[fin]), np.signbit(v[fin]))


def test_e4m3_roundtrip_all_finite_codes():
    v = O.e4m3_values()
    codes = np.array([c for c in range(256) if np.isfinite(v[c])], np.uint8)
    back = O.e4m3_encode(v[codes].astype(np.float32))
    assert np.array_equal(back, codes)


def test_e4m3_encode_exact_rational_rounding():
    rng = np.random.default_rng(7)
    xs = list(rng.standard_normal(3000).astype(np.float32) * np.float32(60))
    xs += list((rng.standard_normal(1000) * 2.0 ** -8).astype(np.float32))   # subnormal range
    # midpoints between neighbouring codes and their fp32 neighbours (ties and near-ties)
    v = O.e4m3_values()[:0x7F]
    mids = (v[:-1] + v[1:]) / 2
    for m in mids:
        m32 = np.float32(m)
        xs += [m32, np.nextafter(m32, np.float32(0)), np.nextafter(m32, np.float32(1000))]
    xs += [np.float32(448), np.float32(449), np.float32(464), np.float32(465), np.float32(1e9)]
    xs = np.array(xs, np.float32)
    xs = np.concatenate([xs, -xs])
    got = O.e4m3_encode(xs)
    dec = O.e4m3_values()
    for x, c in zip(xs, got):
        want = e4m3_exact(Fraction(float(x)))
        assert Fraction(float(dec[c])) == want, (x, c)
        assert bool(c & 0x80) == bool(np.signbit(x))


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(200000) * 50).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), ref)


def test_e4m3_negative_zero_kept():
    got = O.e4m3_encode(np.array([-0.0, -1e-6, 0.0, 1e-6], np.float32))
    assert list(got) == [0x80, 0x80, 0x00, 0x00]


# --------------------------------------------------------------------------- bf16
def test_bf16_round_matches_exact_rationals():
    rng = np.random.default_rng(3)
    vals = list(rng.standard_normal(2000) * 10.0 ** rng.integers(-40, 38, 2000))
    # exact ties: bf16 value + half quantum
    for _ in range(300):
        m = int(rng.integers(128, 256))
        e = int(rng.integers(-120, 120))
        vals.append((m + 0.5) * 2.0 ** e)
        vals.append(-(m + 0.5) * 2.0 ** e)
    vals += [2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 1e-45, 2.0 ** -126 * 0.75,
             3.3895313892515355e38, 3.39e38, 3.4e38, 0.0, -0.0]
    vals = np.array(vals, np.float64)
    got = O.bf16_round(vals)
    for x, g in zip(vals, got):
        want = bf16_exact(Fraction(float(x)))
        if isinstance(want, float):
            assert g == want, x
        else:
            assert Fraction(float(g)) == want, x


def test_bf16_bits_roundtrip():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_bits_to_f64(bits)
    fin = np.isfinite(vals)
    assert np.array_equal(O.f64_to_bf16_bits(vals[fin]), bits[fin])


# --------------------------------------------------------------------------- rotation
def test_hadamard_matches_scipy_sylvester():
    Hs = scipy.linalg.hadamard(128).astype(np.float64)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((50, 128))
    assert np.allclose(O.hadamard128(x), x @ Hs.T, rtol=0, atol=1e-12)
    assert np.array_equal(O.hadamard128(np.eye(128)), Hs)   # H(e_i) = column i


def test_hadamard_orthogonality_and_energy():
    Hm = O.hadamard128(np.eye(128))
    assert np.array_equal(Hm @ Hm.T, 128 * np.eye(128))
    rng = np.random.default_rng(6)
    x = rng.standard_normal((20, 128))
    y = O.hadamard128(x)
    assert np.allclose((y ** 2).sum(-1), 128 * (x ** 2).sum(-1), rtol=1e-13)


def test_scaled_rotation_preserves_query_key_products():
    # The rotation is orthonormal, so q·k is unchanged before quantisation.
    rng = np.random.default_rng(8)
    q = rng.standard_normal((64, 128))
    k = rng.standard_normal((300, 128))
    qr = O.hadamard128(q) * O.INV_SQRT_D_F64
    kr = O.hadamard128(k) * O.INV_SQRT_D_F64
    assert np.allclose(qr @ kr.T, q @ k.T, rtol=0, atol=1e-12 * np.abs(q).sum() / 64)


def test_rotation_constant_is_correctly_rounded():
    c = Fraction(O.INV_SQRT_D_F64)
    # c is the float64 nearest to 2^-3.5: |c^2 - 2^-7| minimal among neighbours
    lo = Fraction(math.nextafter(O.INV_SQRT_D_F64, 0))
    hi = Fraction(math.nextafter(O.INV_SQRT_D_F64, 1))
    target = Fraction(1, 128)
    err = lambda t: abs(t * t - target)
    assert err(c) < err(lo) and err(c) < err(hi)


def test_rotate_equals_exact_signed_sums_then_two_roundings():
    rng = np.random.default_rng(9)
    raw = (rng.standard_normal((40, 128)) * np.where(rng.random(128) < 0.02, 20, 1)).astype(np.float32)
    bits = synth._to_bf16_bits(raw)
    x = O.bf16_bits_to_f64(bits)
    got = O.bf16_bits_to_f64(O.rotate(bits))
    Hs = scipy.linalg.hadamard(128)
    c = Fraction(O.INV_SQRT_D_F64)
    for r in range(x.shape[0]):
        xs = [Fraction(float(v)) for v in x[r]]
        for i in range(128):
            y = sum(xs[j] if Hs[i, j] > 0 else -xs[j] for j in range(128))
            p = Fraction(float(y * c))                # the float64 product (correctly rounded)
            want = bf16_exact(p)
            assert Fraction(float(got[r, i])) == want


def _bf16_rne_bits(p: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of float64 values onto bf16 (normal range only),
    done on the IEEE-754 bit pattern: keep the sign, exponent and top 7
    fraction bits, round on the 45 dropped bits (ties to an even kept field)."""
    u = np.ascontiguousarray(p, np.float64).view(np.uint64)
    drop = np.uint64(45)
    half = np.uint64(1) << np.uint64(44)
    odd = (u >> drop) & np.uint64(1)
    r = (u + (half - np.uint64(1)) + odd) & ~((np.uint64(1) << drop) - np.uint64(1))
    return r.view(np.float64)


def test_rotate_rounds_once_from_float64_on_many_rows():
    """The rotation's reading is one float64 multiply of the exact butterfly sum,
    then ONE round-to-nearest-even to bf16.  A plausible slip is an fp32
    intermediate (round to fp32, then to bf16): it differs only where the fp32
    value lands exactly on a bf16 midpoint, about one row in a thousand.  This
    pin checks 2·10^5 rows of the workloads' distribution against sums taken
    independently of the butterfly (scipy's Hadamard matrix as a BLAS product,
    exact because every partial sum is a multiple of the row's smallest bf16
    quantum below 2^53) and a bit-level rounding, and requires that the rows
    hold enough double-rounding witnesses for the slip to fail it."""
    rng = np.random.default_rng(31)
    rows = 200_000
    raw = rng.standard_normal((rows, 128)).astype(np.float32)
    ch = rng.choice(128, size=2, replace=False)
    raw[:, ch] *= 20
    bits = synth._to_bf16_bits(raw)
    x = O.bf16_bits_to_f64(bits)
    # exactness of the float64 sums: exponent span of each row's nonzero values
    _, e = np.frexp(np.where(x == 0, 1.0, np.abs(x)))
    span = np.where(x == 0, e.min(), e).max(-1) - np.where(x == 0, e.max(), e).min(-1)
    assert span.max() <= 38
    y = x @ scipy.linalg.hadamard(128).astype(np.float64).T
    p = y * O.INV_SQRT_D_F64                       # one IEEE float64 multiply
    want = _bf16_rne_bits(p)
    got = O.bf16_bits_to_f64(O.rotate(bits))
    np.testing.assert_array_equal(got, want)
    # the same check on the fp32 route would fail here: count its witnesses
    f32 = p.astype(np.float32).astype(np.float64)
    double = _bf16_rne_bits(f32)
    witness_rows = np.unique(np.nonzero(double != want)[0])
    assert witness_rows.size >= 50, witness_rows.size
    # and those rows again in exact rationals (Fraction sums, exact rounding)
    Hs = scipy.linalg.hadamard(128)
    c = Fraction(O.INV_SQRT_D_F64)
    for r in witness_rows[:8]:
        cols = np.nonzero(double[r] != want[r])[0]
        xs = [Fraction(float(v)) for v in x[r]]
        for i in cols:
            ysum = sum(xs[j] if Hs[i, j] > 0 else -xs[j] for j in range(128))
            assert Fraction(float(got[r, i])) == bf16_exact(Fraction(float(ysum * c)))


# --------------------------------------------------------------------------- quant
def _rows(seed, n=200):
    rng = np.random.default_rng(seed)
    raw = rng.standard_normal((n, 128)).astype(np.float32)
    raw[:, [3, 77]] *= 20
    return synth._to_bf16_bits(raw)


def test_quant_fp32_amax_maps_to_448():
    bits = _rows(12)
    codes, s = O.quant_rows(bits, O.FMT_FP32)
    x = O.bf16_bits_to_f64(bits)
    am = np.argmax(np.abs(x), axis=-1)
    c = codes[np.arange(len(am)), am]
    assert np.all((c & 0x7F) == 0x7E)
    amax = np.abs(x).max(-1).astype(np.float32)
    assert np.array_equal(s, (amax / np.float32(448)).astype(np.float32))


def test_quant_ue8m0_power_of_two_scales():
    bits = _rows(13)
    codes, s = O.quant_rows(bits, O.FMT_UE8M0)
    assert np.all((s.view(np.uint32) & 0x7FFFFF) == 0)
    amax = np.abs(O.bf16_bits_to_f64(bits)).max(-1)
    ratio = amax / s.astype(np.float64)
    assert np.all(ratio > 224) and np.all(ratio <= 448)


def test_quant_codes_are_nearest_to_scaled_values():
    bits = _rows(14, 50)
    for fmt in (O.FMT_FP32, O.FMT_UE8M0):
        codes, s = O.quant_rows(bits, fmt)
        x = O.bf16_bits_to_f64(bits).astype(np.float32)
        dec = O.e4m3_values()
        for r in range(x.shape[0]):
            for j in range(128):
                y = fp32_exact(Fraction(float(x[r, j])) / Fraction(float(s[r])))  # IEEE quotient
                assert Fraction(float(dec[codes[r, j]])) == e4m3_exact(y)


def test_quant_divides_rather_than_multiplying_by_a_reciprocal():
    # amax 3.0625 gives s = fl32(3.0625/448); for x = 1.3671875 the IEEE quotient
    # and x·fl32(1/s) land on different sides of an e4m3 rounding midpoint.
    row = np.zeros((1, 128), np.float32)
    row[0, 0], row[0, 1] = 3.0625, 1.3671875
    codes, s = O.quant_rows(synth._to_bf16_bits(row), O.FMT_FP32)
    want = e4m3_exact(fp32_exact(Fraction(1.3671875) / Fraction(float(s[0]))))
    assert Fraction(float(O.e4m3_values()[codes[0, 1]])) == want
    assert codes[0, 1] == 0x74


def test_quant_relative_error_bound():
    bits = _rows(15)
    codes, s = O.quant_rows(bits, O.FMT_FP32)
    x = O.bf16_bits_to_f64(bits)
    deq = O.e4m3_decode(codes) * s[:, None].astype(np.float64)
    normal = np.abs(O.e4m3_decode(codes)) >= 2.0 ** -6
    err = np.abs(x - deq)
    bound = s[:, None] * (2.0 ** -4 * np.abs(O.e4m3_decode(codes)) * 1.0001 + 1e-12)
    assert np.all(err[normal] <= bound[normal])


def test_quant_zero_row():
    codes, s = O.quant_rows(np.zeros((1, 128), np.uint16), O.FMT_FP32)
    assert np.all(codes == 0)
    assert s[0] == np.float32(np.float32(1e-4) / np.float32(448))


# --------------------------------------------------------------------------- scores
def brute_scores(qc, w, kc, ks, lengths, causal):
    """Exact rational scores for tiny shapes, straight from the score equation."""
    dec = O.e4m3_values()
    B, n, Hh, d = qc.shape
    out = {}
    for b in range(B):
        for i in range(n):
            vis = O.visible_count(int(lengths[b]), n, i, causal)
            for s in range(vis):
                tot = Fraction(0)
                for h in range(Hh):
                    L = sum(Fraction(float(dec[qc[b, i, h, j]])) * Fraction(float(dec[kc[b, s, j]]))
                            for j in range(d))
                    tot += Fraction(float(w[b, i, h])) * max(L, Fraction(0))
                out[(b, i, s)] = Fraction(float(ks[b, s])) * tot
    return out


@pytest.mark.parametrize("Hh,d,causal", [(1, 1, False), (2, 2, True), (2, 4, False), (1, 4, True)])
def test_scores_exact_rational_brute_force(Hh, d, causal):
    rng = np.random.default_rng(100 + Hh * 10 + d)
    B, n, T = 2, 3, 7
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    qc = rng.choice(finite, (B, n, Hh, d))
    kc = rng.choice(finite, (B, T, d))
    w = rng.standard_normal((B, n, Hh)).astype(np.float32)
    ks = (rng.random((B, T)) + 0.1).astype(np.float32)
    lengths = np.array([7, 5])
    S, E = O.index_scores(qc, w, kc, ks, lengths, causal, ncols=T)
    ex = brute_scores(qc, w, kc, ks, lengths, causal)
    for b in range(B):
        for i in range(n):
            vis = O.visible_count(int(lengths[b]), n, i, causal)
            for s in range(T):
                if s < vis:
                    assert abs(Fraction(S[b, i, s]) - ex[(b, i, s)]) <= Fraction(1e-14) * Fraction(E[b, i, s]) + Fraction(1e-300)
                else:
                    assert S[b, i, s] == -np.inf


def test_fp8_dot_is_exact_in_float64():
    dec = O.e4m3_values()
    rng = np.random.default_rng(21)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    for trial in range(30):
        a = rng.choice(finite, 128)
        b = rng.choice(finite, 128)
        if trial == 0:
            a[:] = 0x7E
            b[:] = 0x7E
        if trial == 1:
            a[:64] = 0x7E; a[64:] = 0x01; b[:] = 0x81
        got = float(dec[a] @ dec[b])
        exact = sum(Fraction(float(dec[x])) * Fraction(float(dec[y])) for x, y in zip(a, b))
        assert Fraction(got) == exact


def _rand_case(seed, B=2, n=2, T=40, lengths=(40, 23), causal=False):
    rng = np.random.default_rng(seed)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    qc = rng.choice(finite, (B, n, 64, 128))
    kc = rng.choice(finite, (B, T, 128))
    w = rng.standard_normal((B, n, 64)).astype(np.float32)
    ks = (rng.random((B, T)) * 0.01 + 1e-3).astype(np.float32)
    return qc, w, kc, ks, np.array(lengths), causal


def test_scores_one_hot_weight_is_single_head_relu_dot():
    qc, w, kc, ks, lengths, causal = _rand_case(31)
    w[:] = 0
    w[..., 17] = 2.5
    S, _ = O.index_scores(qc, w, kc, ks, lengths, causal, ncols=40)
    dec = O.e4m3_values()
    for b in range(2):
        for i in range(2):
            L = dec[kc[b, :lengths[b]]] @ dec[qc[b, i, 17]]
            want = ks[b, :lengths[b]].astype(np.float64) * 2.5 * np.maximum(L, 0)
            assert np.array_equal(S[b, i, :lengths[b]], want)


def test_scores_odd_in_weights_and_linear_when_logits_positive():
    qc, w, kc, ks, lengths, causal = _rand_case(32)
    S1, E = O.index_scores(qc, w, kc, ks, lengths, causal, ncols=40)
    S2, _ = O.index_scores(qc, -w, kc, ks, lengths, causal, ncols=40)
    m = np.isfinite(S1)
    assert np.array_equal(S1[m], -S2[m])
    # with non-negative codes only, every logit is >= 0 and S is linear in w
    qp = qc & 0x7F
    kp = kc & 0x7F
    wa = w
    wb = np.random.default_rng(33).standard_normal(w.shape).astype(np.float32)
    Sa, Ea = O.index_scores(qp, wa, kp, ks, lengths, causal, ncols=40)
    Sb, Eb = O.index_scores(qp, wb, kp, ks, lengths, causal, ncols=40)
    Sab, _ = O.index_scores(qp, (wa.astype(np.float64) + wb).astype(np.float32), kp, ks, lengths, causal, ncols=40)
    m = np.isfinite(Sa)
    tol = 1e-6 * (Ea + Eb)[m] + 1e-30
    assert np.all(np.abs(Sab[m] - (Sa[m] + Sb[m])) <= tol)


def test_batched_row_scores_equal_the_per_row_definition():
    """index_scores_rows (matrix products over all rows and heads) against
    index_scores (one row at a time): the logits are exact in both, so only
    the float64 order of the 64-term head sums may differ."""
    case = synth.make_case("rows", 91, 2, 37, [300, 45], T_cap=512, causal=True, fmt=1)
    kc, ks = np.zeros((2, 512, 128), np.uint8), np.zeros((2, 512), np.float32)
    for b in range(2):
        p = int(case.positions[b])
        O.quant_append(case.k_prior[b:b + 1, :p], [0], kc[b:b + 1], ks[b:b + 1], 1)
    O.quant_append(case.k_new, case.positions, kc, ks, 1)
    qc, _, w = O.quant_queries(case.q, case.w_raw, 1)
    for causal in (True, False):
        S, E = O.index_scores(qc, w, kc, ks, case.lengths, causal, ncols=int(case.lengths.max()))
        for b in range(2):
            L = int(case.lengths[b])
            vis = [O.visible_count(L, 37, i, causal) for i in range(37)]
            S2, E2 = O.index_scores_rows(qc[b], w[b], kc[b], ks[b], vis)
            V = max(vis)
            assert np.array_equal(np.isneginf(S2), np.isneginf(S[b, :, :V]))
            fin = ~np.isneginf(S2)
            assert np.all(np.abs(S2[fin] - S[b, :, :V][fin]) <= 1e-13 * E[b, :, :V][fin])
            assert np.allclose(E2, E[b, :, :V], rtol=1e-13, atol=0)


def test_causal_visibility_rule():
    qc, w, kc, ks, _, _ = _rand_case(34, B=1, n=4, T=10, lengths=(10,))
    S, _ = O.index_scores(qc, w, kc, ks, np.array([10]), True, ncols=10)
    for i in range(4):
        vis = 10 - 4 + i + 1
        assert np.all(np.isfinite(S[0, i, :vis])) and np.all(S[0, i, vis:] == -np.inf)


def test_decode_example_scores_all_cached_keys_including_new():
    g = json.load(open(os.path.join(GOLDEN, "pages_shapes.json")))["decode_example"]
    p = g["start_pos"]
    case = synth.make_case("p1000", 77, 1, 1, [p], T_cap=2048)
    st = {"k_cache": np.zeros((1, 2048, 128), np.uint8), "k_scale_cache": np.zeros((1, 2048), np.float32)}
    O.quant_append(case.k_prior, [0], st["k_cache"], st["k_scale_cache"], 0)
    idx, S, E, _, _ = O.indexer_step(st, case.k_new, case.q, case.w_raw, case.positions, False, 2048, 0)
    assert S.shape == (1, g["query_rows"], g["scored_keys"])
    assert np.all(np.isfinite(S))
    # the key written by this very call is among those scored
    assert np.array_equal(st["k_cache"][0, p], O.rotate_quant(case.k_new[0, 0], 0)[0])
    assert sorted(idx[0, 0][idx[0, 0] >= 0]) == list(range(g["scored_keys"]))


# --------------------------------------------------------------------------- top-k
def test_topk_matches_numpy_stable_sort_and_torch():
    rng = np.random.default_rng(41)
    s = np.round(rng.standard_normal(5000), 2)      # many exact ties
    k = 700
    got = O.topk_row(s, 5000, k)
    ref = np.argsort(-s, kind="stable")[:k]
    assert np.array_equal(got, ref)
    tv, _ = torch.topk(torch.from_numpy(s), k)
    assert np.array_equal(np.sort(s[got])[::-1], tv.numpy())


def test_topk_short_rows_take_everything_and_pad():
    s = np.array([3.0, -1.0, 2.0, -np.inf, -np.inf])
    got = O.topk_row(s, 3, 5)
    assert list(got) == [0, 2, 1, -1, -1]
    assert list(O.topk_row(s, 0, 3)) == [-1, -1, -1]


def test_cache_layout_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "pages_shapes.json")))["cache"]
    assert synth.T_CAP == g["slots_per_sequence"]
    assert O.D == g["head_dim"] == g["block_size"] * g["scales_per_key"]


def test_folded_weights_reproduce_the_unfolded_score_equation():
    """The score equation carries 1/(sqrt(64)·sqrt(128)) explicitly and uses the
    dequantised rotated query and key; folding those factors and the query scale
    into w (and applying the key scale after the head sum) must give the same
    score up to the fold's three fp32 roundings."""
    case = synth.make_case("fold", 55, 2, 3, [37, 12], T_cap=64, fmt=0)
    for fmt in (0, 1):
        st = {"k_cache": np.zeros((2, 64, 128), np.uint8), "k_scale_cache": np.zeros((2, 64), np.float32)}
        for b in range(2):
            p = int(case.positions[b])
            O.quant_append(case.k_prior[b:b + 1, :p], [0], st["k_cache"][b:b + 1], st["k_scale_cache"][b:b + 1], fmt)
        idx, S, E, qc, w = O.indexer_step(st, case.k_new, case.q, case.w_raw, case.positions, True, 16, fmt)
        _, q_scale = O.rotate_quant(case.q, fmt)
        lengths = case.lengths
        for b in range(2):
            kbar = O.e4m3_decode(st["k_cache"][b, :lengths[b]]) * st["k_scale_cache"][b, :lengths[b], None].astype(np.float64)
            for i in range(3):
                qbar = O.e4m3_decode(qc[b, i]) * q_scale[b, i, :, None].astype(np.float64)
                vis = lengths[b] - 3 + i + 1
                page = (1.0 / (math.sqrt(64) * math.sqrt(128))) * (
                    case.w_raw[b, i].astype(np.float64)[:, None] * np.maximum(qbar @ kbar[:vis].T, 0)).sum(0)
                assert np.all(np.abs(S[b, i, :vis] - page) <= 4e-7 * E[b, i, :vis] + 1e-30)


def test_folded_weights_equal_the_page_expression_in_torch_fp32():
    """Bit for bit against the Indexer.forward excerpt ("Index scores" page,
    the two weight lines) evaluated by torch on the CPU in fp32: the weight
    projection times 64^-0.5, then times the query scale, then times the
    softmax scale 128^-0.5, each product rounded to fp32.  A reordered fold
    or a constant one ulp off fails here."""
    rng = np.random.default_rng(77)
    w_raw = rng.standard_normal((512, 64)).astype(np.float32)
    q_bits = synth._to_bf16_bits(rng.standard_normal((512, 64, 128)).astype(np.float32) *
                                 np.exp(rng.uniform(-6, 6, (512, 64, 1))).astype(np.float32))
    for fmt in (0, 1):
        _, q_scale, w = O.quant_queries(q_bits, w_raw, fmt)
        n_heads, head_dim = 64, 128
        wt = torch.from_numpy(w_raw) * n_heads ** -0.5
        wt = wt.unsqueeze(-1) * torch.from_numpy(q_scale).unsqueeze(-1) * head_dim ** -0.5
        np.testing.assert_array_equal(w.view(np.uint32), wt.squeeze(-1).numpy().view(np.uint32))


def test_append_writes_exactly_the_requested_slots():
    case = synth.make_case("app", 56, 3, 4, [0, 9, 28], T_cap=32, fmt=1)
    kc = np.full((3, 32, 128), 0xAB, np.uint8)
    ks = np.full((3, 32), -7.0, np.float32)
    O.quant_append(case.k_new, case.positions, kc, ks, 1)
    for b in range(3):
        p = int(case.positions[b])
        c, s = O.rotate_quant(case.k_new[b], 1)
        assert np.array_equal(kc[b, p:p + 4], c) and np.array_equal(ks[b, p:p + 4], s)
        mask = np.ones(32, bool); mask[p:p + 4] = False
        assert np.all(kc[b, mask] == 0xAB) and np.all(ks[b, mask] == -7.0)
    with pytest.raises(ValueError):
        O.quant_append(case.k_new, [0, 0, 29], kc, ks, 1)


# ---------------------------------------------------------------- variants
def test_e8m0_byte_is_the_ieee_exponent_field():
    """The e8m0 byte of 2^k is the biased exponent field of the fp32 value 2^k
    (IEEE 754 binary32: bits 30…23, bias 127), for every normal power of two."""
    ks = np.arange(-126, 128)
    vals = np.ldexp(1.0, ks)
    field = (vals.astype(np.float32).view(np.uint32) >> 23) & 0xFF
    assert np.array_equal(O.e8m0_encode(vals), field.astype(np.uint8))
    assert np.array_equal(O.e8m0_decode(field), vals)
    assert O.e8m0_encode(np.array([1.0]))[0] == 127


def test_e8m0_round_trips_every_ue8m0_scale_and_rejects_others():
    rng = np.random.default_rng(5)
    amax = np.abs(rng.standard_normal(5000)).astype(np.float32) * np.float32(100)
    amax[:3] = [0.0, 448.0, 3e-5]
    s = O.scale_from_amax(amax, 1)
    assert np.array_equal(O.e8m0_decode(O.e8m0_encode(s)), s.astype(np.float64))
    for bad in (3.0, 0.75, -2.0, 0.0):
        with pytest.raises(AssertionError):
            O.e8m0_encode(np.array([bad]))


def test_mask_bound_is_the_most_negative_finite_bf16():
    import torch
    assert O.MASK_BOUND_BF16 == float(torch.finfo(torch.bfloat16).min)
    assert O.bf16_round(np.array([O.MASK_BOUND_BF16]))[0] == O.MASK_BOUND_BF16
    assert float(np.float32(O.MASK_BOUND_BF16)) == O.MASK_BOUND_BF16
    S = np.array([[1.5, -np.inf, -3.0, -np.inf]])
    assert np.array_equal(O.masked(S, O.MASK_BOUND_BF16), [[1.5, O.MASK_BOUND_BF16, -3.0, O.MASK_BOUND_BF16]])


def test_bf16_scores_match_torch_rounding():
    """Round-to-nearest-even fp32 → bf16, against torch's conversion (ties,
    values next to the rounding boundary, subnormals, large magnitudes)."""
    import torch
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-40, 40, 20000))).astype(np.float32)
    u = rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32)
    u = (u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)          # exact ties
    ties = u.view(np.float32)
    ties = ties[np.isfinite(ties)]
    x = np.concatenate([x, ties, np.float32([1e-40, -3e-39, 3.3e38, -3.39e38])])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.scores_bf16(x)
    fin = np.isfinite(want)
    assert np.array_equal(got[fin], want[fin])


# --------------------------------------------------------------------------- front end
def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_vals(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def test_rope_pairs_feature_i_with_i_plus_32():
    """Non-interleaved pairing: a lone feature i < 32 moves only into i and
    i + 32 (an interleaved or shifted pairing would light other slots)."""
    th = np.linspace(0.1, 1.5, 32).astype(np.float32)
    c, s = np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    for i in [0, 3, 31]:
        x = np.zeros(128, np.float32)
        x[i] = 1.0
        y = _bf16_vals(O.rope_bf16(_bf16_bits(x), c, s))
        assert set(np.flatnonzero(y)) == {i, i + 32}
        assert y[i] == _bf16_vals(_bf16_bits([c[i]]))[0] and y[i + 32] == _bf16_vals(_bf16_bits([s[i]]))[0]
        x = np.zeros(128, np.float32)
        x[i + 32] = 1.0
        y = _bf16_vals(O.rope_bf16(_bf16_bits(x), c, s))
        assert set(np.flatnonzero(y)) == {i, i + 32}
        assert y[i] == -_bf16_vals(_bf16_bits([s[i]]))[0]
    x = np.zeros(128, np.float32)
    x[64:] = np.arange(64) + 1
    assert np.array_equal(O.rope_bf16(_bf16_bits(x), c, s), _bf16_bits(x))   # features 64 … 127 untouched


def test_rope_special_angles_and_inverse():
    rng = np.random.default_rng(4)
    x = _bf16_bits(rng.standard_normal((6, 128)))
    one, zero = np.ones(32, np.float32), np.zeros(32, np.float32)
    assert np.array_equal(O.rope_bf16(x, one, zero), x)                   # θ = 0
    v = _bf16_vals(x)
    y = _bf16_vals(O.rope_bf16(x, zero, one))                            # θ = π/2: (a, b) → (−b, a)
    assert np.array_equal(y[:, :32], -v[:, 32:64]) and np.array_equal(y[:, 32:64], v[:, :32])
    # turning by θ and back stays within two bf16 roundings of the input
    th = rng.uniform(-3, 3, 32)
    f = O.rope_bf16(x, np.cos(th).astype(np.float32), np.sin(th).astype(np.float32))
    back = _bf16_vals(O.rope_bf16(f, np.cos(-th).astype(np.float32), np.sin(-th).astype(np.float32)))
    r = np.hypot(v[:, :32], v[:, 32:64])                                 # each pair's length
    assert np.all(np.abs(back[:, :32] - v[:, :32]) <= 2 ** -7 * r)
    assert np.all(np.abs(back[:, 32:64] - v[:, 32:64]) <= 2 ** -7 * r)
    assert np.array_equal(back[:, 64:], v[:, 64:])


def test_rope_matches_complex_multiplication():
    """(a + i·b) · (cos θ + i·sin θ), numpy complex128, rounded to bf16."""
    rng = np.random.default_rng(5)
    x = _bf16_bits(rng.standard_normal((8, 128)) * 3)
    th = rng.uniform(-np.pi, np.pi, (8, 32))
    c, s = np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    v = _bf16_vals(x)
    z = (v[:, :32] + 1j * v[:, 32:64]) * (c.astype(np.float64) + 1j * s.astype(np.float64))
    want = v.copy()
    want[:, :32], want[:, 32:64] = z.real, z.imag
    want_bits = torch.from_numpy(want).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.rope_bf16(x, c, s), want_bits)


def test_layer_norm_matches_torch_and_its_special_cases():
    rng = np.random.default_rng(6)
    x = _bf16_bits(rng.standard_normal((16, 128)) * rng.uniform(0.1, 30, (16, 1)) + rng.uniform(-5, 5, (16, 1)))
    g = rng.uniform(0.5, 2, 128).astype(np.float32)
    b = rng.uniform(-1, 1, 128).astype(np.float32)
    eps = np.float32(1e-6)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(_bf16_vals(x)), (128,), torch.from_numpy(g).double(),
                                         torch.from_numpy(b).double(), float(eps))
    want = ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.layer_norm_bf16(x, g, b, eps), want)
    # a constant row normalises to the bias; gain 1 / bias 0 gives mean 0 and variance 1
    const = _bf16_bits(np.full((1, 128), 2.5))
    assert np.array_equal(O.layer_norm_bf16(const, g, b, eps), _bf16_bits(b[None]))
    y = _bf16_vals(O.layer_norm_bf16(x, np.ones(128, np.float32), np.zeros(128, np.float32), eps))
    assert np.all(np.abs(y.mean(axis=1)) < 1e-2) and np.all(np.abs(y.var(axis=1) - 1) < 1e-2)


def test_front_orders_layer_norm_before_rope_and_leaves_weights_alone():
    rng = np.random.default_rng(7)
    q = _bf16_bits(rng.standard_normal((2, 64, 128)))
    k = _bf16_bits(rng.standard_normal((2, 128)) * 4 + 1)
    th = rng.uniform(-3, 3, (2, 32))
    c, s = np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    g, b = np.ones(128, np.float32), np.zeros(128, np.float32)
    fq, fk = O.front(q, k, c, s, g, b, 1e-6)
    for t in range(2):
        assert np.array_equal(fq[t], O.rope_bf16(q[t], c[t], s[t]))
    assert np.array_equal(fk, O.rope_bf16(O.layer_norm_bf16(k, g, b, 1e-6), c, s))
    assert not np.array_equal(fk, O.layer_norm_bf16(O.rope_bf16(k, c, s), g, b, 1e-6))


# --------------------------------------------------------------------------- projections
def test_projections_match_torch_and_exact_rounding():
    """project() against torch's float64 matmul on the same exact inputs (the
    bf16 outputs must agree), the head-major view of q pinned by one-hot
    weights (output h·128 + d lands in head h, feature d), and a few outputs
    recomputed in exact rationals then rounded once."""
    pc = synth.make_proj_case(5, 9, hidden=256, q_lora=512)
    q, k, w = O.project(pc.x, pc.qr, pc.wq_b, pc.wk, pc.w_proj)
    assert q.shape == (9, 64, 128) and k.shape == (9, 128) and w.shape == (9, 64) and w.dtype == np.float32
    tx = torch.from_numpy(O.bf16_bits_to_f64(pc.x))
    tq = torch.from_numpy(O.bf16_bits_to_f64(pc.qr))
    tq_ref = tq @ torch.from_numpy(O.bf16_bits_to_f64(pc.wq_b)).T
    tk_ref = tx @ torch.from_numpy(O.bf16_bits_to_f64(pc.wk)).T
    np.testing.assert_array_equal(q.reshape(9, -1), O.f64_to_bf16_bits(O.bf16_round(tq_ref.numpy())))
    np.testing.assert_array_equal(k, O.f64_to_bf16_bits(O.bf16_round(tk_ref.numpy())))
    tw = (tx @ torch.from_numpy(pc.w_proj.astype(np.float64)).T).numpy().astype(np.float32)
    np.testing.assert_array_equal(w.view(np.uint32), tw.view(np.uint32))
    # exact rationals for a handful of outputs
    xs = O.bf16_bits_to_f64(pc.qr)
    ws = O.bf16_bits_to_f64(pc.wq_b)
    for t, o in ((0, 0), (3, 4097), (8, 8191)):
        exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xs[t], ws[o]))
        assert Fraction(float(O.bf16_bits_to_f64(q.reshape(9, -1)[t, o]))) == bf16_exact(exact)
    # head-major layout: a weight row that copies qr feature 0 into output h·128 + d
    wq1 = np.zeros((64 * 128, 512), np.uint16)
    wq1[5 * 128 + 17, 0] = 0x3F80                    # 1.0 in bf16
    q1, _, _ = O.project(pc.x, pc.qr, wq1, pc.wk, pc.w_proj)
    assert np.array_equal(q1[:, 5, 17], pc.qr[:, 0]) and np.count_nonzero(q1) == np.count_nonzero(pc.qr[:, 0])
