"""Rotation + FP8 quantisation + cache append on the GPU, bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import bf16_dev, dev

pytestmark = pytest.mark.gpu


def _rows(seed, n):
    rng = np.random.default_rng(seed)
    raw = rng.standard_normal((n, 128)).astype(np.float32)
    raw[:, rng.choice(128, 2, replace=False)] *= 20
    bits = synth._to_bf16_bits(raw)
    # edge rows: all zero, negative zeros, one spike, tiny (subnormal bf16), huge, alternating signs
    bits[0] = 0
    bits[1] = 0x8000
    bits[2] = 0; bits[2, 5] = 0x3F80
    bits[3] = synth._to_bf16_bits(raw[3] * np.float32(1e-39))
    bits[4] = synth._to_bf16_bits(raw[4] * np.float32(1e35))
    bits[5] = np.where(np.arange(128) % 2 == 0, 0x3F80, 0xBF80).astype(np.uint16)
    bits[6] = 0x0001                       # smallest subnormal everywhere
    bits[7] = 0; bits[7, 100] = 0x7F7F      # largest finite bf16 as a spike
    return bits


@pytest.mark.parametrize("fmt", [0, 1])
def test_quant_rows_bit_exact(fmt):
    from sparse_attention_token_idx_b200 import binding as X
    bits = _rows(1 + fmt, 4099)            # several blocks and a ragged tail
    codes, scale = X.quant(bf16_dev(bits), fmt)
    torch.cuda.synchronize()
    oc, os_ = O.rotate_quant(bits, fmt)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)
    np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("fmt", [0, 1])
def test_quant_queries_bit_exact(fmt):
    from sparse_attention_token_idx_b200 import binding as X
    case = synth.make_case("q", 31 + fmt, 3, 5, [10, 20, 30], T_cap=64, fmt=fmt)
    qc, w = X.quant_queries(bf16_dev(case.q), dev(case.w_raw), fmt)
    torch.cuda.synchronize()
    oc, _, ow = O.quant_queries(case.q, case.w_raw, fmt)
    np.testing.assert_array_equal(qc.cpu().numpy(), oc)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), ow.view(np.uint32))


@pytest.mark.parametrize("fmt", [0, 1])
def test_append_bit_exact_and_in_place(fmt):
    from sparse_attention_token_idx_b200 import binding as X
    B, n, T = 4, 37, 300
    case = synth.make_case("a", 41 + fmt, B, n, [0, 5, 263, 130], T_cap=T, fmt=fmt)
    kc = torch.full((B, T, 128), 0xAB, dtype=torch.uint8, device="cuda")
    ks = torch.full((B, T), -3.0, dtype=torch.float32, device="cuda")
    X.quant_append(bf16_dev(case.k_new), dev(case.positions), kc, ks, fmt)
    assert X.status() == (0, 0)
    okc = np.full((B, T, 128), 0xAB, np.uint8)
    oks = np.full((B, T), -3.0, np.float32)
    O.quant_append(case.k_new, case.positions, okc, oks, fmt)
    np.testing.assert_array_equal(kc.cpu().numpy(), okc)
    np.testing.assert_array_equal(ks.cpu().numpy().view(np.uint32), oks.view(np.uint32))


def test_append_rejects_positions_past_capacity():
    from sparse_attention_token_idx_b200 import binding as X
    B, n, T = 3, 8, 64
    case = synth.make_case("a", 50, B, n, [0, 56, 10], T_cap=T)
    kc = torch.zeros((B, T, 128), dtype=torch.uint8, device="cuda")
    ks = torch.zeros((B, T), dtype=torch.float32, device="cuda")
    bad = np.array([0, 57, -1], np.int32)       # 57 + 8 > 64, and a negative slot
    X.quant_append(bf16_dev(case.k_new), dev(bad), kc, ks, 0)
    code, bits = X.status()
    assert code == -7 and bits & X.DEV_ERR_POSITION
    okc = np.zeros((B, T, 128), np.uint8)
    oks = np.zeros((B, T), np.float32)
    O.quant_append(case.k_new[:1], [0], okc[:1], oks[:1], 0)
    np.testing.assert_array_equal(kc.cpu().numpy(), okc)       # bad sequences untouched
    assert X.status() == (0, 0)                                 # the word was cleared


def test_e4m3_encoder_matches_oracle():
    from sparse_attention_token_idx_b200 import binding as X
    rng = np.random.default_rng(60)
    parts = [rng.standard_normal(2_000_000).astype(np.float32) * np.float32(100),
             (rng.standard_normal(500_000) * 2.0 ** -7).astype(np.float32),
             rng.integers(0, 2 ** 32, 2_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)]
    v = O.e4m3_values()[:0x7F]
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
                           v.astype(np.float32), np.array([448, 449, 463.99, 464, 465, 3e38], np.float32)])
    parts.append(near)
    x = np.concatenate(parts)
    x = x[np.isfinite(x)]
    x = np.concatenate([x, -x])
    got = X.e4m3_encode(dev(x)).cpu().numpy()
    np.testing.assert_array_equal(got, O.e4m3_encode(x))
