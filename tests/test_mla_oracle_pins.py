"""Pins for the sparse latent attention oracle (oracle/mla.py): dense
attention from torch's scaled_dot_product_attention when every position is
selected, the additive −inf mask reading of the selection, the split of the
joined 576-feature product into latent and rotary parts, and the special cases
(one selected position, none, order of the selection).  CPU only."""
import numpy as np
import torch

from oracle import mla as M


def _bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _case(B=2, H=8, T=40, seed=0):
    rng = np.random.default_rng(seed)
    return _bits(rng.standard_normal((B, H, M.DIM))), _bits(rng.standard_normal((B, T, M.DIM)))


def test_full_selection_is_dense_attention():
    q, kv = _case()
    B, H, _ = q.shape
    T = kv.shape[1]
    scale = 192 ** -0.5
    idx = np.tile(np.arange(T), (B, 1))
    o, _ = M.sparse_mla_decode(q, kv, idx, scale)
    qt = torch.from_numpy(M.bf16_bits_to_f64(q))                              # [B, H, 576]
    kt = torch.from_numpy(M.bf16_bits_to_f64(kv))                             # [B, T, 576]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt[:, :, None, :], kt[:, None].expand(B, H, T, M.DIM), kt[:, None, :, :M.LAT].expand(B, H, T, M.LAT),
        scale=scale)[:, :, 0]
    assert np.allclose(o, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_selection_equals_an_additive_minus_inf_mask():
    q, kv = _case(seed=1)
    rng = np.random.default_rng(2)
    T = kv.shape[1]
    idx = np.stack([rng.permutation(T)[:11] for _ in range(2)])
    idx[1, 7:] = -1                                                           # padding selects nothing
    o, P = M.sparse_mla_decode(q, kv, idx, 0.1)
    qf, kf = M.bf16_bits_to_f64(q), M.bf16_bits_to_f64(kv)
    for b in range(2):
        mask = np.full(T, -np.inf)
        mask[idx[b][idx[b] >= 0]] = 0.0
        s = 0.1 * (qf[b] @ kf[b].T) + mask
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        assert np.allclose(o[b], p @ kf[b, :, :M.LAT], rtol=1e-12, atol=1e-13)
        assert np.allclose(P[b][:, idx[b] >= 0], p[:, idx[b][idx[b] >= 0]], rtol=1e-12)
        assert np.all(P[b][:, idx[b] < 0] == 0)


def test_joined_product_is_latent_plus_rotary_scores():
    q, kv = _case(seed=3)
    qf, kf = M.bf16_bits_to_f64(q), M.bf16_bits_to_f64(kv)
    joined = qf[0] @ kf[0].T
    split = qf[0, :, :M.LAT] @ kf[0, :, :M.LAT].T + qf[0, :, M.LAT:] @ kf[0, :, M.LAT:].T
    assert np.allclose(joined, split, rtol=1e-12, atol=1e-12)


def test_special_cases():
    q, kv = _case(seed=4)
    T = kv.shape[1]
    one = np.array([[5], [T - 1]])
    o, P = M.sparse_mla_decode(q, kv, one, 0.3)                               # one position: its latent row
    assert np.array_equal(o[0], np.tile(M.bf16_bits_to_f64(kv[0, 5, :M.LAT]), (q.shape[1], 1)))
    assert np.all(P == 1.0)
    none = np.full((2, 4), -1)
    o, P = M.sparse_mla_decode(q, kv, none, 0.3)
    assert np.all(o == 0) and np.all(P == 0)
    rng = np.random.default_rng(5)
    idx = np.stack([rng.permutation(T)[:9] for _ in range(2)])
    o1, _ = M.sparse_mla_decode(q, kv, idx, 0.3)
    o2, _ = M.sparse_mla_decode(q, kv, idx[:, ::-1], 0.3)                     # a set: order does not matter
    assert np.allclose(o1, o2, rtol=1e-13, atol=1e-14)
