"""Sparse latent attention over the selected positions (idx_sparse_mla_decode)
against the oracle (oracle/mla.py), element by element within a bound derived
from the kernel's fp32 arithmetic:

* a score is a 576-term fp32 sum of exact bf16·bf16 products, so its error is
  at most e_t = 576·u·scale·Σ_d |q_d kv_t,d|  (u = 2^-24);
* errors e_t move each softmax weight by at most a factor exp(±2·max e_t);
* the exponentials, running sums, rescalings and the final division add at
  most (k + 600)·u relative;
so |o_gpu − o| ≤ (exp(2·max e_t) − 1 + (k + 600)·u) · Σ_t p_t |kv_t,j| per
output element.  Blocks of 128 heads run on the tensor cores, where the
softmax weights are rounded to bf16 before the weighted sum (and summed as
rounded): each normalised weight then moves by at most 2·2^-9 of itself, which
adds 2^-8 to the factor."""
import numpy as np
import pytest
import torch

from oracle import mla as M
from tests.helpers import dev

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def _bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("B,H,T_cap,k,scale,fills", [
    (4, 128, 4096, 2048, 192 ** -0.5, [2048, 1000, 1, 0]),   # full, padded, one position, none
    (3, 16, 300, 100, 0.3, [100, 37, 64]),                  # k not a multiple of 32; a peaky softmax
    (2, 32, 1 << 16, 2048, 192 ** -0.5, [2048, 2047]),       # positions spread over a long cache
    (2, 256, 1 << 15, 1000, 0.7, [1000, 999]),               # two 128-head blocks; k not a multiple of 64
    (2, 128, 4096, 300, 3.0, [300, 130]),                    # a very peaky softmax (reference max raised)
])
def test_sparse_mla_decode_matches_oracle(B, H, T_cap, k, scale, fills):
    from sparse_attention_token_idx_b200 import binding as X
    rng = np.random.default_rng(B * 100 + k)
    q = _bits(rng.standard_normal((B, H, M.DIM)))
    kv = _bits(rng.standard_normal((B, T_cap, M.DIM)))
    idx = np.full((B, k), -1, np.int32)
    for b, f in enumerate(fills):
        idx[b, :f] = rng.choice(T_cap, f, replace=False)
        rng.shuffle(idx[b])                                            # padding anywhere in the row
    gpu_idx = idx.copy()
    if B > 1 and fills[1] < k:
        gpu_idx[1, np.flatnonzero(idx[1] < 0)[:3]] = T_cap + 5         # past the cache: also selects nothing
    out = X.sparse_mla_decode(_bf16_dev(q), _bf16_dev(kv), dev(gpu_idx), scale).cpu().numpy()
    assert X.status() == (0, 0)
    o, P = M.sparse_mla_decode(q, kv, idx, scale)
    qf = M.bf16_bits_to_f64(q)
    for b in range(B):
        ok = idx[b] >= 0
        if not ok.any():
            assert np.all(out[b] == 0)
            continue
        kvs = M.bf16_bits_to_f64(kv[b, idx[b][ok]])                       # [n, 576]
        e = 576 * U * abs(scale) * (np.abs(qf[b]) @ np.abs(kvs).T)        # [H, n]
        rel = np.expm1(2 * e.max(axis=1)) + (k + 600) * U                 # [H]
        if H % 128 == 0:
            rel = rel + 2.0 ** -8                                         # bf16 softmax weights
        A = P[b][:, ok] @ np.abs(kvs[:, :M.LAT])                          # [H, 512]
        err = np.abs(out[b].astype(np.float64) - o[b])
        bound = rel[:, None] * A + 1e-30
        assert np.all(err <= bound), f"b={b}: worst err/bound {np.max(err / bound):.3f}"
