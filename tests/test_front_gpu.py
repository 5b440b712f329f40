"""Front end fused with the quantiser (idx_front_quant_append): query RoPE, key
LayerNorm + RoPE, rotation, FP8 quantisation, cache append and weight folding,
bit-exact against the oracle; and one indexer step from the projections on
(Indexer.step_front) against the oracle's scores."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import bf16_dev, check_topk_row, dev

pytestmark = pytest.mark.gpu


def _front_inputs(case, seed):
    """RoPE tables from each token's position (θ_i = 10000^(−i/32)) and a LayerNorm gain / bias."""
    rng = np.random.default_rng(seed)
    pos = case.positions[:, None].astype(np.float64) + np.arange(case.n)[None, :]            # [B, n]
    theta = 10000.0 ** (-np.arange(32) / 32.0)
    ang = pos[..., None] * theta                                                             # [B, n, 32]
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    gain = rng.normal(1.0, 0.2, 128).astype(np.float32)
    bias = rng.normal(0.0, 0.2, 128).astype(np.float32)
    return cos, sin, gain, bias


def _oracle_front(case, cos, sin, gain, bias, eps, T_cap):
    fq, fk = O.front(case.q, case.k_new, cos, sin, gain, bias, eps)
    qc, _, w = O.quant_queries(fq, case.w_raw, case.fmt)
    kc = np.zeros((case.B, T_cap, 128), np.uint8)
    ks = np.zeros((case.B, T_cap), np.float32)
    O.quant_append(fk, case.positions, kc, ks, case.fmt)
    return qc, w, kc, ks


@pytest.mark.parametrize("B,n,positions,fmt,special", [
    (16, 1, list(range(0, 4000, 250)), 1, False),     # decode
    (2, 300, [0, 700], 0, True),                      # prefill; a constant key row and a huge one
    (3, 7, [5, 60, 2000], 1, True),                   # rows not a multiple of the 8 rows per warp
])
def test_front_quant_append_bit_exact(B, n, positions, fmt, special):
    from sparse_attention_token_idx_b200 import binding as X
    T_cap = 4096
    case = synth.make_case("front", 31 + n, B, n, positions, T_cap=T_cap, k=64, fmt=fmt)
    if special:
        k = case.k_new.copy()
        k[0, 0] = 0x4020                                                  # all 2.5: zero variance
        k[-1, -1] = (k[-1, -1].astype(np.uint32) + 0x0C00).astype(np.uint16) & 0x7FFF | (k[-1, -1] & 0x8000)
        case.k_new = k
    cos, sin, gain, bias = _front_inputs(case, 3 + n)
    eps = np.float32(1e-6)
    kc = torch.zeros((B, T_cap, 128), dtype=torch.uint8, device="cuda")
    ks = torch.zeros((B, T_cap), dtype=torch.float32, device="cuda")
    q_fp8, w = X.front_quant_append(bf16_dev(case.q), dev(case.w_raw), bf16_dev(case.k_new), dev(cos), dev(sin),
                                    dev(gain), dev(bias), float(eps), dev(case.positions), kc, ks, fmt)
    assert X.status() == (0, 0)
    qc, ow, okc, oks = _oracle_front(case, cos, sin, gain, bias, eps, T_cap)
    assert np.array_equal(q_fp8.cpu().numpy(), qc), "query codes differ"
    assert np.array_equal(w.cpu().numpy(), ow), "folded weights differ"
    assert np.array_equal(kc.cpu().numpy(), okc), "key cache differs"
    assert np.array_equal(ks.cpu().numpy(), oks), "key scales differ"


def test_step_front_matches_oracle():
    from sparse_attention_token_idx_b200.pipeline import Indexer
    case = synth.make_case("front-step", 77, 4, 1, [3000, 9000, 100, 16000], T_cap=16384, k=512, fmt=1)
    cos, sin, gain, bias = _front_inputs(case, 9)
    eps = np.float32(1e-6)
    ix = Indexer(case.B, case.T_cap, case.fmt, case.k)
    # prior keys as the oracle caches them (rotation + quantisation only)
    okc = np.zeros((case.B, case.T_cap, 128), np.uint8)
    oks = np.zeros((case.B, case.T_cap), np.float32)
    from sparse_attention_token_idx_b200 import binding as X
    for b in range(case.B):
        p = int(case.positions[b])
        O.quant_append(case.k_prior[b:b + 1, :p], [0], okc[b:b + 1], oks[b:b + 1], case.fmt)
        X.quant_append(bf16_dev(case.k_prior[b:b + 1, :p]), dev(np.zeros(1, np.int32)), ix.k_cache[b:b + 1],
                       ix.k_scale_cache[b:b + 1], case.fmt)
    idx = ix.step_front(bf16_dev(case.q), dev(case.w_raw), bf16_dev(case.k_new), dev(cos), dev(sin), dev(gain),
                        dev(bias), dev(case.positions), dev(case.lengths), causal=False,
                        max_len=int(case.lengths.max()), ln_eps=float(eps)).cpu().numpy()
    assert X.status() == (0, 0)
    fq, fk = O.front(case.q, case.k_new, cos, sin, gain, bias, eps)
    O.quant_append(fk, case.positions, okc, oks, case.fmt)
    qc, _, w = O.quant_queries(fq, case.w_raw, case.fmt)
    assert np.array_equal(ix.k_cache.cpu().numpy(), okc)
    S, E = O.index_scores(qc, w, okc, oks, case.lengths, False)
    for b in range(case.B):
        check_topk_row(idx[b, 0], S[b, 0], E[b, 0], int(case.lengths[b]), case.k)
