"""Storage and output variants: e8m0 key-scale bytes (the fp8_index docstring's
"e8m0 here", "Index scores" page), bf16 scores and a finite mask bound (the NKI
indexer page's Notes).  Each is checked against the default path (bit-exact:
an e8m0 byte is the same power of two as the fp32 ue8m0 scale; a bf16 score is
the nearest-even rounding of the fp32 one) and against the oracle."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import bf16_dev, check_scores, check_topk_row, dev, gpu_queries, oracle_queries, oracle_state

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, n, positions, T_cap, causal
    ("decode", 6, 1, [0, 100, 2046, 2048, 3000, 4095], 4096, False),
    ("prefill", 1, 300, [0], 512, True),
    ("chunked", 2, 130, [900, 2500], 4096, True),
]


def _caches(case):
    """The same keys appended twice: fp32 ue8m0 scales, and e8m0 bytes."""
    from sparse_attention_token_idx_b200 import binding as X
    B, T = case.B, case.T_cap
    kc32 = torch.zeros((B, T, 128), dtype=torch.uint8, device="cuda")
    ks32 = torch.zeros((B, T), dtype=torch.float32, device="cuda")
    kc8 = torch.zeros((B, T, 128), dtype=torch.uint8, device="cuda")
    ks8 = torch.zeros((B, T), dtype=torch.uint8, device="cuda")
    for b in range(B):
        p = int(case.positions[b])
        if p:
            X.quant_append(bf16_dev(case.k_prior[b:b + 1, :p]), dev(np.zeros(1, np.int32)), kc32[b:b + 1],
                           ks32[b:b + 1], 1)
            X.quant_append_e8(bf16_dev(case.k_prior[b:b + 1, :p]), dev(np.zeros(1, np.int32)), kc8[b:b + 1],
                              ks8[b:b + 1])
    X.quant_append(bf16_dev(case.k_new), dev(case.positions), kc32, ks32, 1)
    X.quant_append_e8(bf16_dev(case.k_new), dev(case.positions), kc8, ks8)
    return kc32, ks32, kc8, ks8


@pytest.mark.parametrize("name,B,n,positions,T_cap,causal", CASES)
def test_e8m0_cache_matches_fp32_ue8m0_cache(name, B, n, positions, T_cap, causal):
    from sparse_attention_token_idx_b200 import binding as X
    case = synth.make_case(name, 400 + len(name), B, n, positions, T_cap=T_cap, causal=causal, fmt=1, k=64)
    kc32, ks32, kc8, ks8 = _caches(case)
    assert torch.equal(kc32, kc8)
    s32 = ks32.cpu().numpy()
    b8 = ks8.cpu().numpy()
    written = s32 != 0
    # the byte is the exponent field of the fp32 power of two, and the oracle's e8m0 code of it
    assert np.array_equal(b8[written], ((s32[written].view(np.uint32) >> 23) & 0xFF).astype(np.uint8))
    assert np.array_equal(b8[written], O.e8m0_encode(s32[written].astype(np.float64)))
    assert np.all(b8[~written] == 0)
    # scores: bit-identical to the fp32-scale path; selections identical
    qc, w = gpu_queries(case)
    lengths = dev(case.lengths)
    max_len = int(case.lengths.max())
    ref = X.score(qc, w, kc32, ks32, lengths, causal, max_len, ld=max_len)
    got = X.score_ex(qc, w, kc8, ks8, lengths, causal, max_len, ld=max_len)
    assert torch.equal(ref, got)
    for ws_on in (False, True):
        nbytes = X.workspace_size(B, n, max_len, case.k)
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda") if ws_on else None
        a = X.score_topk(qc, w, kc32, ks32, lengths, causal, case.k, max_len, ws=ws)
        b = X.score_topk_ex(qc, w, kc8, ks8, lengths, causal, case.k, max_len, ws=ws)
        assert torch.equal(torch.sort(a, -1).values, torch.sort(b, -1).values)
    assert X.status() == (0, 0)
    # and the e8m0 path against the oracle (its scales decoded from the bytes)
    okc, oks = oracle_state(case)
    assert np.array_equal(O.e8m0_decode(b8[written]), oks[written].astype(np.float64))
    oqc, ow = oracle_queries(case)
    S, E = O.index_scores(oqc, ow, okc, oks, case.lengths, causal, ncols=max_len)
    check_scores(got.cpu().numpy(), S, E)


@pytest.mark.parametrize("name,B,n,positions,T_cap,causal", CASES)
def test_bf16_scores_and_finite_mask(name, B, n, positions, T_cap, causal):
    from sparse_attention_token_idx_b200 import binding as X
    case = synth.make_case(name, 450 + len(name), B, n, positions, T_cap=T_cap, causal=causal, fmt=0, k=64)
    kc32, ks32, _, _ = _caches(synth.make_case(name, 450 + len(name), B, n, positions, T_cap=T_cap,
                                               causal=causal, fmt=1, k=64))
    qc, w = gpu_queries(case)
    lengths = dev(case.lengths)
    max_len = int(case.lengths.max())
    ld = max_len + 9
    ref = X.score(qc, w, kc32, ks32, lengths, causal, max_len, ld=ld)
    fin = X.score_ex(qc, w, kc32, ks32, lengths, causal, max_len, ld=ld, mask_value=X.MASK_BOUND_BF16)
    b16 = X.score_ex(qc, w, kc32, ks32, lengths, causal, max_len, ld=ld, dtype=torch.bfloat16,
                     mask_value=X.MASK_BOUND_BF16)
    inf16 = X.score_ex(qc, w, kc32, ks32, lengths, causal, max_len, ld=ld, dtype=torch.bfloat16)
    assert X.status() == (0, 0)
    r = ref.cpu().numpy()
    masked = np.isneginf(r)
    f = fin.cpu().numpy()
    # finite bound exactly where idx_score has −inf, the same scores elsewhere
    assert np.all(f[masked] == np.float32(O.MASK_BOUND_BF16)) and np.array_equal(f[~masked], r[~masked])
    # bf16: the nearest-even rounding of the fp32 scores (the oracle's rounding, checked against torch's)
    g = b16.float().cpu().numpy().astype(np.float64)
    want = O.scores_bf16(O.masked(r, O.MASK_BOUND_BF16))
    assert np.array_equal(g, want)
    assert np.all(np.isneginf(inf16.float().cpu().numpy()[masked]))
    # against the oracle: within the fp32 tolerance plus half a bf16 unit
    okc, oks = oracle_state(synth.make_case(name, 450 + len(name), B, n, positions, T_cap=T_cap, causal=causal,
                                            fmt=1, k=64))
    oqc, ow = oracle_queries(case)
    S, E = O.index_scores(oqc, ow, okc, oks, case.lengths, causal, ncols=ld)
    v = ~np.isneginf(S)
    bound = 1e-5 * E[v] + 2.0 ** -8 * (np.abs(S[v]) + 1e-5 * E[v])
    assert np.all(np.abs(g[v] - S[v]) <= bound)
    assert np.all(g[~v] == O.MASK_BOUND_BF16)
