"""Standalone top-k (idx_topk) on exactly known scores, and the fused
score + top-k (idx_score_topk) against the oracle and against idx_score."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import (check_topk_exact_row, check_topk_row, dev, gpu_queries, gpu_state, oracle_queries,
                           oracle_state)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,n,lengths,causal,k,ties", [
    (4, 1, [1, 2047, 2049, 16384], False, 2048, False),
    (3, 1, [5000, 9000, 3000], False, 100, True),      # heavy ties at the threshold
    (1, 1, [131072], False, 2048, False),               # longest row: full cluster
    (2, 40, [40, 3000], True, 64, True),
    (16, 1, list(range(1000, 17000, 1000)), False, 2048, True),
])
def test_topk_exact(B, n, lengths, causal, k, ties):
    from sparse_attention_token_idx_b200 import binding as X
    rng = np.random.default_rng(sum(lengths) + k)
    ld = max(lengths)
    sc = rng.standard_normal((B, n, ld)).astype(np.float32)
    if ties:
        sc = np.round(sc * 8) / 8                     # a few hundred distinct values
    sc[:, :, ::97] = -sc[:, :, ::97] * 1e30           # very large magnitudes of both signs
    lengths = np.array(lengths, np.int32)
    got = X.topk(dev(sc), dev(lengths), causal, k, ld).cpu().numpy()
    assert X.status() == (0, 0)
    for b in range(B):
        for i in range(n):
            vis = O.visible_count(int(lengths[b]), n, i, causal)
            check_topk_exact_row(got[b, i], sc[b, i], vis, k)


# Many rows: one CTA per row, rows fetched by bulk copies, the candidate list
# kept while the keys are counted (used when the k best are a small share).
ROWS = [
    # name, rows, longest row, ld, k, score order
    ("gauss", 128, 16384, 16384, 2048, "random"),
    ("ties", 96, 12000, 12000, 2048, "ties"),          # bin-b1 candidates overflow their list
    ("best-first", 64, 16384, 16384, 2048, "desc"),    # the early bound overshoots: slice fallback
    ("best-last", 64, 16384, 16384, 2048, "asc"),      # the list overflows: slice fallback
    ("large-k", 64, 16384, 16384, 4096, "random"),     # positions written without staging
    ("ragged", 80, 16381, 16384, 512, "random"),       # lengths not multiples of 4 (ld is)
    ("unaligned-ld", 70, 3001, 3001, 700, "random"),   # ld % 4 != 0: cluster kernel
    ("strided-low", 64, 16384, 16384, 2048, "strided"),   # every 4th position far below the rest
]


@pytest.mark.parametrize("name,rows,L,ld,k,order", ROWS)
def test_topk_many_rows(name, rows, L, ld, k, order):
    from sparse_attention_token_idx_b200 import binding as X
    rng = np.random.default_rng(rows * 7 + L + k)
    sc = rng.standard_normal((rows, 1, ld)).astype(np.float32)
    if order == "ties":
        sc = np.round(sc * 4) / 4
    elif order == "desc":
        sc = sc - np.float32(0.01) * np.arange(ld, dtype=np.float32)
    elif order == "asc":
        sc = sc + np.float32(0.01) * np.arange(ld, dtype=np.float32)
    elif order == "strided":
        sc[:, :, ::4] -= np.float32(100.0)
    lengths = rng.integers(max(1, L - 700), L + 1, rows).astype(np.int32)
    lengths[0] = L
    lengths[1] = min(L, k)                       # every visible key selected
    got = X.topk(dev(sc), dev(lengths), False, k, L).cpu().numpy()
    assert X.status() == (0, 0)
    for r in range(rows):
        check_topk_exact_row(got[r, 0], sc[r, 0], int(lengths[r]), k)


def test_topk_negative_zero_and_infinities():
    from sparse_attention_token_idx_b200 import binding as X
    s = np.array([[[0.0, -0.0, 1.0, -np.inf, np.inf, -1.0, 0.0, -0.0]]], np.float32)
    got = X.topk(dev(s), dev(np.array([8], np.int32)), False, 5, 8).cpu().numpy()
    # +inf, 1.0, then three of the four zeros (−0 and +0 compare equal as scores)
    sel = set(got[0, 0].tolist())
    assert {4, 2} <= sel and len(sel) == 5 and sel - {4, 2} <= {0, 1, 6, 7}


FUSED = [
    ("decode-mixed", 6, 1, [0, 100, 2046, 2048, 5000, 16383], 16384, False, 0, 2048),
    ("decode-single", 1, 1, [4095], 4096, False, 1, 2048),
    ("decode-small-k", 4, 1, [511, 2000, 777, 3333], 4096, False, 0, 17),
    ("prefill", 1, 300, [0], 512, True, 0, 64),
    ("chunked", 2, 130, [900, 2500], 4096, True, 1, 512),
    # 64 decode rows, fewer than the SMs: the fused kernel splits each row over
    # a cluster of 2 CTAs that select through distributed shared memory
    ("decode-many", 64, 1, list(range(1000, 2024, 16)), 2048, False, 1, 256),
    # more than half as many rows as SMs: one CTA per row, ragged lengths
    ("decode-100", 100, 1, [1000 + 31 * i for i in range(100)], 4096, False, 0, 256),
    ("decode-n2", 60, 2, [500 + 60 * i for i in range(60)], 4096, True, 1, 128),
]


@pytest.mark.parametrize("use_ws", [False, True])
@pytest.mark.parametrize("name,B,n,positions,T_cap,causal,fmt,k", FUSED)
def test_fused_topk_matches_oracle_and_unfused(name, B, n, positions, T_cap, causal, fmt, k, use_ws):
    from sparse_attention_token_idx_b200 import binding as X
    case = synth.make_case(name, 300 + len(name), B, n, positions, T_cap=T_cap, causal=causal, fmt=fmt, k=k)
    kc, ks, lengths = gpu_state(case)
    qc, w = gpu_queries(case)
    max_len = int(case.lengths.max())
    ws = None
    if use_ws:
        nbytes = X.workspace_size(B, n, max_len, k)
        # a decode-shaped call needs none: one offered anyway must leave the result as it is
        ws = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device="cuda")
    idx = X.score_topk(qc, w, kc, ks, lengths, causal, k, max_len, ws=ws).cpu().numpy()
    sc = X.score(qc, w, kc, ks, lengths, causal, max_len, ld=max_len).cpu().numpy()
    assert X.status() == (0, 0)
    okc, oks = oracle_state(case)
    oqc, ow = oracle_queries(case)
    S, E = O.index_scores(oqc, ow, okc, oks, case.lengths, causal, ncols=max_len)
    for b in range(B):
        for i in range(n):
            vis = O.visible_count(int(case.lengths[b]), n, i, causal)
            check_topk_row(idx[b, i], S[b, i], E[b, i], vis, k)
            # the fused kernel selects from the very fp32 scores idx_score writes
            check_topk_exact_row(idx[b, i], sc[b, i], vis, k)


@pytest.mark.parametrize("zeroed", ["all", "every-4th"])
def test_fused_topk_with_zeroed_keys(zeroed):
    """The fused decode selection on degenerate score rows: keys zeroed at
    every position (all scores tie at 0) or at every 4th of 16 384 positions
    (a quarter of the row ties at 0).  The top-k must still be exact."""
    from sparse_attention_token_idx_b200 import binding as X
    B, T_cap, k = 4, 16384, 2048
    case = synth.make_case("zeroed-" + zeroed, 77, B, 1, [T_cap - 1] * B, T_cap=T_cap, causal=False, fmt=1, k=k)
    if zeroed == "all":
        case.k_prior[:] = 0
        case.k_new[:] = 0
    else:
        case.k_prior[:, ::4] = 0
    kc, ks, lengths = gpu_state(case)
    qc, w = gpu_queries(case)
    idx = X.score_topk(qc, w, kc, ks, lengths, False, k, T_cap).cpu().numpy()
    sc = X.score(qc, w, kc, ks, lengths, False, T_cap, ld=T_cap).cpu().numpy()
    assert X.status() == (0, 0)
    for b in range(B):
        check_topk_exact_row(idx[b, 0], sc[b, 0], T_cap, k)
