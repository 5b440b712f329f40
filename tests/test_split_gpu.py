"""Split-T selection on one GPU: a sequence's keys cut into G slices, each
slice's top-k turned into (score, global position) candidates by
idx_gather_scores, the candidates stacked as an all-gather lays them out, and
idx_merge_topk selecting the row's k best.  Checked against exactly known
scores (the whole row's top-k) and end to end against the oracle's scores."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from sparse_attention_token_idx_b200.parallel import key_slice, slice_candidates, slice_counts
from tests.helpers import check_topk_exact_row, check_topk_row, dev, gpu_queries, gpu_state, oracle_queries, oracle_state

pytestmark = pytest.mark.gpu


# G, rows, T, slice alignment, k, ties, ragged lengths
MERGE = [
    (2, 64, 16384, 128, 2048, False, False),
    (4, 32, 32768, 128, 2048, True, True),      # ties at the threshold; some rows shorter than k
    (8, 16, 65536, 128, 2048, False, True),     # G·k = 16384 candidates (the limit)
    (3, 40, 3000, 1, 100, True, True),          # slices of 1000 keys, candidates not a multiple of 4
    (3, 6, 15, 1, 7, False, True),              # tiny: rows of ≤ 7 keys keep every candidate (k_t = valid)
    (1, 8, 5000, 128, 256, False, True),        # one slice: the merge passes the slice top-k through
]


@pytest.mark.parametrize("G,rows,T,align,k,ties,ragged", MERGE)
def test_gather_merge_exact(G, rows, T, align, k, ties, ragged):
    from sparse_attention_token_idx_b200 import binding as X
    rng = np.random.default_rng(G * 1000 + rows + T + k)
    sc = rng.standard_normal((rows, T)).astype(np.float32)
    if ties:
        sc = np.round(sc * 8) / 8
    sc[:, ::89] *= -1e30                              # very large magnitudes of both signs
    L = rng.integers(1, T + 1, rows).astype(np.int32) if ragged else np.full(rows, T, np.int32)
    if ragged:
        L[0], L[-1] = T, 1                            # a full row and a one-key row
    cands = []
    for g in range(G):
        lo, hi = key_slice(T, g, G, align)
        cnt = slice_counts(L, lo, hi)
        loc = np.stack([O.topk_row(sc[r, lo:hi], int(cnt[r]), k) for r in range(rows)])
        span = max(hi - lo, 1)
        part = np.zeros((rows, span), np.float32)
        part[:, :hi - lo] = sc[:, lo:hi]
        cands.append(X.gather_scores(dev(part), dev(loc), lo, counts=dev(cnt)))
    got = X.merge_topk(torch.stack(cands), k).cpu().numpy()
    assert X.status() == (0, 0)
    for r in range(rows):
        check_topk_exact_row(got[r], sc[r], int(L[r]), k)


def test_gather_marks_positions_past_the_count_empty():
    from sparse_attention_token_idx_b200 import binding as X
    sc = np.arange(24, dtype=np.float32).reshape(2, 12)
    idx = np.array([[0, 5, -1, 11], [3, 2, 7, 1]], np.int32)
    cnt = np.array([6, 3], np.int32)
    c = X.gather_scores(dev(sc), dev(idx), 100, counts=dev(cnt)).cpu().numpy()
    pos, val = c[..., 1], c[..., 0].view(np.float32)
    assert pos.tolist() == [[100, 105, -1, -1], [-1, 102, -1, 101]]
    assert val[0, :2].tolist() == [0.0, 5.0] and np.all(np.isneginf(val[0, 2:]))
    assert val[1, 1] == 14.0 and val[1, 3] == 13.0 and np.isneginf(val[1, 0]) and np.isneginf(val[1, 2])


@pytest.mark.parametrize("G,T_cap,positions,k,fmt", [
    (4, 65536, [50000, 9000], 2048, 1),   # the second sequence leaves three slices empty
    (2, 16384, [16383, 3000, 12000], 512, 0),
])
def test_split_t_decode_matches_oracle(G, T_cap, positions, k, fmt):
    from sparse_attention_token_idx_b200 import binding as X
    case = synth.make_case("split-t", 5 + G, len(positions), 1, positions, T_cap=T_cap, k=k, fmt=fmt)
    kc, ks, lengths = gpu_state(case)
    q_fp8, w = gpu_queries(case)
    cands = []
    for g in range(G):
        lo, hi = key_slice(T_cap, g, G)
        cands.append(slice_candidates(q_fp8, w, kc[:, lo:hi].contiguous(), ks[:, lo:hi].contiguous(), lengths,
                                      lo, hi, k))
    got = X.merge_topk(torch.stack(cands), k).cpu().numpy()
    assert X.status() == (0, 0)
    okc, oks = oracle_state(case)
    qc, ow = oracle_queries(case)
    S, E = O.index_scores(qc, ow, okc, oks, case.lengths, False)
    for b in range(case.B):
        check_topk_row(got[b], S[b, 0], E[b, 0], int(case.lengths[b]), k)
