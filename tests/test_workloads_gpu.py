"""The five benchmark workloads at full size, through the same Indexer.step
call (and launch configuration) the benchmark times.  The cache bytes and
scales, the query codes and folded weights are compared bit for bit; the top-k
sets of sampled rows against the oracle (which quantises those sequences'
keys itself from the raw inputs)."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import bf16_dev, check_topk_row, dev, oracle_state

pytestmark = pytest.mark.gpu

SAMPLE_SEQS = {0: [0], 1: None, 2: [0, 37, 127], 3: [0], 4: [0, 1]}
SAMPLE_ROWS = {3: [0, 1, 127, 128, 2046, 2047, 2048, 3001, 4095], 4: [0, 1, 700, 2047]}


@pytest.mark.parametrize("widx", [0, 1, 2, 3, 4])
def test_workload(widx):
    from sparse_attention_token_idx_b200.pipeline import Indexer
    case = synth.workload(widx)
    B, n = case.B, case.n
    ix = Indexer(B, case.T_cap, case.fmt, case.k)
    P = case.k_prior.shape[1]
    if P:
        if np.all(case.positions == P):
            ix.append(bf16_dev(case.k_prior), dev(np.zeros(B, np.int32)))
        else:
            for b in range(B):
                p = int(case.positions[b])
                if p:
                    kp = bf16_dev(case.k_prior[b:b + 1, :p])
                    X_k = ix.k_cache[b:b + 1]
                    from sparse_attention_token_idx_b200 import binding as X
                    X.quant_append(kp, dev(np.zeros(1, np.int32)), X_k, ix.k_scale_cache[b:b + 1], case.fmt)
    max_len = int(case.lengths.max())
    idx = ix.step(bf16_dev(case.k_new), bf16_dev(case.q), dev(case.w_raw), dev(case.positions),
                  dev(case.lengths), causal=case.causal, max_len=max_len)
    from sparse_attention_token_idx_b200 import binding as X
    assert X.status() == (0, 0)
    idx = idx.cpu().numpy()
    seqs = SAMPLE_SEQS[widx] if SAMPLE_SEQS[widx] is not None else range(B)
    okc, oks = oracle_state(case, seqs)
    kc = ix.k_cache.cpu().numpy()
    ks = ix.k_scale_cache.cpu().numpy()
    for b in seqs:
        L = int(case.lengths[b])
        np.testing.assert_array_equal(kc[b, :L], okc[b, :L])
        np.testing.assert_array_equal(ks[b, :L].view(np.uint32), oks[b, :L].view(np.uint32))
    qc, _, w = O.quant_queries(case.q[list(seqs)], case.w_raw[list(seqs)], case.fmt)
    np.testing.assert_array_equal(ix._bufs["q_fp8"].cpu().numpy()[list(seqs)], qc)
    np.testing.assert_array_equal(ix._bufs["w"].cpu().numpy()[list(seqs)].view(np.uint32), w.view(np.uint32))
    rows = SAMPLE_ROWS.get(widx)
    oq, _, ow = O.quant_queries(case.q, case.w_raw, case.fmt) if B * n <= 4096 else (None, None, None)
    if oq is None:
        oq = np.zeros(case.q.shape, np.uint8)
        ow = np.zeros(case.w_raw.shape, np.float32)
        oq[list(seqs)] = qc
        ow[list(seqs)] = w
    S, E = O.index_scores(oq, ow, okc, oks, case.lengths, case.causal, ncols=max_len, rows=rows, seqs=seqs)
    for b in seqs:
        for i in (rows if rows is not None else range(n)):
            vis = O.visible_count(int(case.lengths[b]), n, i, case.causal)
            check_topk_row(idx[b, i], S[b, i], E[b, i], vis, case.k)
