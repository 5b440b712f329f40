"""The five benchmark workloads at full size, through the same Indexer.step
call (and launch configuration) the benchmark times.  Every sequence and every
query row is checked: the cache bytes and scales, the query codes and folded
weights bit for bit, and every row's top-k set against the oracle, which
quantises all keys itself from the raw inputs.  The oracle's logits are exact
whatever the summation order (FP8 products in float64), so it computes them as
matrix products; its work is spread over a process pool."""
import numpy as np
import pytest

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import bf16_dev, dev, oracle_check_rows, oracle_pool, oracle_seq_cache

pytestmark = pytest.mark.gpu

ROWS_PER_TASK = 32


@pytest.fixture(scope="module")
def pool():
    with oracle_pool() as p:
        yield p


@pytest.mark.parametrize("widx", [0, 1, 2, 3, 4])
def test_workload_every_row(widx, pool):
    from sparse_attention_token_idx_b200 import binding as X
    from sparse_attention_token_idx_b200.pipeline import Indexer
    case = synth.workload(widx)
    B, n = case.B, case.n
    # oracle caches of every sequence, started before the GPU work
    cache_jobs = [pool.submit(oracle_seq_cache, (case.k_prior[b, :int(case.positions[b])], case.k_new[b], case.T_cap,
                                                 case.fmt)) for b in range(B)]
    ix = Indexer(B, case.T_cap, case.fmt, case.k)
    P = case.k_prior.shape[1]
    if P:
        if np.all(case.positions == P):
            ix.append(bf16_dev(case.k_prior), dev(np.zeros(B, np.int32)))
        else:
            for b in range(B):
                p = int(case.positions[b])
                if p:
                    X.quant_append(bf16_dev(case.k_prior[b:b + 1, :p]), dev(np.zeros(1, np.int32)),
                                   ix.k_cache[b:b + 1], ix.k_scale_cache[b:b + 1], case.fmt)
    max_len = int(case.lengths.max())
    idx = ix.step(bf16_dev(case.k_new), bf16_dev(case.q), dev(case.w_raw), dev(case.positions),
                  dev(case.lengths), causal=case.causal, max_len=max_len)
    assert X.status() == (0, 0)
    idx = idx.cpu().numpy()
    kc = ix.k_cache.cpu().numpy()
    ks = ix.k_scale_cache.cpu().numpy()
    qc_gpu = ix._bufs["q_fp8"].cpu().numpy()
    w_gpu = ix._bufs["w"].cpu().numpy()
    # query codes and folded weights of every row, bit for bit
    qc, _, w = O.quant_queries(case.q, case.w_raw, case.fmt)
    np.testing.assert_array_equal(qc_gpu, qc)
    np.testing.assert_array_equal(w_gpu.view(np.uint32), w.view(np.uint32))
    # cache bytes and scales of every sequence, bit for bit
    caches = [j.result() for j in cache_jobs]
    for b in range(B):
        L = int(case.lengths[b])
        okc, oks = caches[b]
        np.testing.assert_array_equal(kc[b, :L], okc, err_msg=f"cache codes of sequence {b}")
        np.testing.assert_array_equal(ks[b, :L].view(np.uint32), oks.view(np.uint32),
                                      err_msg=f"cache scales of sequence {b}")
    # every row's top-k set against the oracle's scores
    jobs = []
    for b in range(B):
        L = int(case.lengths[b])
        okc, oks = caches[b]
        for i0 in range(0, n, ROWS_PER_TASK):
            rows = list(range(i0, min(n, i0 + ROWS_PER_TASK)))
            vis = [O.visible_count(L, n, i, case.causal) for i in rows]
            V = max(vis)
            jobs.append(pool.submit(oracle_check_rows, (qc[b, rows], w[b, rows], okc[:V], oks[:V], vis,
                                                        idx[b, rows], case.k, [(b, i) for i in rows])))
    checked = sum(j.result() for j in jobs)
    assert checked == B * n
