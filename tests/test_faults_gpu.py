"""Argument errors are rejected on the host; data-dependent errors raise bits in
the device error word; a bounded wait that is made to expire (a barrier that
nothing signals) ends the kernel with IDX_DEV_ERR_TIMEOUT and leaves the
context usable.  No test here faults, traps or hangs the GPU."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_token_idx_b200 import synth
from tests.helpers import dev, gpu_queries, gpu_state

pytestmark = pytest.mark.gpu


def _small():
    case = synth.make_case("f", 400, 2, 1, [300, 1000], T_cap=2048)
    kc, ks, lengths = gpu_state(case)
    qc, w = gpu_queries(case)
    return case, kc, ks, lengths, qc, w


def test_host_argument_errors():
    from sparse_attention_token_idx_b200 import binding as X
    lib = X.load()
    case, kc, ks, lengths, qc, w = _small()
    out = torch.empty((2, 1, 64), dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    P = lambda t: t.data_ptr()
    args = [P(qc), P(w), P(kc), P(ks), P(lengths), 2, 1, 2048, 1001, 0, 64, P(out), None, 0, s]
    assert lib.idx_score_topk(*args) == 0
    bad = list(args); bad[0] = None
    assert lib.idx_score_topk(*bad) == -1                    # NULL
    bad = list(args); bad[10] = 0
    assert lib.idx_score_topk(*bad) == -4                    # k <= 0
    bad = list(args); bad[8] = 4096
    assert lib.idx_score_topk(*bad) == -2                    # max_len > T_cap
    bad = list(args); bad[9] = 2
    assert lib.idx_score_topk(*bad) == -2                    # causal not 0/1
    bad = list(args); bad[2] = P(kc) + 8
    assert lib.idx_score_topk(*bad) == -5                    # misaligned cache
    assert lib.idx_quant(P(qc), 1, P(qc), P(w), 3, s) == -3  # bad fmt
    assert lib.idx_quant(None, 0, None, None, 0, s) == 0     # empty is fine
    assert X.status() == (0, 0)


def test_lengths_beyond_max_len_are_reported_and_rows_emptied():
    from sparse_attention_token_idx_b200 import binding as X
    case, kc, ks, lengths, qc, w = _small()
    idx = X.score_topk(qc, w, kc, ks, lengths, False, 64, 512)      # lengths 301 and 1001 > 512
    code, bits = X.status()
    assert code == -7 and bits & X.DEV_ERR_LENGTH
    got = idx.cpu().numpy()
    assert np.all(got[1] == -1)                                     # the bad sequence is skipped
    assert np.all(got[0, 0, :64] >= 0)                              # the good one is served
    assert X.status() == (0, 0)


def test_bounded_wait_expires_cleanly():
    from sparse_attention_token_idx_b200 import binding as X
    case, kc, ks, lengths, qc, w = _small()
    try:
        X.debug_set(1, 20_000_000)                   # 20 ms budget, one wait on a barrier nobody signals
        X.score_topk(qc, w, kc, ks, lengths, False, 64, 1001)
        code, bits = X.status()
        assert code == -7 and bits & X.DEV_ERR_TIMEOUT
    finally:
        X.debug_set(0, 0)
    # the context is still usable and results are right afterwards
    idx = X.score_topk(qc, w, kc, ks, lengths, False, 64, 1001)
    assert X.status() == (0, 0)
    assert np.all(idx.cpu().numpy() >= 0)


def _prefill():
    from tests.helpers import gpu_queries, gpu_state
    case = synth.make_case("fault-prefill", 77, 2, 130, [200, 900], T_cap=2048, causal=True, fmt=1, k=64)
    kc, ks, lengths = gpu_state(case)
    qc, w = gpu_queries(case)
    return case, kc, ks, lengths, qc, w


def test_prefill_route_bounded_wait_expires_cleanly():
    """The workspace route (flat-partition scorer, then the top-k kernel): a
    scorer CTA that gives up reports a timeout; the next call is served."""
    from sparse_attention_token_idx_b200 import binding as X
    case, kc, ks, lengths, qc, w = _prefill()
    max_len = int(case.lengths.max())
    ws = torch.empty(X.workspace_size(2, 130, max_len, 64), dtype=torch.uint8, device="cuda")
    try:
        X.debug_set(1, 20_000_000)
        X.score_topk(qc, w, kc, ks, lengths, True, 64, max_len, ws=ws)
        code, bits = X.status()
        assert code == -7 and bits & X.DEV_ERR_TIMEOUT
    finally:
        X.debug_set(0, 0)
    idx = X.score_topk(qc, w, kc, ks, lengths, True, 64, max_len, ws=ws)
    ref = X.score_topk(qc, w, kc, ks, lengths, True, 64, max_len)          # the single-kernel path
    assert X.status() == (0, 0)
    assert torch.equal(torch.sort(idx, -1).values, torch.sort(ref, -1).values)


def test_prefill_route_lengths_beyond_max_len_are_reported_and_rows_emptied():
    from sparse_attention_token_idx_b200 import binding as X
    case, kc, ks, lengths, qc, w = _prefill()
    max_len = 400                                    # sequence 1 has 1030 keys
    ws = torch.empty(X.workspace_size(2, 130, max_len, 64), dtype=torch.uint8, device="cuda")
    idx = X.score_topk(qc, w, kc, ks, lengths, True, 64, max_len, ws=ws).cpu().numpy()
    code, bits = X.status()
    assert code == -7 and bits & X.DEV_ERR_LENGTH
    assert np.all(idx[1] == -1)
    assert np.all(idx[0, :, :64][idx[0, :, :64] >= 0] < 330)
    assert X.status() == (0, 0)
