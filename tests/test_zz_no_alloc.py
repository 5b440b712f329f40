"""idx_score_topk_noalloc — the score + top-k entry point for callers that
cannot allocate device memory when they call (for example while their stream
is being captured into a CUDA graph): it keeps the prefill score workspace in
a fixed buffer of the library instead of a caller-provided one.

Checked through the C ABI against idx_score_topk with a caller workspace, on
consecutive calls (the fixed buffer keeps the previous call's contents), and
for the size limit.  Collected last (file name) so that a failure here does
not hide the other tests' results; it also runs alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_token_idx_b200 import synth
from tests.helpers import gpu_queries, gpu_state

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, n, positions, T_cap, causal, fmt, k
    ("prefill", 1, 300, [0], 512, True, 0, 64),
    ("chunked", 2, 130, [900, 2500], 4096, True, 1, 512),
]


def _prepare(name, B, n, positions, T_cap, causal, fmt, k):
    case = synth.make_case(name, 700 + len(name), B, n, positions, T_cap=T_cap, causal=causal, fmt=fmt, k=k)
    kc, ks, lengths = gpu_state(case)
    qc, w = gpu_queries(case)
    return case, kc, ks, lengths, qc, w


def _with_workspace(X, case, kc, ks, lengths, qc, w):
    max_len = int(case.lengths.max())
    ws = torch.empty(X.workspace_size(case.B, case.n, max_len, case.k), dtype=torch.uint8, device="cuda")
    return X.score_topk(qc, w, kc, ks, lengths, case.causal, case.k, max_len, ws=ws).cpu().numpy()


def _noalloc(X, case, kc, ks, lengths, qc, w):
    lib = X.load()
    max_len = int(case.lengths.max())
    out = torch.full((case.B, case.n, case.k), -7, dtype=torch.int32, device="cuda")
    code = lib.idx_score_topk_noalloc(qc.data_ptr(), w.data_ptr(), kc.data_ptr(), ks.data_ptr(), lengths.data_ptr(),
                                      case.B, case.n, case.T_cap, max_len, int(case.causal), case.k, out.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert code == 0, lib.idx_error_string(code)
    return out.cpu().numpy()


def _same_sets(a, b):
    assert a.shape == b.shape
    np.testing.assert_array_equal(np.sort(a, axis=-1), np.sort(b, axis=-1))


def test_noalloc_matches_the_workspace_path_on_consecutive_calls():
    from sparse_attention_token_idx_b200 import binding as X
    prepared = [_prepare(*c) for c in CASES]
    refs = [_with_workspace(X, *p) for p in prepared]
    # two different calls in a row, then the first again: each must match
    for i in (0, 1, 0):
        got = _noalloc(X, *prepared[i])
        _same_sets(got, refs[i])
    assert X.status() == (0, 0)


def test_noalloc_rejects_calls_beyond_its_scratch():
    from sparse_attention_token_idx_b200 import binding as X
    lib = X.load()
    tiny_u8 = torch.zeros(64, dtype=torch.uint8, device="cuda")
    tiny_f = torch.zeros(64, dtype=torch.float32, device="cuda")
    tiny_i = torch.zeros(64, dtype=torch.int32, device="cuda")
    # 1 × 4097 rows × 4097 columns of fp32 scores exceed the 64 MiB buffer; rejected before any launch
    code = lib.idx_score_topk_noalloc(tiny_u8.data_ptr(), tiny_f.data_ptr(), tiny_u8.data_ptr(), tiny_f.data_ptr(),
                                      tiny_i.data_ptr(), 1, 4097, 8192, 4097, 1, 2048, tiny_i.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert code == -10
    assert b"scratch" in lib.idx_error_string(code)
    assert X.status() == (0, 0)



def test_noalloc_first_call_decode_shaped_then_prefill_allocates_nothing():
    """The first call here is decode-shaped: in a fresh process it is the call
    that looks up the fixed buffer's address, whatever its shape.  A
    prefill-shaped call after it must still match the workspace path, and a
    call leaves the device's free memory exactly as it was (no allocation)."""
    from sparse_attention_token_idx_b200 import binding as X
    lib = X.load()
    dec = _prepare("decode", 3, 1, [1000, 77, 3000], 4096, False, 0, 256)
    got_dec = _noalloc(X, *dec)
    _same_sets(got_dec, _with_workspace(X, *dec))
    case, kc, ks, lengths, qc, w = _prepare(*CASES[1])
    ref = _with_workspace(X, case, kc, ks, lengths, qc, w)
    max_len = int(case.lengths.max())
    out = torch.full((case.B, case.n, case.k), -7, dtype=torch.int32, device="cuda")
    args = (qc.data_ptr(), w.data_ptr(), kc.data_ptr(), ks.data_ptr(), lengths.data_ptr(), case.B, case.n, case.T_cap,
            max_len, int(case.causal), case.k, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out.fill_(-7)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        assert lib.idx_score_topk_noalloc(*args) == 0
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
        _same_sets(out.cpu().numpy(), ref)
    assert X.status() == (0, 0)
