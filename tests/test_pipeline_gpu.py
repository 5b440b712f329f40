"""The indexer call as the pipeline issues it: one fused quantise launch
(queries + new keys) and the fused score + top-k; the CUDA-graph replay of the
same step gives the same result as the eager call."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import bf16_dev, dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", [0, 1])
def test_fused_quant_launch_matches_oracle(fmt):
    from sparse_attention_token_idx_b200 import binding as X
    case = synth.make_case("qa", 500 + fmt, 5, 3, [0, 7, 100, 61, 3], T_cap=128, fmt=fmt)
    kc = torch.full((5, 128, 128), 0x5A, dtype=torch.uint8, device="cuda")
    ks = torch.full((5, 128), 9.0, dtype=torch.float32, device="cuda")
    q_out = torch.empty(case.q.shape, dtype=torch.uint8, device="cuda")
    w_out = torch.empty(case.w_raw.shape, dtype=torch.float32, device="cuda")
    X.quant_queries_append(bf16_dev(case.q), dev(case.w_raw), bf16_dev(case.k_new), dev(case.positions), kc, ks, fmt,
                           q_out, w_out)
    assert X.status() == (0, 0)
    oq, _, ow = O.quant_queries(case.q, case.w_raw, fmt)
    okc = np.full((5, 128, 128), 0x5A, np.uint8)
    oks = np.full((5, 128), 9.0, np.float32)
    O.quant_append(case.k_new, case.positions, okc, oks, fmt)
    np.testing.assert_array_equal(q_out.cpu().numpy(), oq)
    np.testing.assert_array_equal(w_out.cpu().numpy().view(np.uint32), ow.view(np.uint32))
    np.testing.assert_array_equal(kc.cpu().numpy(), okc)
    np.testing.assert_array_equal(ks.cpu().numpy().view(np.uint32), oks.view(np.uint32))


def test_graph_replay_equals_eager_step():
    from sparse_attention_token_idx_b200.pipeline import Indexer
    case = synth.make_case("g", 510, 8, 1, [500, 3000, 16383, 1, 2047, 9000, 12000, 7], T_cap=16384, fmt=1)
    args = (bf16_dev(case.k_new), bf16_dev(case.q), dev(case.w_raw), dev(case.positions), dev(case.lengths))
    ix = Indexer(case.B, case.T_cap, case.fmt, case.k)
    from sparse_attention_token_idx_b200 import binding as X
    for b in range(case.B):
        p = int(case.positions[b])
        if p:
            X.quant_append(bf16_dev(case.k_prior[b:b + 1, :p]), dev(np.zeros(1, np.int32)), ix.k_cache[b:b + 1],
                           ix.k_scale_cache[b:b + 1], case.fmt)
    eager = ix.step(*args, causal=False, max_len=16384).clone()
    g, out = ix.capture(*args, causal=False, max_len=16384)
    out.fill_(-7)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert X.status() == (0, 0)
    np.testing.assert_array_equal(out.cpu().numpy(), eager.cpu().numpy())


@pytest.mark.parametrize("n,positions,causal", [(1, [500, 3000, 16383, 1, 2047, 9000, 12000, 7], False),
                                                (48, [0, 700, 4000, 100, 9000, 12, 16000, 300], True)])
def test_e8m0_scale_storage_selects_the_same_sets(n, positions, causal):
    """Indexer with one e8m0 byte per key (129 cache bytes per key) against the
    fp32 ue8m0 cache, eager and through a CUDA graph."""
    from sparse_attention_token_idx_b200.pipeline import Indexer
    from sparse_attention_token_idx_b200 import binding as X
    positions = [min(p, 16384 - n) for p in positions]
    case = synth.make_case("e8", 520 + n, 8, n, positions, T_cap=16384, causal=causal, fmt=1, k=256)
    args = (bf16_dev(case.k_new), bf16_dev(case.q), dev(case.w_raw), dev(case.positions), dev(case.lengths))
    ixs = [Indexer(case.B, case.T_cap, 1, case.k), Indexer(case.B, case.T_cap, 1, case.k, scale_storage="e8m0")]
    for b in range(case.B):
        p = int(case.positions[b])
        if p:
            kp, z = bf16_dev(case.k_prior[b:b + 1, :p]), dev(np.zeros(1, np.int32))
            X.quant_append(kp, z, ixs[0].k_cache[b:b + 1], ixs[0].k_scale_cache[b:b + 1], 1)
            X.quant_append_e8(kp, z, ixs[1].k_cache[b:b + 1], ixs[1].k_scale_cache[b:b + 1])
    max_len = int(case.lengths.max())
    ref = ixs[0].step(*args, causal=causal, max_len=max_len).clone()
    got = ixs[1].step(*args, causal=causal, max_len=max_len).clone()
    g, out = ixs[1].capture(*args, causal=causal, max_len=max_len)
    out.fill_(-7)
    g.replay()
    torch.cuda.synchronize()
    assert X.status() == (0, 0)
    assert ixs[1].k_scale_cache.dtype == torch.uint8
    assert torch.equal(ixs[0].k_cache, ixs[1].k_cache)
    srt = lambda t: torch.sort(t, -1).values.cpu().numpy()
    np.testing.assert_array_equal(srt(got), srt(ref))
    np.testing.assert_array_equal(srt(out), srt(ref))
