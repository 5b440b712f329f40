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


def test_host_pipeline_matches_eager_steps_in_order():
    """Six decode steps fed from pinned host memory through HostPipeline (copies
    and compute overlapped, two slots) select the same sets as six eager steps,
    and leave the same cache.  Each step's new key is built to score at the top
    of every later step (features 1000·N(0, 1): the score grows with the key's
    norm, positive head weights), so a step that ran before the previous
    append landed would miss it."""
    from sparse_attention_token_idx_b200 import binding as X
    from sparse_attention_token_idx_b200.pipeline import HostPipeline, Indexer
    B, steps, k = 4, 6, 64
    base = np.array([1000, 2000, 3000, 500], np.int32)
    case = synth.make_case("hp", 520, B, 1, base, T_cap=4096, k=k, fmt=1)
    q = case.q
    w_raw = np.abs(case.w_raw) + 0.5
    rng = np.random.default_rng(521)
    ks_new = []
    for j in range(steps):
        v = 1000.0 * rng.standard_normal((B, 1, 128)).astype(np.float32)
        ks_new.append((np.ascontiguousarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16))
    ixs = [Indexer(B, case.T_cap, case.fmt, k), Indexer(B, case.T_cap, case.fmt, k)]
    for ix in ixs:
        for b in range(B):
            X.quant_append(bf16_dev(case.k_prior[b:b + 1, :base[b]]), dev(np.zeros(1, np.int32)), ix.k_cache[b:b + 1],
                           ix.k_scale_cache[b:b + 1], case.fmt)
    eager = []
    for j in range(steps):
        pos = base + j
        out = ixs[0].step(bf16_dev(ks_new[j]), bf16_dev(q), dev(w_raw), dev(pos), dev(pos + 1), causal=False,
                          max_len=int(pos.max()) + 1 + steps)
        eager.append(out.cpu().numpy().copy())
    max_len = int(base.max()) + 1 + steps
    hp = HostPipeline(ixs[1], B, 1, causal=False, max_len=max_len)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    h_q, h_w = pin(q.view(np.int16)).view(torch.bfloat16), pin(w_raw)
    outs = []
    for j in range(steps):
        pos = base + j
        h_out = torch.empty((B, 1, k), dtype=torch.int32).pin_memory()
        hp.submit(pin(ks_new[j].view(np.int16)).view(torch.bfloat16), h_q, h_w, pin(pos), pin(pos + 1), h_out)
        outs.append(h_out)
    hp.join()
    torch.cuda.synchronize()
    assert X.status() == (0, 0)
    for j in range(steps):
        got = outs[j].numpy()
        for b in range(B):
            assert set(got[b, 0].tolist()) == set(eager[j][b, 0].tolist()), f"step {j} sequence {b}"
            newer = set(range(base[b], base[b] + j))                # keys appended by the earlier steps
            assert newer <= set(got[b, 0].tolist()), f"step {j} sequence {b} misses an earlier step's key"
    assert torch.equal(ixs[0].k_cache, ixs[1].k_cache) and torch.equal(ixs[0].k_scale_cache, ixs[1].k_scale_cache)


def test_host_pipeline_packed_inputs_match_separate_ones():
    """The same decode step submitted from host_inputs() views (one upload)
    and from separate pinned tensors (five uploads) selects the same sets."""
    from sparse_attention_token_idx_b200 import binding as X
    from sparse_attention_token_idx_b200.pipeline import HostPipeline, Indexer
    B, k = 3, 64
    case = synth.make_case("hp-packed", 530, B, 1, [700, 1500, 90], T_cap=2048, k=k, fmt=0)
    outs = []
    for packed in (False, True):
        ix = Indexer(B, case.T_cap, case.fmt, k)
        for b in range(B):
            p = int(case.positions[b])
            X.quant_append(bf16_dev(case.k_prior[b:b + 1, :p]), dev(np.zeros(1, np.int32)), ix.k_cache[b:b + 1],
                           ix.k_scale_cache[b:b + 1], case.fmt)
        hp = HostPipeline(ix, B, 1, causal=False, max_len=int(case.lengths.max()))
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
        srcs = (pin(case.k_new.view(np.int16)).view(torch.bfloat16), pin(case.q.view(np.int16)).view(torch.bfloat16),
                pin(case.w_raw), pin(case.positions), pin(case.lengths))
        if packed:
            hs = hp.host_inputs()
            for h, src in zip(hs, srcs):
                h.copy_(src)
            assert hp._packed_of(hs) is not None
        else:
            hs = srcs
            assert hp._packed_of(hs) is None
        h_out = torch.empty((B, 1, k), dtype=torch.int32).pin_memory()
        hp.submit(*hs, h_out)
        hp.join()
        torch.cuda.synchronize()
        assert X.status() == (0, 0)
        outs.append(h_out.numpy().copy())
    for b in range(B):
        assert set(outs[0][b, 0].tolist()) == set(outs[1][b, 0].tolist())
