"""Scores (unfused idx_score) against the oracle: within 1e-5·E, −inf exactly
where masked.  Shapes span several key tiles, ragged tails, clusters of CTAs
(few sequences), causal prefill and chunked prefill."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import check_scores, gpu_queries, gpu_state, oracle_queries, oracle_state

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, n, positions, T_cap, causal, fmt
    ("decode-ragged", 5, 1, [0, 126, 128, 999, 4095], 4096, False, 0),
    ("decode-one-seq", 1, 1, [1000], 2048, False, 1),
    ("decode-two-rows", 3, 2, [0, 300, 1600], 2048, True, 0),
    ("prefill-causal", 1, 300, [0], 512, True, 0),
    ("prefill-chunked", 2, 261, [200, 517], 1024, True, 1),
    ("prefill-noncausal", 2, 70, [0, 129], 256, False, 0),
]


@pytest.mark.parametrize("name,B,n,positions,T_cap,causal,fmt", CASES)
def test_scores_match_oracle(name, B, n, positions, T_cap, causal, fmt):
    from sparse_attention_token_idx_b200 import binding as X
    case = synth.make_case(name, 200 + len(name), B, n, positions, T_cap=T_cap, causal=causal, fmt=fmt)
    kc, ks, lengths = gpu_state(case)
    qc, w = gpu_queries(case)
    max_len = int(case.lengths.max())
    ld = max_len + 37                              # columns past every length must be −inf
    sc = X.score(qc, w, kc, ks, lengths, causal, max_len, ld=ld)
    assert X.status() == (0, 0)
    okc, oks = oracle_state(case)
    oqc, ow = oracle_queries(case)
    S, E = O.index_scores(oqc, ow, okc, oks, case.lengths, causal, ncols=ld)
    check_scores(sc.cpu().numpy(), S, E)


def test_scores_ld_shorter_than_length_writes_only_ld_columns():
    from sparse_attention_token_idx_b200 import binding as X
    case = synth.make_case("ld", 250, 2, 1, [700, 300], T_cap=1024)
    kc, ks, lengths = gpu_state(case)
    qc, w = gpu_queries(case)
    ld = 512
    buf = torch.empty((2, 1, ld), device="cuda")
    X.score(qc, w, kc, ks, lengths, False, 701, ld=ld, out=buf)
    assert X.status() == (0, 0)
    okc, oks = oracle_state(case)
    oqc, ow = oracle_queries(case)
    S, E = O.index_scores(oqc, ow, okc, oks, case.lengths, False, ncols=ld)
    check_scores(buf.cpu().numpy(), S, E)


def test_logits_exact_single_head_probe():
    """One-hot weights and unit key scales turn S into ReLU(q·k) of one head, so
    the FP8 tensor-core accumulation can be compared with the exact dot product
    on adversarial codes (wide magnitude spread, heavy cancellation).  The
    observed error stays within a few fp32 roundings of Σ|q·k| (2^-20 bound)."""
    from sparse_attention_token_idx_b200 import binding as X
    rng = np.random.default_rng(9)
    B, T = 1, 512
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    kc = rng.choice(finite, (B, T, 128)).astype(np.uint8)
    qc = rng.choice(finite, (B, 1, 64, 128)).astype(np.uint8)
    kc[0, :64, :] = 0x7E                  # 448s
    kc[0, 64:128, ::2] = 0x01             # 2^-9 mixed with large values
    ks = np.ones((B, T), np.float32)
    lengths = np.array([T], np.int32)
    for h in (0, 17, 63):
        w = np.zeros((B, 1, 64), np.float32)
        w[0, 0, h] = 1.0
        sc = X.score(torch.from_numpy(qc).cuda(), torch.from_numpy(w).cuda(), torch.from_numpy(kc).cuda(),
                     torch.from_numpy(ks).cuda(), torch.from_numpy(lengths).cuda(), False, T, ld=T)
        S, _ = O.index_scores(qc, w, kc, ks, lengths, False, ncols=T)
        dec = O.e4m3_values()
        mag = np.abs(dec[kc[0]]) @ np.abs(dec[qc[0, 0, h]])      # Σ|q·k| per key
        err = np.abs(sc.cpu().numpy()[0, 0] - S[0, 0])
        ratio = (err / np.maximum(mag, 1e-30)).max()
        print(f"head {h}: max |err| / sum|q*k| = {ratio:.3e} (2^{np.log2(max(ratio, 1e-300)):.2f})")
        assert np.all(err <= 2.0 ** -20 * mag + 1e-30), err.max()


VISIBLE = [
    # name, B, n, positions, T_cap, causal, fmt — decode batches, ragged and zero
    # lengths, causal and chunked prefill, more row blocks than SMs
    ("decode-batch", 150, 1, None, 2048, False, 1),
    ("decode-ragged", 5, 1, [0, 126, 128, 999, 4095], 4096, False, 0),
    ("prefill-causal", 1, 300, [0], 512, True, 0),
    ("prefill-chunked", 2, 261, [200, 517], 1024, True, 1),
    ("many-blocks", 3, 200, [0, 100, 600], 1024, True, 0),
]


@pytest.mark.parametrize("name,B,n,positions,T_cap,causal,fmt", VISIBLE)
def test_score_visible_matches_oracle(name, B, n, positions, T_cap, causal, fmt):
    """idx_score_visible (flat partition, one persistent CTA per SM): the oracle's
    scores on every visible key, −inf up to the end of each row's last key tile."""
    from sparse_attention_token_idx_b200 import binding as X
    kw = dict(lengths_draw=(1, T_cap - 1)) if positions is None else {}
    case = synth.make_case(name, 250 + len(name), B, n, positions, T_cap=T_cap, causal=causal, fmt=fmt, **kw)
    kc, ks, lengths = gpu_state(case)
    qc, w = gpu_queries(case)
    max_len = int(case.lengths.max())
    ld = max_len + 5
    out = torch.full((B, n, ld), 12345.0, dtype=torch.float32, device="cuda")
    X.score_visible(qc, w, kc, ks, lengths, causal, max_len, ld=ld, out=out)
    assert X.status() == (0, 0)
    got = out.cpu().numpy()
    okc, oks = oracle_state(case)
    oqc, ow = oracle_queries(case)
    S, E = O.index_scores(oqc, ow, okc, oks, case.lengths, causal, ncols=ld)
    for b in range(B):
        blocks = {}
        for i in range(n):
            vis = O.visible_count(int(case.lengths[b]), n, i, causal)
            blk = i // 4 if n > 2 else i
            blocks[blk] = max(blocks.get(blk, 0), vis)
        for i in range(n):
            vis = O.visible_count(int(case.lengths[b]), n, i, causal)
            end = min(ld, -(-blocks[i // 4 if n > 2 else i] // 128) * 128)   # the row block's last key tile
            check_scores(got[b, i:i + 1, :vis][None], S[b, i:i + 1, :vis][None], E[b, i:i + 1, :vis][None])
            assert np.all(np.isneginf(got[b, i, vis:end])), "−inf up to the end of the last key tile"
            assert np.all(got[b, i, end:] == 12345.0), "columns past the last key tile untouched"
