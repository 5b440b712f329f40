"""The projections (idx_project) against the oracle's float64 products, and the
chain projections → front end → cache / queries / weights against the oracle
started from the GPU's own projection outputs.

Tolerance, from the arithmetic (u = 2^-24, the fp32 unit roundoff): each
output is a K-term sum of exact products accumulated in fp32 by the tensor
cores, split-K slices added in a fixed order.  Any fp32 summation of K terms is
within γ = 2·K·u·Σ|a·b| of the exact sum; the bf16 outputs q, k round that
once, so they may differ from the oracle's correctly rounded value by γ plus
one bf16 ulp.  The head weights multiply x by the fp32 weights split into three
bf16 parts (hi + mid + lo = w within u·|w|, every product exact in fp32), sum
each part's K products in fp32 and add the three sums with two fp32 additions:
γ_w = (2·K + 4)·u·Σ|a·b| (split, three group sums dominated by hi, two
additions), plus one fp32 ulp."""
import numpy as np
import pytest
import torch

from oracle import indexer as O
from sparse_attention_token_idx_b200 import synth
from tests.helpers import bf16_dev, dev

pytestmark = pytest.mark.gpu


def _ulp(v, mant_bits):
    v = np.maximum(np.abs(v), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(v)).astype(np.int64) - mant_bits)


def _check(got, want, a, b, mant_bits, what, extra_terms=0):
    """got, want: float64 values [T, N]; a [T, K], b [N, K] the exact inputs."""
    K = a.shape[1]
    gamma = (2.0 * K + extra_terms) * 2.0 ** -24 * (np.abs(a) @ np.abs(b).T)
    tol = gamma + _ulp(np.abs(want) + gamma, mant_bits)
    err = np.abs(got - want)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} outputs out of tolerance, worst {np.max(err - tol):.3e}"


CASES = [
    # tokens, hidden, q_lora
    (1, 256, 512),
    (5, 256, 512),
    (130, 1024, 1536),
    (128, synth.HIDDEN, synth.Q_LORA),       # one decode token per sequence, B = 128: split over K
    (1024, 1024, synth.Q_LORA),              # enough rows for 256-column tiles, no split
]


@pytest.mark.parametrize("tokens,hidden,q_lora", CASES)
def test_projections_within_fp32_accumulation_bound(tokens, hidden, q_lora):
    from sparse_attention_token_idx_b200 import binding as X
    pc = synth.make_proj_case(40 + tokens, tokens, hidden=hidden, q_lora=q_lora)
    q, k, w = X.project(bf16_dev(pc.x), bf16_dev(pc.qr), bf16_dev(pc.wq_b), bf16_dev(pc.wk), dev(pc.w_proj))
    assert X.status() == (0, 0)
    oq, ok, ow = O.project(pc.x, pc.qr, pc.wq_b, pc.wk, pc.w_proj)
    gq = O.bf16_bits_to_f64(q.view(torch.int16).cpu().numpy().view(np.uint16)).reshape(tokens, -1)
    gk = O.bf16_bits_to_f64(k.view(torch.int16).cpu().numpy().view(np.uint16))
    gw = w.cpu().numpy().astype(np.float64)
    x, qr = O.bf16_bits_to_f64(pc.x), O.bf16_bits_to_f64(pc.qr)
    _check(gq, O.bf16_bits_to_f64(oq).reshape(tokens, -1), qr, O.bf16_bits_to_f64(pc.wq_b), 7, "q_proj")
    _check(gk, O.bf16_bits_to_f64(ok), x, O.bf16_bits_to_f64(pc.wk), 7, "k_proj")
    _check(gw, ow.astype(np.float64), x, pc.w_proj.astype(np.float64), 23, "w_raw", extra_terms=4)
    # most outputs round to the same bf16 value as the exact product
    assert np.mean(gq == O.bf16_bits_to_f64(oq).reshape(tokens, -1)) > 0.95


def test_projections_need_the_workspace_and_are_deterministic():
    """The workspace holds the split head weights and the split-K partial sums:
    a smaller one is refused before anything is enqueued (IDX_ERR_SCRATCH), none
    at all with IDX_ERR_NULL.  With fixed-order sums two calls agree bit for bit."""
    from sparse_attention_token_idx_b200 import binding as X
    pc = synth.make_proj_case(77, 128, hidden=synth.HIDDEN, q_lora=synth.Q_LORA)
    args = (bf16_dev(pc.x), bf16_dev(pc.qr), bf16_dev(pc.wq_b), bf16_dev(pc.wk), dev(pc.w_proj))
    need = X.project_workspace_size(128, synth.HIDDEN, synth.Q_LORA)
    assert need >= 3 * 64 * synth.HIDDEN * 2
    with pytest.raises(X.IdxError, match=r"status -10,"):
        X.project(*args, ws=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(X.IdxError, match=r"status -1,"):
        X.project(*args, ws=torch.empty(0, dtype=torch.uint8, device="cuda"))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    q0, k0, w0 = X.project(*args, ws=ws)
    q1, k1, w1 = X.project(*args, ws=ws)
    assert torch.equal(q0, q1) and torch.equal(k0, k1) and torch.equal(w0, w1)
    assert X.status() == (0, 0)


def test_hidden_state_to_cache_chain_is_bit_exact_given_the_projections():
    """Indexer.step_hidden: projections, then RoPE / LayerNorm / rotation /
    quantisation / append, then score + top-k.  Given the GPU's own projection
    outputs, the oracle's front end must produce the same cache bytes, query
    codes and folded weights bit for bit."""
    from sparse_attention_token_idx_b200 import binding as X
    from sparse_attention_token_idx_b200.pipeline import Indexer
    B, n, T_cap, hidden, q_lora = 3, 5, 512, 1024, 1536
    pc = synth.make_proj_case(11, B * n, hidden=hidden, q_lora=q_lora)
    rng = np.random.default_rng(12)
    positions = np.array([40, 0, 300], np.int32)
    lengths = positions + n
    pos = positions[:, None] + np.arange(n)[None, :]
    theta = 10000.0 ** (-np.arange(32) / 32.0)
    ang = pos[..., None] * theta
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    gain = (1 + 0.2 * rng.standard_normal(128)).astype(np.float32)
    bias = (0.2 * rng.standard_normal(128)).astype(np.float32)
    ix = Indexer(B, T_cap, 0, 64)
    idx = ix.step_hidden(bf16_dev(pc.x).view(B, n, hidden), bf16_dev(pc.qr).view(B, n, q_lora), bf16_dev(pc.wq_b),
                         bf16_dev(pc.wk), dev(pc.w_proj), dev(cos), dev(sin), dev(gain), dev(bias), dev(positions),
                         dev(lengths), causal=True, max_len=int(lengths.max()))
    assert X.status() == (0, 0)
    qp, kp, wr = (t.cpu() for t in ix.projections())
    qp = qp.view(torch.int16).numpy().view(np.uint16).reshape(B, n, 64, 128)
    kp = kp.view(torch.int16).numpy().view(np.uint16).reshape(B, n, 128)
    wr = wr.numpy().reshape(B, n, 64)
    oq, okey = O.front(qp, kp, cos, sin, gain, bias, 1e-6)
    codes, _, w = O.quant_queries(oq, wr, 0)
    np.testing.assert_array_equal(ix._bufs["q_fp8"].cpu().numpy(), codes)
    np.testing.assert_array_equal(ix._bufs["w"].cpu().numpy().view(np.uint32), w.view(np.uint32))
    kc = np.zeros((B, T_cap, 128), np.uint8)
    ks = np.zeros((B, T_cap), np.float32)
    O.quant_append(okey, positions, kc, ks, 0)
    got_kc = ix.k_cache.cpu().numpy()
    got_ks = ix.k_scale_cache.cpu().numpy()
    for b in range(B):
        p = int(positions[b])
        np.testing.assert_array_equal(got_kc[b, p:p + n], kc[b, p:p + n])
        np.testing.assert_array_equal(got_ks[b, p:p + n].view(np.uint32), ks[b, p:p + n].view(np.uint32))
    assert idx.shape == (B, n, 64)
