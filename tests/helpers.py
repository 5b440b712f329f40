"""Shared test helpers: moving synthetic inputs to the GPU, running the oracle
and the CUDA path on the same seeded case, and the acceptance checks
(bit-exact bytes; scores within 1e-5·E; top-k as a set up to the tolerance band)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import indexer as O

RTOL = 1e-5   # |S_gpu − S| ≤ RTOL · E,  E = |k_scale| · Σ_h |w·L|


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


# ------------------------------------------------------------------ oracle side
def oracle_state(case, seqs=None):
    """Oracle cache after the prior keys and this call's keys are appended.
    ``seqs`` restricts the work to some sequences (others stay empty)."""
    B = case.B
    seqs = range(B) if seqs is None else seqs
    kc = np.zeros((B, case.T_cap, 128), np.uint8)
    ks = np.zeros((B, case.T_cap), np.float32)
    for b in seqs:
        p = int(case.positions[b])
        if p:
            O.quant_append(case.k_prior[b:b + 1, :p], [0], kc[b:b + 1], ks[b:b + 1], case.fmt)
        O.quant_append(case.k_new[b:b + 1], [p], kc[b:b + 1], ks[b:b + 1], case.fmt)
    return kc, ks


def oracle_queries(case):
    codes, _, w = O.quant_queries(case.q, case.w_raw, case.fmt)
    return codes, w


# ------------------------------------------------------------------ GPU side
def gpu_state(case, B_alloc=None):
    """Device cache [B, T_cap, 128] filled with the prior keys and this call's keys
    through idx_quant_append; returns (k_cache, k_scale_cache, lengths)."""
    from sparse_attention_token_idx_b200 import binding as X
    B = case.B
    kc = torch.zeros((B, case.T_cap, 128), dtype=torch.uint8, device="cuda")
    ks = torch.zeros((B, case.T_cap), dtype=torch.float32, device="cuda")
    P = case.k_prior.shape[1]
    if P:
        if np.all(case.positions == P):
            X.quant_append(bf16_dev(case.k_prior), dev(np.zeros(B, np.int32)), kc, ks, case.fmt)
        else:
            for b in range(B):
                p = int(case.positions[b])
                if p:
                    X.quant_append(bf16_dev(case.k_prior[b:b + 1, :p]), dev(np.zeros(1, np.int32)), kc[b:b + 1],
                                   ks[b:b + 1], case.fmt)
    X.quant_append(bf16_dev(case.k_new), dev(case.positions), kc, ks, case.fmt)
    return kc, ks, dev(case.lengths)


def gpu_queries(case):
    from sparse_attention_token_idx_b200 import binding as X
    return X.quant_queries(bf16_dev(case.q), dev(case.w_raw), case.fmt)


# ------------------------------------------------------------------ checks
def check_scores(gpu: np.ndarray, S: np.ndarray, E: np.ndarray, rtol=RTOL):
    """gpu, S, E: [..., cols]; masked entries of S are −inf and must be −inf on the GPU."""
    masked = np.isneginf(S)
    assert np.all(np.isneginf(gpu[masked])), "masked entries must be -inf"
    v = ~masked
    err = np.abs(gpu[v].astype(np.float64) - S[v])
    bound = rtol * E[v]
    bad = err > bound
    if bad.any():
        i = np.argmax(err - bound)
        raise AssertionError(f"{bad.sum()} scores out of tolerance; worst err {err[i]:.3e} bound {bound[i]:.3e} "
                             f"S {S[v][i]:.6e} gpu {gpu[v][i]:.6e}")


def check_topk_row(got_row: np.ndarray, S: np.ndarray, E: np.ndarray, vis: int, k: int, rtol=RTOL):
    """Top-k of one row as a set.  Positions that must be selected whatever the
    scores' rounding (fewer than k_t others can reach them) must be present;
    positions that at least k_t others certainly beat must be absent."""
    kt = min(k, vis)
    got = np.asarray(got_row[:kt], np.int64)
    assert np.all(np.asarray(got_row[kt:]) == -1), "slots past k_t must hold -1"
    if kt == 0:
        return
    assert got.min() >= 0 and got.max() < vis, "index out of the visible range"
    assert len(np.unique(got)) == kt, "duplicate indices"
    if kt == vis:
        return
    s = S[:vis].astype(np.float64)
    e = rtol * E[:vis]
    lo, hi = s - e, s + e
    hs, ls = np.sort(hi), np.sort(lo)
    reach = len(hi) - np.searchsorted(hs, lo, "left") - 1    # others whose hi ≥ my lo
    beaten = len(lo) - np.searchsorted(ls, hi, "right")      # others whose lo > my hi
    must_in = reach < kt
    must_out = beaten >= kt
    sel = np.zeros(vis, bool)
    sel[got] = True
    missing = np.flatnonzero(must_in & ~sel)
    extra = np.flatnonzero(must_out & sel)
    assert missing.size == 0, f"{missing.size} certain members missing, e.g. {missing[:5]}"
    assert extra.size == 0, f"{extra.size} certain non-members selected, e.g. {extra[:5]}"


def check_topk_exact_row(got_row: np.ndarray, scores: np.ndarray, vis: int, k: int):
    """Top-k of exactly known scores: all strictly above the k_t-th value, and
    the right number of ties at it."""
    kt = min(k, vis)
    got = np.asarray(got_row[:kt], np.int64)
    assert np.all(np.asarray(got_row[kt:]) == -1)
    if kt == 0:
        return
    assert got.min() >= 0 and got.max() < vis and len(np.unique(got)) == kt
    s = scores[:vis]
    tau = np.sort(s)[::-1][kt - 1]
    sel = np.zeros(vis, bool)
    sel[got] = True
    assert np.all(sel[s > tau]), "an element above the threshold is missing"
    assert not np.any(sel[s < tau]), "an element below the threshold is selected"
    assert sel[s == tau].sum() == kt - np.count_nonzero(s > tau)


# ------------------------------------------------------------------ full-size checks in a process pool
def oracle_pool(workers=None):
    """Process pool for oracle work at full size.  Started with spawn, so that
    it is safe after the parent has used the GPU."""
    import multiprocessing
    import os
    from concurrent.futures import ProcessPoolExecutor
    n = workers or max(1, min(32, os.cpu_count() or 1))
    return ProcessPoolExecutor(max_workers=n, mp_context=multiprocessing.get_context("spawn"))


def _one_thread():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def oracle_seq_cache(task):
    """Worker: one sequence's oracle cache (prior keys, then this call's keys).
    task = (k_prior bits [p,128], k_new bits [n,128], T_cap, fmt); returns
    (codes [p+n,128], scales [p+n])."""
    _one_thread()
    k_prior, k_new, T_cap, fmt = task
    p, n = k_prior.shape[0], k_new.shape[0]
    kc = np.zeros((1, p + n, 128), np.uint8)
    ks = np.zeros((1, p + n), np.float32)
    if p:
        O.quant_append(k_prior[None], [0], kc, ks, fmt)
    O.quant_append(k_new[None], [p], kc, ks, fmt)
    return kc[0], ks[0]


def oracle_check_rows(task):
    """Worker: the oracle's scores of some rows of one sequence, then the
    top-k set check of the GPU's rows.  task = (q codes [R,64,128], w [R,64],
    cache codes, scales, visible counts [R], GPU indices [R,k], k, row ids).
    Returns the number of rows checked."""
    _one_thread()
    qc, w, kc, ks, vis, got, k, rows = task
    S, E = O.index_scores_rows(qc, w, kc, ks, vis)
    for r in range(len(vis)):
        try:
            check_topk_row(got[r], S[r], E[r], int(vis[r]), k)
        except AssertionError as e:
            raise AssertionError(f"row {rows[r]}: {e}") from None
    return len(vis)
