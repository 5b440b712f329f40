"""Multi-rank host logic on CPU: two gloo ranks shard a batch of sequences,
each rank checks the oracle on its own shard, and the timing reduction takes
the maximum over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_token_idx_b200.parallel import max_over_ranks, shard_range, weak_scaling_total


def test_shard_range_covers_every_item_once():
    for n in [0, 1, 7, 128, 129]:
        for world in [1, 2, 3, 8]:
            seen = []
            for r in range(world):
                lo, hi = shard_range(n, r, world)
                seen.extend(range(lo, hi))
                assert hi - lo in (n // world, n // world + 1)
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import indexer as O
        from sparse_attention_token_idx_b200 import synth
        case = synth.make_case("dp", 77, 6, 1, [10, 40, 3, 90, 25, 60], T_cap=128, k=16)
        lo, hi = shard_range(case.B, rank, world)
        kc = np.zeros((case.B, 128, 128), np.uint8)
        ks = np.zeros((case.B, 128), np.float32)
        for b in range(lo, hi):
            p = int(case.positions[b])
            O.quant_append(case.k_prior[b:b + 1, :p], [0], kc[b:b + 1], ks[b:b + 1], 0)
        st = {"k_cache": kc[lo:hi], "k_scale_cache": ks[lo:hi]}
        idx, *_ = O.indexer_step(st, case.k_new[lo:hi], case.q[lo:hi], case.w_raw[lo:hi], case.positions[lo:hi],
                                 False, 16, 0)
        mx = max_over_ranks([float(rank) + 0.5, 10.0 - rank])
        total = weak_scaling_total(hi - lo)
        q.put((rank, lo, hi, idx.shape, mx, total))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [(r[1], r[2]) for r in res] == [(0, 3), (3, 6)]
    assert all(r[3] == (3, 1, 16) for r in res)
    assert all(r[4] == [1.5, 10.0] for r in res)          # max over ranks, element-wise
    assert all(r[5] == 6 for r in res)


# ---------------------------------------------------------------------------- split-T
from sparse_attention_token_idx_b200.parallel import exchange_candidates, key_slice, slice_counts  # noqa: E402


def test_key_slice_covers_every_position_once():
    for T in [0, 1, 127, 128, 1000, 65536]:
        for world in [1, 2, 3, 8]:
            seen = []
            for r in range(world):
                lo, hi = key_slice(T, r, world)
                assert lo % 128 == 0 or lo == T
                seen.extend(range(lo, hi))
            assert seen == list(range(T))
    with pytest.raises(ValueError):
        key_slice(128, 1, 1)


def test_slice_counts_add_up_to_the_lengths():
    import torch
    L = np.array([0, 1, 200, 511, 512, 513, 1000], np.int32)
    tot = np.zeros_like(L)
    for r in range(3):
        lo, hi = key_slice(1024, r, 3)
        c = slice_counts(L, lo, hi)
        assert c.dtype == np.int32 and np.all((c >= 0) & (c <= hi - lo))
        assert np.array_equal(slice_counts(torch.from_numpy(L), lo, hi).numpy(), c)
        tot += c
    assert np.array_equal(tot, np.minimum(L, 1024))


def _split_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch
        from oracle import indexer as O
        from sparse_attention_token_idx_b200 import synth
        T, k = 1024, 48
        # two sequences: one reaching into every slice, one ending inside rank 0's slice
        case = synth.make_case("split", 91, 2, 1, [900, 300], T_cap=T, k=k)
        kc = np.zeros((case.B, T, 128), np.uint8)
        ks = np.zeros((case.B, T), np.float32)
        for b in range(case.B):
            p = int(case.positions[b])
            O.quant_append(case.k_prior[b:b + 1, :p], [0], kc[b:b + 1], ks[b:b + 1], 0)
        O.quant_append(case.k_new, case.positions, kc, ks, 0)
        qc, _, w = O.quant_queries(case.q, case.w_raw, 0)

        def candidates(r):   # rank r's slice top-k as (score bits, global position) pairs
            lo, hi = key_slice(T, r, world)
            cnt = slice_counts(case.lengths, lo, hi)
            S, _ = O.index_scores(qc, w, kc[:, lo:hi], ks[:, lo:hi], cnt, False, ncols=hi - lo, with_bound=False)
            c = np.zeros((case.B, k, 2), np.int32)
            for b in range(case.B):
                t = O.topk_row(S[b, 0], int(cnt[b]), k)
                ok = t >= 0
                c[b, :, 0] = np.where(ok, S[b, 0][np.maximum(t, 0)], -np.inf).astype(np.float32).view(np.int32)
                c[b, :, 1] = np.where(ok, t + lo, -1)
            return c

        got = exchange_candidates(torch.from_numpy(candidates(rank))).numpy()
        expect = np.stack([candidates(r) for r in range(world)])
        S, _ = O.index_scores(qc, w, kc, ks, case.lengths, False, with_bound=False)
        merged_ok = []
        for b in range(case.B):
            cs = got[:, b, :, 0].reshape(-1).view(np.float32).astype(np.float64)
            cp = got[:, b, :, 1].reshape(-1)
            valid = cp >= 0
            full = O.topk_row(S[b, 0], int(case.lengths[b]), k)
            pick = O.topk_row(cs[valid], int(valid.sum()), k)
            merged = cp[valid][pick[pick >= 0]]
            merged_ok.append(set(merged.tolist()) == set(full[full >= 0].tolist()))
        q.put((rank, bool(np.array_equal(got, expect)), merged_ok))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_t_exchange_and_merge():
    """The all-gather lays candidates out rank-major, and the k best of the
    union of slice top-ks are the whole sequence's top-k (oracle scores)."""
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[1] for r in res), "exchanged candidates are not in rank order"
    assert all(all(r[2]) for r in res), "merged slice top-ks differ from the full top-k"


def _orchestration_worker(rank, world, port, q):
    """split_t_decode on CPU tensors, the library calls replaced by stand-ins
    computed with the oracle: the host logic (slice counts, the one-key
    stand-in for empty slices, position offsets, the exchange) runs as is."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch
        from oracle import indexer as O
        from sparse_attention_token_idx_b200 import binding as X
        from sparse_attention_token_idx_b200 import parallel as PL
        from sparse_attention_token_idx_b200 import synth

        def score_visible(q_fp8, w, kc, ks, lengths, causal, max_len, stream=None):
            S, _ = O.index_scores(q_fp8.numpy(), w.numpy(), kc.numpy(), ks.numpy(), lengths.numpy(), causal,
                                  ncols=max_len, with_bound=False)
            return torch.from_numpy(S.astype(np.float32))

        def topk(scores, lengths, causal, k, max_len, stream=None):
            return torch.from_numpy(O.topk(scores.numpy().astype(np.float64), lengths.numpy(), causal, k))

        def gather_scores(scores, idx, offset, counts=None, stream=None):
            s, i = scores.numpy(), idx.numpy()
            c = counts.numpy() if counts is not None else np.full(len(i), s.shape[1])
            valid = (i >= 0) & (i < c[:, None])
            out = np.zeros(i.shape + (2,), np.int32)
            out[..., 0] = np.where(valid, np.take_along_axis(s, np.maximum(i, 0), 1), -np.inf).astype(
                np.float32).view(np.int32)
            out[..., 1] = np.where(valid, i + offset, -1)
            return torch.from_numpy(out)

        def merge_topk(cand, k, out=None, stream=None):
            c = cand.numpy()
            G, rows, kin, _ = c.shape
            res = np.full((rows, k), -1, np.int32)
            for r in range(rows):
                sc = c[:, r, :, 0].reshape(-1).view(np.float32).astype(np.float64)
                ps = c[:, r, :, 1].reshape(-1)
                ok = ps >= 0
                pick = O.topk_row(sc[ok], int(ok.sum()), k)
                res[r, :(pick >= 0).sum()] = ps[ok][pick[pick >= 0]]
            return torch.from_numpy(res)

        X.score_visible, X.topk, X.gather_scores, X.merge_topk = score_visible, topk, gather_scores, merge_topk
        T, k = 1024, 40
        case = synth.make_case("split-orch", 93, 3, 1, [1000, 200, 600], T_cap=T, k=k)
        kc = np.zeros((case.B, T, 128), np.uint8)
        ks = np.zeros((case.B, T), np.float32)
        for b in range(case.B):
            p = int(case.positions[b])
            O.quant_append(case.k_prior[b:b + 1, :p], [0], kc[b:b + 1], ks[b:b + 1], 0)
        O.quant_append(case.k_new, case.positions, kc, ks, 0)
        qc, _, w = O.quant_queries(case.q, case.w_raw, 0)
        lo, hi = PL.key_slice(T, rank, world)
        got = PL.split_t_decode(torch.from_numpy(qc), torch.from_numpy(w), torch.from_numpy(kc[:, lo:hi].copy()),
                                torch.from_numpy(ks[:, lo:hi].copy()), torch.from_numpy(case.lengths), lo, hi,
                                k).numpy()
        S, _ = O.index_scores(qc, w, kc, ks, case.lengths, False, with_bound=False)
        same = [set(got[b][got[b] >= 0].tolist()) == set(O.topk_row(S[b, 0], int(case.lengths[b]), k).tolist())
                for b in range(case.B)]
        q.put((rank, same, int((got >= 0).sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_t_decode_orchestration():
    """Rank 1 holds no key of the second sequence (length 201 < 512): its slice
    is scored as one key and dropped; every rank ends with the full top-k."""
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_orchestration_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(all(r[1]) for r in res), "split-T result differs from the whole-sequence top-k"
    assert all(r[2] == 3 * 40 for r in res)


def test_empty_key_slice_contributes_only_empty_candidates():
    """A rank whose slice holds no positions (more ranks than 128-position
    blocks) returns (−inf, −1) pairs without calling the library."""
    import torch
    from sparse_attention_token_idx_b200.parallel import slice_candidates
    lo, hi = key_slice(256, 3, 4)
    assert lo == hi == 256
    c = slice_candidates(torch.zeros((2, 1, 64, 128), dtype=torch.uint8), torch.zeros((2, 1, 64)),
                         torch.zeros((2, 0, 128), dtype=torch.uint8), torch.zeros((2, 0)),
                         torch.tensor([200, 256], dtype=torch.int32), lo, hi, 16)
    assert c.shape == (2, 16, 2) and torch.all(c[..., 1] == -1)
    assert torch.all(torch.isneginf(c[..., 0].contiguous().view(torch.float32)))
