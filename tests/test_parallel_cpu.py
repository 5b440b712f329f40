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
