"""Benchmark of the lightning-indexer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ours|reference]
                    [--no-prefill] [--no-cpu-baseline]
    python bench.py --row merge|front|project128|project4096|mla [--steps K] [--warmup W]

A step is one whole indexer call on one batch: append the new keys to the FP8
cache (rotate + quantise + store), quantise the queries and fold the head
weights, then score + top-k over every visible cached key.  The headline
workload is the bandwidth-bound decode case (B = 128 sequences, 16 384 cached
keys each, ue8m0 scales, k = 2048): its 277 MB FP8 cache is larger than the
126 MB L2, so consecutive steps stream it from HBM.  The same run then times
the two prefill workloads (4096 causal rows from position 0; 2 × 2048 rows
appended at 14 336) and reports them under "prefill" with their FP8 TFLOP/s
against the tensor peak; their steps are timed one by one with an L2 flush
between them.  --workload 0…4 times one workload alone.

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
sequences (weak scaling, no data-path collective); times are the max over
ranks.  ``--impl reference`` times the CPU oracle (the only reference
implementation there is) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = 2
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_PER_BF16 = 2.0            # nominal dense fp8 : bf16 tensor ratio on B200
DATASHEET_FP8_TFLOPS = 4500.0  # B200 dense FP8, datasheet (context beside the measured-derived peak)
NOMINAL_HBM_GBS = 8000.0      # HBM3e nominal figure the decode target is also quoted against
PREFILL_WORKLOADS = (3, 4)
KEY_BYTES = 128 + 4           # one cached key: 128 e4m3 codes + fp32 scale
ROW_BYTES_IN = 64 * 128 + 64 * 4   # one query row: 64 heads of e4m3 codes + 64 fp32 weights
PROFILE_SCORE = os.path.join(ROOT, "profiles", "score_topk_decode_b128_t16384.md")
KERNEL_SOURCES = ["score.cu", "select.cuh", "ptx.cuh"]
# the prefill scorer's capture (workload 3, one launch) and the sources it was taken from
PROFILE_FLAT = os.path.join(ROOT, "profiles", "flat_score_prefill_b1_s4096.md")
FLAT_SOURCES = ["flat_score.cu", "epilogue.cuh", "ptx.cuh"]
FLAT_PROFILE_WORKLOAD = 3


def env_rank():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return d.get("hbm_gbs"), d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def kernel_source_hash(files=None):
    h = hashlib.sha256()
    for f in files or KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "sparse_attention_token_idx_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profile_values(path, files):
    """The `- key: value` lines of a committed ncu summary, or None when it is
    missing or its source_sha256 no longer matches the kernel's sources."""
    try:
        kv = {}
        for line in open(path):
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                kv[k.strip()] = v.strip().strip("`")
        return kv if kv.get("source_sha256") == kernel_source_hash(files) else None
    except Exception:
        return None


def profile_traffic(path, launch_units):
    """DRAM bytes per launch from a committed ncu summary, scaled to this launch's
    units, or None when the summary is missing or the kernel source changed."""
    kv = profile_values(path, KERNEL_SOURCES)
    try:
        return float(kv["dram_bytes_per_key"]) * launch_units if kv else None
    except (KeyError, ValueError):
        return None


def flat_profile_traffic(widx):
    """DRAM bytes of one prefill-scorer launch, from the committed capture of the
    workload it was taken on (None for other workloads or a changed source)."""
    if widx != FLAT_PROFILE_WORKLOAD:
        return None
    kv = profile_values(PROFILE_FLAT, FLAT_SOURCES)
    try:
        return float(kv["dram_bytes_per_launch"]) if kv else None
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = [name for bit, name in self.REASONS.items() if self.reasons & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------- workload
def workload_numbers(case):
    """Algorithmic per-step units: keys scored, bytes the fused kernel must move, FLOPs."""
    n = case.n
    keys = 0
    for b in range(case.B):
        L = int(case.lengths[b])
        if case.causal:
            keys += int(np.arange(L - n + 1, L + 1).sum())    # row i sees L - n + i + 1 keys
        else:
            keys += L * n
    flops = 2 * 64 * 128 * keys
    key_rows = int(case.lengths.sum())                  # each cached key read once per launch
    rows = case.B * n
    score_bytes = key_rows * KEY_BYTES + rows * (ROW_BYTES_IN + 4 * case.k) + case.B * 4
    return keys, flops, key_rows, score_bytes


def l2_flush_buffer(torch, dev):
    """A buffer twice the L2 size; writing it evicts the previous step's lines."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size or (126 << 20)
    return torch.empty(2 * l2, dtype=torch.uint8, device=dev)


def measure(args, widx, dev, world, headline):
    """One workload on this rank's GPU: fill the cache, capture the step in a
    CUDA graph, warm up, then time K whole steps, the dominant kernel(s) on
    their own, and K end-to-end steps from pinned host memory.  Decode steps
    stream a cache larger than L2 back to back; prefill steps are timed one
    by one with an L2 flush between them (not timed)."""
    import torch
    import torch.distributed as dist

    from sparse_attention_token_idx_b200 import binding as X
    from sparse_attention_token_idx_b200 import synth
    from sparse_attention_token_idx_b200.parallel import max_over_ranks
    from sparse_attention_token_idx_b200.pipeline import HostPipeline, Indexer

    case = synth.workload(widx)
    B, n = case.B, case.n
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    e8m0 = headline and getattr(args, "scale_storage", "f32") == "e8m0"
    if e8m0 and (case.fmt != 1 or case.n > 2):
        raise SystemExit("--scale-storage e8m0 applies to the ue8m0 decode workload (2)")
    ix = Indexer(B, case.T_cap, case.fmt, case.k, device=dev, scale_storage="e8m0" if e8m0 else "f32")
    P = case.k_prior.shape[1]
    if P:
        if np.all(case.positions == P):
            ix.append(bf(case.k_prior), dv(np.zeros(B, np.int32)))
        else:
            for b in range(B):
                p = int(case.positions[b])
                if p:
                    X.quant_append(bf(case.k_prior[b:b + 1, :p]), dv(np.zeros(1, np.int32)), ix.k_cache[b:b + 1],
                                   ix.k_scale_cache[b:b + 1], case.fmt)
    k_new, q, w_raw = bf(case.k_new), bf(case.q), dv(case.w_raw)
    positions, lengths = dv(case.positions), dv(case.lengths)
    max_len = int(case.lengths.max())
    out = torch.empty((B, n, case.k), dtype=torch.int32, device=dev)
    q_fp8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
    w = torch.empty(w_raw.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    keys, flops, key_rows, score_bytes = workload_numbers(case)
    if e8m0:   # one scale byte per cached key instead of four
        score_bytes -= 3 * key_rows

    # the kernel the roofline is about: the tcgen05 scorer writing the
    # workspace when the step uses one (its top-k timed apart), else the fused
    # score + top-k
    ws_bytes = X.workspace_size(B, n, max_len, case.k)
    if ws_bytes:   # the scorer writes fp32 score rows instead of indices
        score_bytes += B * n * (4 * max_len - 4 * case.k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    sc_view = ws.view(torch.float32).view(B, n, max_len) if ws_bytes else None

    def score_only():
        if ws_bytes:
            X.score_visible(q_fp8, w, ix.k_cache, ix.k_scale_cache, lengths, case.causal, max_len, ld=max_len,
                            out=sc_view)
        else:
            X.score_topk_ex(q_fp8, w, ix.k_cache, ix.k_scale_cache, lengths, case.causal, case.k, max_len, out=out)

    def topk_only():
        X.topk(sc_view, lengths, case.causal, case.k, max_len, out=out)

    graph, g_out = ix.capture(k_new, q, w_raw, positions, lengths, causal=case.causal, max_len=max_len)
    flush = None if key_rows * KEY_BYTES > 2 * 126e6 else l2_flush_buffer(torch, dev)

    if e8m0:
        X.quant_queries(q, w_raw, case.fmt, q_fp8, w)
        X.quant_append_e8(k_new, positions, ix.k_cache, ix.k_scale_cache)
    else:
        X.quant_queries_append(q, w_raw, k_new, positions, ix.k_cache, ix.k_scale_cache, case.fmt, q_fp8, w)
    for _ in range(args.warmup):
        graph.replay()
        score_only()
    torch.cuda.synchronize()
    code, bits = X.status()
    if code != 0:
        raise RuntimeError(f"device error during warm-up: status {code}, bits {bits}")

    def back_to_back(fn, count):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(count):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    # -------------------------------------------------------------- timed region: whole steps
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    with sampler:
        if flush is None:
            ms = back_to_back(graph.replay, args.steps)
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for a, b in evs:
                flush.zero_()
                a.record(stream)
                graph.replay()
                b.record(stream)
            torch.cuda.synchronize()
            ms = sum(a.elapsed_time(b) for a, b in evs)
    if world > 1:
        dist.barrier()
    # the dominant kernel alone: n_k launches recorded in a CUDA graph (no host
    # gaps between them) and replayed between two events; n_k sized for about
    # 10 ms of work, a burst like the measured peaks' (a loop of seconds runs
    # into the 1 kW power cap and lower clocks)
    step_s_est = ms / 1e3 / args.steps
    n_k = max(3, min(200, int(10e-3 / max(step_s_est, 1e-6))))

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n_k):
                fn()
        return g

    g_score = graph_of(score_only)
    g_topk = graph_of(topk_only) if ws_bytes else None
    g_score.replay()
    torch.cuda.synchronize()
    kernel_sampler = ClockSampler(torch.cuda.current_device())
    with kernel_sampler:
        score_ms = back_to_back(g_score.replay, 1) / n_k
    topk_ms = None
    if g_topk is not None:
        g_topk.replay()
        torch.cuda.synchronize()
        topk_ms = back_to_back(g_topk.replay, 1) / n_k
    del g_score, g_topk
    code, bits = X.status()
    if code != 0:
        raise RuntimeError(f"device error in the timed region: status {code}, bits {bits}")

    # -------------------------------------------------------------- end to end from pinned host memory
    # uploads, compute and downloads on three streams, two slots of device buffers (HostPipeline);
    # the step's inputs sit in one pinned buffer with the device layout: one upload per step
    hp = HostPipeline(ix, B, n, causal=case.causal, max_len=max_len)
    h_k, h_q, h_w, h_p, h_l = hp.host_inputs()
    h_k.copy_(case_pinned(torch, case.k_new.view(np.int16)).view(torch.bfloat16))
    h_q.copy_(case_pinned(torch, case.q.view(np.int16)).view(torch.bfloat16))
    h_w.copy_(case_pinned(torch, case.w_raw))
    h_p.copy_(case_pinned(torch, case.positions))
    h_l.copy_(case_pinned(torch, case.lengths))
    h_out = torch.empty((B, n, case.k), dtype=torch.int32).pin_memory()
    h2d = hp.packed_bytes
    d2h = h_out.numel() * h_out.element_size()

    def step_e2e():
        hp.submit(h_k, h_q, h_w, h_p, h_l, h_out)

    e2e_steps = max(3, min(args.steps, 2000))
    for _ in range(max(args.warmup, 2)):             # the first use of each slot captures its graph
        step_e2e()
    hp.join(stream)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    hp.wait(e0)
    for _ in range(e2e_steps):
        step_e2e()
    hp.join(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    code, bits = X.status()
    if code != 0:
        raise RuntimeError(f"device error in the end-to-end loop: status {code}, bits {bits}")

    # -------------------------------------------------------------- reduce over ranks (max time)
    ms, score_ms, e2e_ms = max_over_ranks([ms, score_ms, e2e_ms], device=dev)
    if topk_ms is not None:
        topk_ms = max_over_ranks([topk_ms], device=dev)[0]
    topk_bytes = B * n * 4 * (max_len + case.k) if ws_bytes else None   # score rows read, indices written
    launches_per_step = (3 if (ws_bytes or e8m0) else 2)
    del graph, hp, ix, ws
    return dict(widx=widx, case=case, e8m0=e8m0, keys=keys, flops=flops, key_rows=key_rows, score_bytes=score_bytes,
                ms=ms, score_ms=score_ms, e2e_ms=e2e_ms, e2e_steps=e2e_steps, h2d=h2d, d2h=d2h,
                clocks=sampler.summary(), launches=launches_per_step * args.steps, topk_ms=topk_ms,
                topk_bytes=topk_bytes, two_pass=bool(ws_bytes), l2_flushed=flush is not None, n_k=n_k,
                kernel_clocks=kernel_sampler.summary())


def case_pinned(torch, a):
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


# ---------------------------------------------------------------------------- oracle timing
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_step_timer(case, seqs, key_limit=None):
    """Build the oracle's cache for ``seqs`` (untimed) and return a function that
    runs one oracle step on them (append this call's keys, quantise queries,
    fp64 scores, full-sort top-k) and the keys it scores."""
    from oracle import indexer as O
    B, n = case.B, case.n
    kc = np.zeros((B, case.T_cap, 128), np.uint8)
    ks = np.zeros((B, case.T_cap), np.float32)
    for b in seqs:
        p = int(case.positions[b])
        lim = p if key_limit is None else min(p, key_limit)
        if lim:
            O.quant_append(case.k_prior[b:b + 1, :lim], [0], kc[b:b + 1], ks[b:b + 1], case.fmt)
    lengths = case.lengths.copy()
    positions = case.positions.copy()
    if key_limit is not None:
        positions = np.minimum(positions, key_limit)
        lengths = positions + n
    sel = list(seqs)

    def run():
        st = {"k_cache": kc[sel], "k_scale_cache": ks[sel]}
        O.indexer_step(st, case.k_new[sel], case.q[sel], case.w_raw[sel], positions[sel], case.causal, case.k,
                       case.fmt)

    if case.causal:
        keys = sum(int(((np.arange(lengths[b] - n + 1, lengths[b] + 1)).sum())) for b in sel)
    else:
        keys = sum(int(lengths[b]) * n for b in sel)
    return run, keys


def cpu_baseline(case, target_s=12.0):
    """Time the oracle on a bounded sample of the workload, scaled to keys/s:
    whole oracle steps (append, quantise queries, fp64 scores, full-sort top-k)
    over as many sequences as fit about target_s of CPU time, repeated until
    that much time has passed."""
    run, keys = oracle_step_timer(case, [0])
    t = time.perf_counter()
    run()
    one = max(time.perf_counter() - t, 1e-4)
    nseq = int(max(1, min(case.B, target_s / 2 / one)))
    seqs = list(range(nseq))
    if nseq > 1:
        run, keys = oracle_step_timer(case, seqs)
    reps, dt = 0, 0.0
    t = time.perf_counter()
    while reps == 0 or dt < target_s:
        run()
        reps += 1
        dt = time.perf_counter() - t
    return {"value": keys * reps / dt, "unit": "keys/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{len(seqs)} of {case.B} sequences of '{case.name}', {reps} full oracle steps "
                      f"(append, quantise queries, fp64 scores, full-sort top-{case.k}) in {dt:.1f} s"}


def run_reference(args, rank, world):
    from sparse_attention_token_idx_b200 import synth
    case = synth.workload(args.workload)
    budget_s = 150.0
    per_step = budget_s / max(1, args.steps + args.warmup)
    # size each step: one sequence, its first `limit` cached keys, so the whole run stays bounded
    run, keys = oracle_step_timer(case, [0])
    t = time.perf_counter()
    run()
    full = time.perf_counter() - t
    limit = None
    if full > per_step:
        limit = max(128, int(int(case.positions[0]) * per_step / full))
        run, keys = oracle_step_timer(case, [0], key_limit=limit)
    for _ in range(args.warmup):
        run()
    t = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t
    value = keys * args.steps / dt
    sample = (f"1 of {case.B} sequences of '{case.name}' per step"
              + (f", its first {limit} cached keys" if limit else "") + ", full oracle step")
    return case, value, dt, sample


# ---------------------------------------------------------------------------- widened rows
ROWS = ("merge", "front", "project128", "project4096", "mla")


def row_bench(args, dev, hbm, bf16):
    """One widened row's launch alone, timed with CUDA events after warm-up, with
    its algorithmic bytes or FLOPs: the split-T merge (128 rows, 8 × 2048
    candidates), the fused front end (decode B = 128), the projections (128 and
    4096 tokens, hidden 7168, q_lora 1536) and the sparse latent attention
    (B = 128, 128 heads, k = 2048, 16 384 cached positions).  Inputs are random
    and resident on the device; one L2 flush before the timed launches."""
    import torch
    from sparse_attention_token_idx_b200 import binding as X
    from sparse_attention_token_idx_b200 import synth
    g = torch.Generator(device=dev).manual_seed(3)
    row = args.row
    info = {}
    if row == "merge":
        G, rows, kin, k = 8, 128, 2048, 2048
        sc = torch.randn((G, rows, kin), device=dev, generator=g)
        pos = torch.stack([torch.randperm(G * kin, device=dev, generator=g).view(G, kin) for _ in range(rows)], 1)
        cand = torch.stack([sc.view(torch.int32), pos.to(torch.int32)], -1).contiguous()
        out = torch.empty((rows, k), dtype=torch.int32, device=dev)
        fn = lambda: X.merge_topk(cand, k, out=out)
        info = {"bound": "hbm", "algorithmic_bytes": G * rows * kin * 8 + rows * k * 4, "kernel": "merge_topk_kernel",
                "config": {"rows": rows, "G": G, "kin": kin, "k": k}}
    elif row == "front":
        B, T_cap = 128, 16384
        qp = torch.randn((B, 1, 64, 128), device=dev, generator=g).to(torch.bfloat16)
        kp = torch.randn((B, 1, 128), device=dev, generator=g).to(torch.bfloat16)
        wr = torch.randn((B, 1, 64), device=dev, generator=g)
        ang = torch.rand((B, 1, 32), device=dev, generator=g) * 6.28
        cos, sin = torch.cos(ang), torch.sin(ang)
        gain, bias = torch.ones(128, device=dev), torch.zeros(128, device=dev)
        pos = torch.full((B,), 100, dtype=torch.int32, device=dev)
        kc = torch.zeros((B, T_cap, 128), dtype=torch.uint8, device=dev)
        ks = torch.zeros((B, T_cap), dtype=torch.float32, device=dev)
        q8 = torch.empty((B, 1, 64, 128), dtype=torch.uint8, device=dev)
        w8 = torch.empty((B, 1, 64), dtype=torch.float32, device=dev)
        fn = lambda: X.front_quant_append(qp, wr, kp, cos, sin, gain, bias, 1e-6, pos, kc, ks, 0, q_out=q8, w_out=w8)
        moved = B * (64 * 128 * 2 + 128 * 2 + 64 * 4 + 2 * 32 * 4) + B * (64 * 128 + 64 * 4 + 128 + 4)
        info = {"bound": "hbm", "algorithmic_bytes": moved, "kernel": "quant_kernel<1> (front end fused)",
                "config": {"B": B, "n": 1}}
    elif row in ("project128", "project4096"):
        T = 128 if row == "project128" else 4096
        pc = synth.make_proj_case(9, T)
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        x, qr, wq, wk = bf(pc.x), bf(pc.qr), bf(pc.wq_b), bf(pc.wk)
        wp = torch.from_numpy(pc.w_proj).to(dev)
        ws = torch.empty(X.project_workspace_size(T, synth.HIDDEN, synth.Q_LORA), dtype=torch.uint8, device=dev)
        qo = torch.empty((T, 64, 128), dtype=torch.bfloat16, device=dev)
        ko = torch.empty((T, 128), dtype=torch.bfloat16, device=dev)
        wo = torch.empty((T, 64), dtype=torch.float32, device=dev)
        fn = lambda: X.project(x, qr, wq, wk, wp, q_out=qo, k_out=ko, w_out=wo, ws=ws)
        flops = 2.0 * T * (8192 * synth.Q_LORA + 128 * synth.HIDDEN + 64 * synth.HIDDEN)
        weights = 8192 * synth.Q_LORA * 2 + 128 * synth.HIDDEN * 2 + 64 * synth.HIDDEN * 4
        acts = T * (synth.HIDDEN * 2 + synth.Q_LORA * 2 + 8192 * 2 + 128 * 2 + 64 * 4)
        info = {"bound": "tensor" if T >= 1024 else "hbm", "algorithmic_flops": flops,
                "algorithmic_bytes": weights + acts, "kernel": "gemm_bf16_kernel (q, k, head weights)",
                "config": {"tokens": T, "hidden": synth.HIDDEN, "q_lora": synth.Q_LORA}}
    elif row == "mla":
        B, H, T, k = 128, 128, 16384, 2048
        q = torch.randn((B, H, 576), device=dev, generator=g).to(torch.bfloat16)
        kv = torch.randn((B, T, 576), device=dev, generator=g).to(torch.bfloat16)
        idx = torch.stack([torch.randperm(T, device=dev, generator=g)[:k] for _ in range(B)]).to(torch.int32)
        out = torch.empty((B, H, 512), device=dev, dtype=torch.float32)
        fn = lambda: X.sparse_mla_decode(q, kv, idx, 576 ** -0.5, out=out)
        info = {"bound": "tensor", "algorithmic_flops": 2.0 * B * H * k * (576 + 512),
                "algorithmic_bytes": B * k * 576 * 2 + B * H * (576 * 2 + 512 * 4),
                "kernel": "sparse_mla_tc_kernel", "config": {"B": B, "H": H, "k": k, "T_cap": T}}
    else:
        raise SystemExit(f"--row: one of {', '.join(ROWS)}")
    flush = l2_flush_buffer(torch, dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(max(1, args.steps)):
        flush.zero_()
        # keep the GPU busy while the host enqueues the launch, so that the
        # events bracket the kernel and not the host's launch latency
        torch.cuda._sleep(400_000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize(dev)
        times.append(a.elapsed_time(b) * 1e3)
    us = statistics.median(times)
    line = {"row": row, "us": us, "us_min": min(times), "steps": len(times), "warmup": args.warmup,
            "status": list(X.status()), "l2": "flushed before each launch", "data": "synthetic", **info}
    if "algorithmic_bytes" in info:
        line["achieved_gbs"] = info["algorithmic_bytes"] / (us * 1e-6) / 1e9
        line["frac_of_measured_hbm"] = line["achieved_gbs"] / hbm
    if "algorithmic_flops" in info:
        line["achieved_tflops"] = info["algorithmic_flops"] / (us * 1e-6) / 1e12
        line["frac_of_measured_bf16"] = line["achieved_tflops"] / bf16
    print(json.dumps(line))


# ---------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="time only the selected workload (by default the decode headline also runs "
                         "the two prefill workloads and reports them under 'prefill')")
    ap.add_argument("--scale-storage", choices=["f32", "e8m0"], default="f32",
                    help="key scales as float32 (the workloads' layout) or one e8m0 byte per key "
                         "(ue8m0 workloads only)")
    ap.add_argument("--row", choices=ROWS, default=None,
                    help="time one widened row's launch alone (for its own numbers and ncu captures)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local_rank = env_rank()
    if args.row is not None:
        import torch
        torch.cuda.set_device(local_rank)
        hbm, bf16, _, _ = measured_peaks()
        row_bench(args, torch.device("cuda", local_rank), hbm, bf16)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        case, value, dt, sample = run_reference(args, rank, world)
        unit = "keys/s"
        line = {"metric": metric_name(case), "value": value, "unit": unit, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": case.name, "B": case.B, "n": case.n, "T_cap": case.T_cap, "k": case.k},
                "cpu_baseline": {"value": value, "unit": unit, "cores": oracle_threads(), "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    hbm, bf16, bf16_sus, peak_src = measured_peaks()
    r = measure(args, args.workload, dev, world, headline=True)
    line = result_line(r, args, world, hbm, bf16, peak_src)
    if args.workload == DEFAULT_WORKLOAD and not args.no_prefill:
        # the prefill half of the metric: FP8 TFLOP/s of the two prefill workloads
        line["prefill"] = {}
        for widx in PREFILL_WORKLOADS:
            rp = measure(args, widx, dev, world, headline=False)
            sub = result_line(rp, args, world, hbm, bf16, peak_src)
            for key in ("metric", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "vs_baseline",
                        "data"):
                sub.pop(key, None)
            line["prefill"][str(widx)] = sub
        line["gpu_launches"] += sum(p["gpu_launches"] for p in line["prefill"].values())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(r["case"])
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def result_line(r, args, world, hbm, bf16, peak_src):
    case = r["case"]
    step_s = r["ms"] / 1e3 / args.steps
    value = r["keys"] * world / step_s
    e2e_value = r["keys"] * world / (r["e2e_ms"] / 1e3 / r["e2e_steps"])
    score_s = r["score_ms"] / 1e3
    if case.causal:
        achieved = r["flops"] / score_s / 1e12
        peak = bf16 * FP8_PER_BF16
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": flat_profile_traffic(r["widx"]) if r["two_pass"] and not r["e8m0"] else None,
                "peak_source": f"{peak_src} bf16 burst x nominal fp8/bf16 ratio {FP8_PER_BF16}",
                "frac_of_datasheet_fp8": achieved / DATASHEET_FP8_TFLOPS,
                "kernel": "flat_score_kernel (tcgen05 FP8 scorer, fp32 scores to the workspace)",
                "kernel_us": r["score_ms"] * 1e3, "algorithmic_flops": r["flops"],
                "timing": f"{r['n_k']} launches recorded back to back in a CUDA graph (about 10 ms), one replay "
                          "between two CUDA events", "clocks": r["kernel_clocks"]}
    else:
        achieved = r["score_bytes"] / score_s / 1e9
        traffic = (profile_traffic(PROFILE_SCORE, r["key_rows"])
                   if args.workload == DEFAULT_WORKLOAD and not r["e8m0"] else None)
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": traffic, "peak_source": f"{peak_src} copy bandwidth",
                "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                "target_basis": "the 70% decode target is read against the measured copy peak (frac); "
                                "frac_of_nominal_8tbs is the same time against 8 TB/s",
                "kernel": "flat_score_kernel (tcgen05 FP8 scorer, fp32 scores to the workspace)" if r["two_pass"]
                else "score_kernel (fused score + top-k)",
                "kernel_us": r["score_ms"] * 1e3, "algorithmic_bytes": r["score_bytes"],
                "timing": f"{r['n_k']} launches recorded back to back in a CUDA graph (about 10 ms), one replay "
                          "between two CUDA events", "clocks": r["kernel_clocks"]}
    l2 = ("L2 flushed (a write of twice the L2 size) before each step, outside the timed events"
          if r["l2_flushed"] else
          "inputs larger than L2: %.0f MB FP8 cache streamed per step"
          % (r["key_rows"] * (KEY_BYTES - 3 * r["e8m0"]) / 1e6))
    line = {
        "metric": metric_name(case), "value": value, "unit": "keys/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms"] / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8-e4m3 x fp8-e4m3 -> fp32", "data": "synthetic",
        "config": {"workload": case.name + (", e8m0 scale bytes" if r["e8m0"] else ""), "B": case.B, "n": case.n,
                   "T_cap": case.T_cap, "k": case.k,
                   "scale_storage": "e8m0 bytes (129 B/key)" if r["e8m0"] else "fp32 (132 B/key)",
                   "heads": 64, "head_dim": 128, "fmt": ["fp32", "ue8m0"][case.fmt], "l2": l2,
                   "parallelism": f"dp{world} (independent sequences per rank)"},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "keys/s", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "steps": r["e2e_steps"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    if case.causal:
        line["tflops"] = r["flops"] * world / step_s / 1e12      # whole step (quantise + score + top-k)
        line["e2e"]["tflops"] = r["flops"] * world / (r["e2e_ms"] / 1e3 / r["e2e_steps"]) / 1e12
    if r["topk_ms"] is not None:
        line["topk"] = {"kernel": "topk_row_kernel", "us": r["topk_ms"] * 1e3,
                        "algorithmic_bytes": r["topk_bytes"],
                        "achieved_gbs": r["topk_bytes"] / (r["topk_ms"] / 1e3) / 1e9,
                        "frac_of_measured_hbm": r["topk_bytes"] / (r["topk_ms"] / 1e3) / 1e9 / hbm}
    return line


def metric_name(case):
    return "prefill keys scored+top-k/s (FP8 TFLOP/s in tflops)" if case.causal else "decode keys scored+top-k/s"


if __name__ == "__main__":
    main()
