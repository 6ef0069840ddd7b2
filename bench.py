"""Benchmark of the HySparse2 hybrid-block decode step on B200.

`python bench.py --gpus N --steps K --warmup W [--impl hs2|reference] [--config C]`

One step = one hybrid block over one batch of synthetic decode queries: the full-attention
layer (pass 1: output + log-sum-exp; pass 2: importance scores), the token top-k + forced
window selection, and every sparse layer, all through `hs2_block_decode` (C ABI). The default
workload is the 128k-context decode batch: 8 sequences with contexts drawn uniformly from
65,536..131,072 tokens, 32 query heads on one bf16 K/V head, 3 sparse layers, top-1,024 +
window 128. Its K/V cache (~400 MB) is larger than the 126 MB L2, so no flush is needed
between steps. Workloads whose cache fits in L2 (the 4k decode, the 32k prefill) time every step
alone, after a 256 MB write that evicts the cache, and report the back-to-back time as "warm".

Multi-GPU (torchrun): every rank runs its own batch (independent sequences, no exchange);
`value` is all ranks' tokens over the slowest rank's time (weak scaling).
`--impl reference` times the fp64 CPU oracle on the same workload (rank 0 only).
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "hybrid-block decode tokens/s at 128k/1M ctx; achieved % of HBM roofline"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="hs2", choices=["hs2", "reference"])
    ap.add_argument("--config", type=int, default=1, help="workload id (0..2 decode)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    a.steps = max(a.steps, 1)
    return a


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]),
                "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def causal_pairs(w) -> int:
    """Sum over query rows of the visible prefix length p + 1."""
    tot = 0
    for t in w.kv_len.astype(np.int64):
        first = int(t) - w.n_q + 1
        tot += w.n_q * first + w.n_q * (w.n_q - 1) // 2
    return tot


def tensor_flops(w) -> dict:
    """Dense FLOPs of the full layer: per visible (query, token) pair and head, 2 * 128 for
    q.k and 2 * 128 for p.v (pass 1), 2 * 128 for q.k again (score pass)."""
    pairs = causal_pairs(w) * w.n_heads
    return dict(pass1=pairs * 4 * w.head_dim, pass2=pairs * 2 * w.head_dim)


def algorithmic_bytes(w) -> dict:
    """Bytes each step must move at least once, per kernel (see the design notes):
    pass 1 reads K and V of every cached token once; pass 2 reads K again and writes one fp32
    score per token; the selection reads every score once; each sparse layer gathers
    topk + window K/V rows per query. Queries, outputs, lse and indices are counted too."""
    T = int(w.kv_len.astype(np.int64).sum())
    H, d, B = w.n_heads, w.head_dim, w.batch
    elem = 2 if w.kv_dtype == "bf16" else 1
    row = d * elem + (4 if w.kv_dtype == "fp8" else 0)          # one K (or V) row + scale
    q = B * H * d * 2
    o = B * H * d * 4
    p1 = T * 2 * row + q + o + B * H * 4
    p2 = T * row + T * 4 + q + B * H * 4
    tk = T * 4 + B * (w.topk + w.window) * 4
    sel = [min(int(t), w.topk + w.window) for t in w.kv_len]
    sp = sum(sel) * 2 * row + q + o + sum(sel) * 4
    total = p1 + p2 + tk + w.n_sparse * sp
    # B_min: the same step if K were read only once (a design that kept the logits would need
    # no second K read); reported beside the fraction so that it is not flattered
    return dict(pass1=p1, pass2=p2, topk=tk, sparse=sp, total=total, total_k_once=total - T * row)


L2_BYTES = 126 * 1000 * 1000


def cache_bytes(w) -> int:
    """K and V (and their FP8 scales) of the workload's cache."""
    return int(w.k.nbytes + w.v.nbytes + (w.k_scale.nbytes + w.v_scale.nbytes
                                          if w.kv_dtype == "fp8" else 0))


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _poll(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.005)

    def sample(self):
        if self.nv is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for b, name in self.REASONS.items():
                if bits & b and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        self.t = threading.Thread(target=self._poll, daemon=True)
        self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self.t.join()
        self.sample()

    def result(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def slowest(x: float, dist=None, device=None) -> float:
    """The largest x over the ranks (the slowest rank's time); x itself without a process group.
    The reduction runs on `device` (CUDA for NCCL, CPU for gloo)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(units_per_rank: int, world: int, ms: float) -> float:
    """Whole-job rate: every rank's units over the slowest rank's time (weak scaling)."""
    return world * units_per_rank / (ms / 1e3)


def dist_setup(a):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_baseline(w, budget_s=12.0):
    """The oracle as it stands, on the host cores, over whole batches of the same workload."""
    import oracle
    oracle.build()
    rows = np.arange(w.n_rows)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.block(w, rows=rows)
        reps += 1
        el = time.perf_counter() - t0
        if el > budget_s or reps >= 200:
            break
    tok = reps * w.n_rows
    return {"value": tok / el, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{reps} full batch(es) of {w.n_rows} decode queries (all "
                      f"{int(w.kv_len.sum())} cached tokens, all layers), {el:.1f} s"}


def run_reference(a, w):
    world, rank, _ = dist_setup(a)
    if rank != 0:
        return
    import oracle
    oracle.build()
    rows = np.arange(w.n_rows)
    for _ in range(a.warmup if a.warmup <= 3 else 3):
        oracle.block(w, rows=rows)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        oracle.block(w, rows=rows)
    el = time.perf_counter() - t0
    value = a.steps * w.n_rows / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": el / a.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"each step: the full batch of {w.n_rows} decode queries"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bench_kv_append(hs2, dev, hbm, rows=262144, iters=20):
    """The cache append (the step before the block) on a bulk of rows into an e4m3 cache: bytes
    = rows x (K and V: 256 B read, 128 B codes + 4 B scale written), over the event time. The
    262,144 rows move 203 MB per call, more than the 126 MB L2, so repeats do not hit in L2."""
    k = torch.zeros((rows, 128), dtype=torch.uint8, device=dev)
    v = torch.zeros_like(k)
    ks = torch.zeros(rows, dtype=torch.float32, device=dev)
    vs = torch.zeros_like(ks)
    cache = hs2.KvCache(k, v, [0], [rows], rows, 32, ks, vs)
    nk = torch.randn((1, rows, 128), device=dev).to(torch.bfloat16)
    nv = torch.randn((1, rows, 128), device=dev).to(torch.bfloat16)
    for _ in range(3):
        hs2.kv_append(cache, nk, nv)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(iters):
        hs2.kv_append(cache, nk, nv)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / iters * 1e3
    nbytes = rows * 2 * (256 + 128 + 4)
    gbs = nbytes / (us / 1e6) / 1e9
    return {"kernel": "kv_append_kernel", "rows": rows, "kv_dtype": "fp8-e4m3", "us": us,
            "bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / hbm}


def bench_kv_bridge(hs2, dev, hbm, tf_burst, tokens=32768, d_model=4096, iters=10):
    """KV Bridging on a prefill of `tokens` prompt tokens (hidden size d_model, synthetic
    weights): K and V rows = hidden . [W_K; W_V]^T into a bf16 cache. FLOPs 2 x tokens x d_model
    x 256; bytes = hidden + weights read, K and V rows written."""
    g = torch.Generator(device=dev).manual_seed(7)
    hidden = torch.randn((1, tokens, d_model), device=dev, generator=g).to(torch.bfloat16)
    w = (torch.randn((256, d_model), device=dev, generator=g) / d_model ** 0.5).to(torch.bfloat16)
    k = torch.empty((tokens, 128), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    cache = hs2.KvCache(k, v, [0], [tokens], tokens, 32)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    for _ in range(3):
        hs2.kv_bridge(cache, hidden, w, ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(iters):
        hs2.kv_bridge(cache, hidden, w, ws)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / iters * 1e3
    flops = 2.0 * tokens * d_model * 256
    nbytes = tokens * d_model * 2 + 256 * d_model * 2 + tokens * 2 * 256
    tf = flops / (us / 1e6) / 1e12
    gbs = nbytes / (us / 1e6) / 1e9
    return {"kernel": "kv_bridge_kernel", "tokens": tokens, "d_model": d_model, "us": us,
            "flops": flops, "tflops": tf, "frac_of_bf16_burst_peak": tf / tf_burst,
            "bytes": nbytes, "achieved_gbs": gbs, "frac_of_hbm": gbs / hbm,
            "note": "hidden states (%.0f MB) exceed L2; no flush" % (tokens * d_model * 2 / 1e6)}


def bench_cp_shard(hs2, w, d, dev, world=8, iters=10):
    """Context-parallel decode of this one-sequence workload over `world` ranks: the kernels of
    one rank's block step (the last shard, which holds the window), timed on this GPU with the
    all-gathers replaced by a local copy (only one GPU here: the NCCL exchanges are not timed)."""
    from token_level_sparse_hs2_b200 import cp
    T, H, L = int(w.kv_len[0]), w.n_heads, w.n_sparse
    bounds = [T * k // world for k in range(world + 1)]
    off, tl = bounds[-2], bounds[-1] - bounds[-2]
    cache = hs2.KvCache(d["k"], d["v"], [int(w.kv_start[0]) + off], [tl], 1, H, d["k_scale"],
                        d["v_scale"])
    ws = torch.empty(hs2.workspace_size(cache, w.topk, min(w.window, tl)), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((1, 1, H, 128), dtype=torch.float32, device=dev)
    outs = [torch.empty_like(out) for _ in range(L)]
    sizes = []

    def gather(x):
        sizes.append(x.numel() * x.element_size())
        return x.unsqueeze(0).expand((world,) + tuple(x.shape)).contiguous()

    def step():
        cp.cp_block_decode(cache, off, T, d["q_full"], d["q_sparse"], out, outs, ws, gather,
                           topk=w.topk, window=w.window)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(3):
            step()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    # one step captured in a CUDA graph and replayed, so that the host's per-call cost (Python,
    # argument checks) does not show in the device time
    n0 = hs2.launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    launches = hs2.launch_count() - n0
    graph.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(iters):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    del graph
    return {"world": world, "shard_tokens": tl, "us_per_rank_step": e0.elapsed_time(e1) / iters * 1e3,
            "timing": "CUDA graph of one step, replayed %d times" % iters,
            "library_launches_per_step": launches,
            "allgathers_per_step": 2 + L, "bytes_per_rank_per_allgather": sizes[:2 + L],
            "note": "one rank's kernels; the all-gathers (NCCL over NVLink) are replaced by a "
                    "local copy on this one-GPU run and not timed"}


def bench_block_select(hs2, cache, scores, w, dev, token_ms, block_size=64, iters=20):
    """Block-level selection (HySparse's granularity at the same budget) on the step's own
    scores, beside the token-level selection's traced time: pooling + per-row select."""
    R = w.n_rows
    cap = min(int(w.kv_len.max()), w.topk + w.window)
    idx = torch.empty((R, cap), dtype=torch.int32, device=dev)
    cnt = torch.empty(R, dtype=torch.int32, device=dev)
    ws = torch.empty(hs2.topk_select_blocks_workspace_size(cache, block_size, w.topk, w.window),
                     dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(3):
            hs2.topk_select_blocks(cache, scores, idx, cnt, ws, block_size, w.topk, w.window)
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    # the calls are replayed from a CUDA graph so that the host's per-call cost does not show
    n0 = hs2.launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(iters):
            hs2.topk_select_blocks(cache, scores, idx, cnt, ws, block_size, w.topk, w.window)
    launches = (hs2.launch_count() - n0) / iters
    graph.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    del graph
    return {"kernels": ["block_pool_kernel", "block_select_kernel"] if w.n_rows < 148
            else ["block_select_kernel (pooling fused)"], "block_size": block_size,
            "blocks_kept": w.topk // block_size, "us": e0.elapsed_time(e1) / iters * 1e3,
            "launches_per_call": launches, "timing": "CUDA graph of %d calls" % iters,
            "token_topk_us_traced": token_ms * 1e3}


def config_of(w):
    return {"workload": w.name, "batch": w.batch, "queries_per_seq": w.n_q,
            "context_tokens_total": int(w.kv_len.astype(np.int64).sum()),
            "context_min": int(w.kv_len.min()), "context_max": int(w.kv_len.max()),
            "n_heads": w.n_heads, "kv_heads": 1, "head_dim": w.head_dim,
            "n_sparse_layers": w.n_sparse, "topk": w.topk, "window": w.window,
            "kv_dtype": w.kv_dtype, "seed": w.seed}


def measure_block(a, w, hs2, dev, local, pg, world):
    """Times `a.steps` hybrid-block steps of workload `w` on this rank (after `a.warmup`
    untimed ones), then the same steps with an event between kernels, then end to end through
    the public API with host copies. Returns the measurements plus the device buffers."""
    d = W.to_device(w, dev)
    cache = hs2.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, w.n_q, w.n_heads,
                        d["k_scale"], d["v_scale"])
    R, H, L = w.n_rows, w.n_heads, w.n_sparse
    stride = int(w.kv_len.max())
    cap = min(stride, w.topk + w.window)
    out = torch.empty((w.batch, w.n_q, H, 128), dtype=torch.bfloat16, device=dev)
    outs = [torch.empty_like(out) for _ in range(L)]
    lse = torch.empty((w.batch, w.n_q, H), dtype=torch.float32, device=dev)
    scores = torch.empty((R, stride), dtype=torch.float32, device=dev)
    idx = torch.empty((R, cap), dtype=torch.int32, device=dev)
    cnt = torch.empty(R, dtype=torch.int32, device=dev)
    ws = torch.empty(hs2.workspace_size(cache, w.topk, w.window), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        hs2.block_decode(cache, d["q_full"], d["q_sparse"], out, outs, lse, scores, idx, cnt, ws,
                         topk=w.topk, window=w.window)

    for _ in range(a.warmup):
        step()
    hs2.read_device_status(ws)
    torch.cuda.synchronize()

    def barrier():
        if pg:
            pg.barrier()
        torch.cuda.synchronize()

    # ---- timed region: K steps back to back, events only at the two ends. A cache that fits
    # in L2 would stay there from step to step, so for such workloads every step is timed
    # alone after a 256 MB write that evicts it (the back-to-back time is reported as "warm").
    fits_l2 = cache_bytes(w) < L2_BYTES
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if fits_l2 else None
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    n0 = hs2.launch_count()
    with ClockSampler(local) as clk:
        if fits_l2:
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(a.steps)]
            for e0, e1 in pairs:
                flush.zero_()
                e0.record(stream)
                step()
                e1.record(stream)
        t_start.record(stream)
        for _ in range(a.steps):
            step()
        t_end.record(stream)
        torch.cuda.synchronize()
    launches = (hs2.launch_count() - n0) // (2 if fits_l2 else 1)
    barrier()
    hs2.read_device_status(ws)
    ms_warm = t_start.elapsed_time(t_end) / a.steps
    ms = sum(e0.elapsed_time(e1) for e0, e1 in pairs) / a.steps if fits_l2 else ms_warm
    ms_max = slowest(ms, pg, dev)
    ms_warm_max = slowest(ms_warm, pg, dev)

    # ---- the same K steps again with an event between consecutive kernels (per-kernel times;
    # the events break the programmatic-launch overlap, so this step time runs a little longer)
    n_ev = 6 + L
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(a.steps)]
    for row in evs:            # torch creates the CUDA event on first record
        for e in row:
            e.record(stream)
    barrier()
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0e.record(stream)
    for k in range(a.steps):
        hs2.block_decode_traced(cache, d["q_full"], d["q_sparse"], out, outs, lse, scores,
                                idx, cnt, ws, evs[k], topk=w.topk, window=w.window)
    t1e.record(stream)
    torch.cuda.synchronize()
    ms_traced = t0e.elapsed_time(t1e) / a.steps
    names = ["clear", "pass1", "merge1", "pass2", "topk"] + [f"sparse{l}" for l in range(L)]
    per = {n: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(a.steps))
           for i, n in enumerate(names)}

    # ---- end to end through the public API: host queries in, host results out, every step
    e2e = None
    if not a.no_e2e:
        # One pinned host buffer in and one out per step: the queries of every layer packed
        # together, and the outputs, indices and counts written into one device buffer. Two
        # device slots let the copies of one step overlap the kernels of another, as a serving
        # loop would: step k's queries go into slot k % 2 on a copy stream while step k - 1
        # computes, the block waits for them, and its results return on the copy stream once
        # the block has ended. A slot is refilled only after the block that read it has ended,
        # and only after its previous results have been copied out.
        qn = d["q_full"].numel()
        hq_all = torch.cat([d["q_full"].reshape(-1)] + [q.reshape(-1) for q in d["q_sparse"]]) \
            .cpu().pin_memory()
        on = out.numel()
        o_bytes, i_bytes, c_bytes = (1 + L) * on * 2, idx.numel() * 4, cnt.numel() * 4
        slots = []
        for _ in range(2):
            dq_all = torch.empty_like(hq_all, device=dev)
            dbuf = torch.empty(o_bytes + i_bytes + c_bytes, dtype=torch.uint8, device=dev)
            o_all = dbuf[:o_bytes].view(torch.bfloat16)
            slots.append(dict(
                dq_all=dq_all, dbuf=dbuf,
                dq=dq_all[:qn].view(d["q_full"].shape),
                dqs=[dq_all[(l + 1) * qn:(l + 2) * qn].view(d["q_sparse"][l].shape) for l in range(L)],
                eo=o_all[:on].view(out.shape),
                eos=[o_all[(l + 1) * on:(l + 2) * on].view(out.shape) for l in range(L)],
                eidx=dbuf[o_bytes:o_bytes + i_bytes].view(torch.int32).view(idx.shape),
                ecnt=dbuf[o_bytes + i_bytes:].view(torch.int32).view(cnt.shape),
                hbuf=torch.empty(dbuf.numel(), dtype=torch.uint8).pin_memory()))
        h2d = hq_all.numel() * 2
        d2h = slots[0]["hbuf"].numel()
        cstream = torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = torch.cuda.Event()

        def e2e_run(n, start=None):
            """n pipelined steps; returns after enqueueing them (stream waits for the last copy)."""
            if start is not None:
                cstream.wait_event(start)
            with torch.cuda.stream(cstream):
                slots[0]["dq_all"].copy_(hq_all, non_blocking=True)
                ev_in[0].record(cstream)
            for k in range(n):
                sk, sl = k % 2, slots[k % 2]
                stream.wait_event(ev_in[sk])
                hs2.block_decode(cache, sl["dq"], sl["dqs"], sl["eo"], sl["eos"], lse, scores,
                                 sl["eidx"], sl["ecnt"], ws, topk=w.topk, window=w.window)
                ev_done[sk].record(stream)
                with torch.cuda.stream(cstream):
                    if k + 1 < n:   # the next step's queries, into the slot step k - 1 read
                        if k >= 1:
                            cstream.wait_event(ev_done[1 - sk])
                        slots[1 - sk]["dq_all"].copy_(hq_all, non_blocking=True)
                        ev_in[1 - sk].record(cstream)
                    cstream.wait_event(ev_done[sk])
                    sl["hbuf"].copy_(sl["dbuf"], non_blocking=True)
            ev_out.record(cstream)
            stream.wait_event(ev_out)

        e2e_run(3)
        torch.cuda.synchronize()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        e2e_run(a.steps, start=a0)
        a1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = slowest(a0.elapsed_time(a1) / a.steps, pg, dev)
        e2e = {"value": throughput(R, world, ems), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ems}
    return dict(ms=ms_max, ms_warm=ms_warm_max, fits_l2=fits_l2, per=per, ms_traced=ms_traced,
                launches=int(launches), clocks=clk.result(), e2e=e2e, d=d, cache=cache,
                scores=scores)


def rooflines(w, m):
    """The dominant kernel's roofline (pass 1) and the whole step's, from measurements m."""
    hbm, tf_burst, tf_sust, how = peaks()
    ab = algorithmic_bytes(w)
    per = m["per"]
    p1_s = per["pass1"] / 1e3
    ach = ab["pass1"] / p1_s / 1e9
    traffic = None
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            traffic = json.load(f).get(w.name, {}).get("pass1")
    except Exception:
        pass
    if w.n_q == 1:   # decode: the passes stream the cache once each (HBM-bound)
        roofline = {"kernel": "full-attention pass 1", "bound": "hbm", "achieved": ach,
                    "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "traffic": traffic,
                    "peak_source": how + " copy bandwidth", "bytes_per_launch": ab["pass1"],
                    "ms_per_launch": per["pass1"]}
        extra = {}
    else:            # chunks / prefill: dense products over the causal prefix (tensor-bound)
        fl = tensor_flops(w)
        a1 = fl["pass1"] / p1_s / 1e12
        a2 = fl["pass2"] / (per["pass2"] / 1e3) / 1e12
        roofline = {"kernel": "full-attention pass 1", "bound": "tensor", "achieved": a1,
                    "peak": tf_burst, "unit": "TFLOP/s", "frac": a1 / tf_burst,
                    "frac_of_sustained_peak": a1 / tf_sust, "traffic": traffic,
                    "peak_source": how + " bf16 GEMM, burst (the timed region is well under "
                                         "a second)",
                    "flops_per_launch": fl["pass1"], "ms_per_launch": per["pass1"]}
        extra = {"score_pass_roofline": {
            "kernel": "score pass 2 (tcgen05)" if w.kv_dtype == "bf16" else "score pass 2",
            "bound": "tensor", "achieved": a2, "peak": tf_burst, "unit": "TFLOP/s",
            "frac": a2 / tf_burst, "frac_of_sustained_peak": a2 / tf_sust,
            "flops_per_launch": fl["pass2"], "ms_per_launch": per["pass2"]}}
    ms = m["ms"]
    block = {"bytes_per_step": ab["total"],
             "achieved_gbs": ab["total"] / (ms / 1e3) / 1e9,
             "frac": ab["total"] / (ms / 1e3) / 1e9 / hbm,
             "bytes_min_k_once": ab["total_k_once"],
             "frac_min_k_once": ab["total_k_once"] / (ms / 1e3) / 1e9 / hbm}
    return roofline, extra, block


def l2_note(w, m):
    if m["fits_l2"]:
        return ("K/V cache %.1f MB fits in L2: every timed step follows a 256 MB write that "
                "evicts it; warm back-to-back steps: %.4f ms" % (cache_bytes(w) / 1e6, m["ms_warm"]))
    return "inputs larger than L2 (K/V cache %.0f MB > 126 MB); no flush" % (cache_bytes(w) / 1e6)


SECOND_DECODE = 2   # the 1M-token FP8 decode, the metric's other context length


def main():
    a = parse()
    world, rank, local = dist_setup(a)
    w = W.make_workload(a.config)
    if a.impl == "reference":
        run_reference(a, w)
        return
    import token_level_sparse_hs2_b200 as hs2
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    m = measure_block(a, w, hs2, dev, local, pg, world)
    R = w.n_rows
    hbm, tf_burst, _, _ = peaks()
    roofline, extra, block = rooflines(w, m)
    line = {
        "metric": METRIC, "value": throughput(R, world, m["ms"]), "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": m["ms"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.kv_dtype == "bf16" else "fp8-e4m3 (bf16/f16 math)",
        "data": "synthetic",
        "config": dict(config_of(w), parallelism=f"replicas x{world} (independent batches)",
                       l2=l2_note(w, m)),
        "roofline": roofline,
        **extra,
        "block_roofline": block,
        "ms_per_kernel": m["per"], "ms_per_step_traced": m["ms_traced"],
        "gpu_launches": m["launches"],
        "clocks": m["clocks"],
    }
    if m["e2e"]:
        line["e2e"] = m["e2e"]
    # the metric's other context length: the 1M-token FP8 decode, measured in the same run
    # (every rank its own replica, max over ranks) and reported beside the headline
    if a.config != SECOND_DECODE and a.config in (0, 1):
        w2 = W.make_workload(SECOND_DECODE)
        m2 = measure_block(a, w2, hs2, dev, local, pg, world)
        r2, _, b2 = rooflines(w2, m2)
        sec = {"config": dict(config_of(w2), l2=l2_note(w2, m2)),
               "value": throughput(w2.n_rows, world, m2["ms"]), "unit": UNIT,
               "ms_per_step": m2["ms"], "roofline": r2, "block_roofline": b2,
               "ms_per_kernel": m2["per"], "ms_per_step_traced": m2["ms_traced"],
               "gpu_launches": m2["launches"], "clocks": m2["clocks"]}
        if m2["e2e"]:
            sec["e2e"] = m2["e2e"]
        if rank == 0 and world == 1 and not a.no_cpu_baseline:
            sec["cpu_baseline"] = cpu_baseline(w2, budget_s=10.0)
        sec["cp_decode"] = bench_cp_shard(hs2, w2, m2["d"], dev)
        line["decode_1m_fp8"] = sec
        del m2
    line["kv_append"] = bench_kv_append(hs2, dev, hbm)
    line["kv_bridge"] = bench_kv_bridge(hs2, dev, hbm, tf_burst)
    if w.batch == 1 and w.n_q == 1 and int(w.kv_len[0]) >= 65536:
        line["cp_decode"] = bench_cp_shard(hs2, w, m["d"], dev)
    line["block_select"] = bench_block_select(hs2, m["cache"], m["scores"], w, dev,
                                              m["per"]["topk"])
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
