"""GPU parity for context-parallel decode ("HySparse2: Hybrid Sparse Attention with Two-Level KV
Sharing", bullet "Inference cost": 1M-token contexts; the block's layers as in "HySparse2: How
Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse and Token-Level
Sparse Selection"), against the oracle over the whole context.

One GPU stands in for the ranks: each rank is a host thread that runs the library's kernels on
its own shard (a view of its token range of one cache) and the all-gathers are host exchanges
between the threads, so no kernel ever waits for another rank's kernel. Checked: the merged
full-layer output and lse (tolerances as for one GPU), the shards' scores, the global selection
bit for bit against the oracle's fp32 selector fed the scores the shards computed, and every
sparse layer against the oracle's attention over that selection."""
import threading

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from token_level_sparse_hs2_b200 import build
    build.build()
    oracle.build()


def run_cp(w, bounds, topk, window):
    import token_level_sparse_hs2_b200 as m
    from token_level_sparse_hs2_b200 import cp
    d = W.to_device(w)
    T, start, H = int(w.kv_len[0]), int(w.kv_start[0]), w.n_heads
    world = len(bounds) - 1
    barrier = threading.Barrier(world, timeout=120)
    box = [None] * world
    results, errors = [None] * world, []

    def gather_for(rank):
        def gather(x):
            torch.cuda.synchronize()
            box[rank] = x.clone()
            barrier.wait()
            out = torch.stack(list(box))
            barrier.wait()            # every rank has read before the next exchange
            return out
        return gather

    def worker(rank):
        try:
            torch.cuda.set_device(0)
            off, tl = bounds[rank], bounds[rank + 1] - bounds[rank]
            cache = m.KvCache(d["k"], d["v"], [start + off], [tl], 1, H, d["k_scale"], d["v_scale"])
            ws = torch.empty(m.workspace_size(cache, topk, min(window, tl)), dtype=torch.uint8,
                             device="cuda")
            out = torch.empty((1, 1, H, 128), dtype=torch.float32, device="cuda")
            outs = [torch.empty_like(out) for _ in range(w.n_sparse)]
            res = cp.cp_block_decode(cache, off, T, d["q_full"], d["q_sparse"], out, outs, ws,
                                     gather_for(rank), topk=topk, window=window)
            m.read_device_status(ws)
            torch.cuda.synchronize()
            results[rank] = dict(o=out.cpu().numpy(), outs=[o.cpu().numpy() for o in outs],
                                 lse=res["lse"].cpu().numpy(), idx=res["idx"].cpu().numpy(),
                                 count=res["count"].cpu().numpy(),
                                 scores=res["scores"].cpu().numpy())
        except BaseException as e:   # noqa: BLE001 - reported below
            errors.append(e)
            barrier.abort()

    threads = [threading.Thread(target=worker, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    return results


def check(w, bounds, res, topk, window):
    from tests import gpu_helpers as G
    T = int(w.kv_len[0])
    for r in res[1:]:                 # every rank holds the same merged results
        assert np.array_equal(r["o"], res[0]["o"]) and np.array_equal(r["idx"], res[0]["idx"])
        assert np.array_equal(r["lse"], res[0]["lse"])
    r0 = res[0]
    o_ref, lse_ref, s_ref = oracle.full_attn(w, rows=[0])
    tol = G.O_TOL[w.kv_dtype]
    assert np.abs(r0["o"].reshape(o_ref.shape) - o_ref).max() <= tol
    dl = np.abs(r0["lse"].reshape(lse_ref.shape) - lse_ref)
    assert (dl <= 1e-4 + 1e-5 * np.abs(lse_ref)).all(), dl.max()
    s = np.zeros((1, T), dtype=np.float32)
    for k in range(len(bounds) - 1):
        s[0, bounds[k]:bounds[k + 1]] = res[k]["scores"][0]
    G.check_scores(w, [0], s, s_ref)
    ref, rc = oracle.select_rows(w, [0], s, topk, window, fp32=True)
    c = int(r0["count"][0])
    assert c == rc[0] and np.array_equal(r0["idx"][0, :c], ref[0, :c])
    for l in range(w.n_sparse):
        sp = oracle.sparse_attn(w, w.q_sparse[l], [0], r0["idx"], r0["count"])
        assert np.abs(r0["outs"][l].reshape(sp.shape) - sp).max() <= tol, l


def workload(T, kv_dtype="bf16", H=32, seed=31, needles=16):
    return W.make_workload(dict(name="cp", batch=1, n_q=1, n_heads=H, n_sparse=2,
                                kv_dtype=kv_dtype, lengths=(T,), needles=needles), seed=seed)


@pytest.mark.parametrize("T,bounds,kv_dtype", [
    (4096, [0, 2048, 4096], "bf16"),
    (4096, [0, 1000, 2500, 4000, 4096], "bf16"),      # last shard inside the window
    (20000, [0, 7000, 7100, 20000], "fp8"),            # a shard of 100 positions
    (131072, [0, 32768, 65536, 98304, 131072], "bf16"),
])
def test_cp_decode_matches_the_whole_context(T, bounds, kv_dtype):
    w = workload(T, kv_dtype)
    res = run_cp(w, bounds, w.topk, w.window)
    check(w, bounds, res, w.topk, w.window)


def test_cp_small_budget_with_shards_outside_the_selection():
    """topk 16 over 8 shards: some shards hold none of the selection (empty sparse parts)."""
    w = workload(6000, H=16, needles=4)
    bounds = [0, 700, 1500, 2200, 3000, 3700, 4500, 5300, 6000]
    res = run_cp(w, bounds, 16, 16)
    check(w, bounds, res, 16, 16)


def test_cp_short_context_keeps_everything():
    w = workload(900, H=16, needles=2)
    bounds = [0, 300, 900]
    res = run_cp(w, bounds, w.topk, w.window)
    assert int(res[0]["count"][0]) == 900
    check(w, bounds, res, w.topk, w.window)


def test_cp_shards_starting_inside_tiles():
    """Shard boundaries that are not multiples of the 64-row tile, including a one-token shard
    and the window split over two shards."""
    w = workload(10_000, H=32, needles=8)
    bounds = [0, 37, 38, 5001, 9_930, 10_000]
    res = run_cp(w, bounds, w.topk, w.window)
    check(w, bounds, res, w.topk, w.window)
