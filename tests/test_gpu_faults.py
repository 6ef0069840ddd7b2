"""Failure detection on the GPU without a fault: bounded waits that run out and device-side
checks of out-of-range inputs report through the status word; the context stays usable.

"HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs" describes no failure
handling; these tests cover the library's own contract (include/hs2.h).
"""
import pytest
import torch

import token_level_sparse_hs2_b200 as hs2
import workloads as W
from tests.gpu_helpers import run_block

pytestmark = pytest.mark.gpu

HS2_ERR_TIMEOUT, HS2_ERR_DEVICE_CHECK = 6, 5


def test_bounded_wait_runs_out_and_reports_timeout():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert hs2.selftest_wait_timeout(ws, limit_us=20000) == HS2_ERR_TIMEOUT
    # the context is still usable: a normal block runs and matches afterwards
    w = W.make_workload(0, lengths=[600])
    run_block(w)


def test_out_of_range_indices_are_clamped_and_reported():
    w = W.make_workload(0, lengths=[700], n_sparse=1)
    dev = torch.device("cuda")
    d = W.to_device(w, dev)
    cache = hs2.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, w.n_q, w.n_heads, d["k_scale"], d["v_scale"])
    cap = min(int(w.kv_len.max()), w.topk + w.window)
    idx = torch.arange(cap, dtype=torch.int32, device=dev).reshape(1, cap).contiguous()
    idx[0, 5] = 10 ** 6            # beyond the sequence
    idx[0, 9] = -3                 # negative
    cnt = torch.full((1,), cap, dtype=torch.int32, device=dev)
    out = torch.empty((1, 1, w.n_heads, 128), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(hs2.workspace_size(cache, w.topk, w.window), dtype=torch.uint8, device=dev)
    hs2.sparse_gather_attn(cache, d["q_sparse"][0], idx, cnt, out, ws)
    with pytest.raises(hs2.HS2Error) as e:
        hs2.read_device_status(ws)
    assert e.value.status == HS2_ERR_DEVICE_CHECK
    assert torch.isfinite(out.float()).all()


def test_count_out_of_range_is_clamped_and_reported():
    w = W.make_workload(0, lengths=[700], n_sparse=1)
    dev = torch.device("cuda")
    d = W.to_device(w, dev)
    cache = hs2.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, w.n_q, w.n_heads, d["k_scale"], d["v_scale"])
    cap = min(int(w.kv_len.max()), w.topk + w.window)
    idx = torch.arange(cap, dtype=torch.int32, device=dev).reshape(1, cap).contiguous()
    cnt = torch.full((1,), cap + 100, dtype=torch.int32, device=dev)
    out = torch.empty((1, 1, w.n_heads, 128), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(hs2.workspace_size(cache, w.topk, w.window), dtype=torch.uint8, device=dev)
    hs2.sparse_gather_attn(cache, d["q_sparse"][0], idx, cnt, out, ws)
    with pytest.raises(hs2.HS2Error) as e:
        hs2.read_device_status(ws)
    assert e.value.status == HS2_ERR_DEVICE_CHECK


def test_negative_or_nan_scores_are_reported_by_the_selection():
    """hs2_topk_select on caller scores that break the non-negative order: the call completes
    and the device status reports a check, for a split row and for many unsplit rows."""
    dev = torch.device("cuda")
    for lens, n_q, bad in (((50000,), 1, float("nan")), ((3000, 3100), 80, -0.0)):
        k = torch.zeros((max(lens), 128), dtype=torch.bfloat16, device=dev)
        cache = hs2.KvCache(k, k, [0] * len(lens), lens, n_q, 16)
        rows = len(lens) * n_q      # 160 rows: one CTA per row; one row: split over segments
        s = torch.rand((rows, max(lens)), device=dev)
        s[-1, 1000] = bad
        idx = torch.empty((rows, 1152), dtype=torch.int32, device=dev)
        cnt = torch.empty(rows, dtype=torch.int32, device=dev)
        ws = torch.empty(hs2.workspace_size(cache), dtype=torch.uint8, device=dev)
        hs2.topk_select(cache, s, idx, cnt, ws)
        with pytest.raises(hs2.HS2Error) as e:
            hs2.read_device_status(ws)
        assert e.value.status == HS2_ERR_DEVICE_CHECK
        s[-1, 1000] = 0.5
        hs2.topk_select(cache, s, idx, cnt, ws)
        hs2.read_device_status(ws)
