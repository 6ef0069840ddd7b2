"""hs2_topk_select_noalloc -- the selection step for callers that cannot allocate device memory
(for example a plugin whose host runtime has already reserved the whole device, or a
latency-critical path that must not call cudaMalloc) -- checked through the C ABI against
hs2_topk_select with a caller workspace. Selection is integer work, so the two must agree
exactly, on two calls in a row (the built-in scratch keeps the previous call's contents).
This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import token_level_sparse_hs2_b200 as hs2
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from token_level_sparse_hs2_b200 import build
    build.build()


def scores_for(lens, seed, quant):
    rng = np.random.default_rng(seed)
    s = rng.lognormal(0, 2, size=(len(lens), max(lens))).astype(np.float32)
    if quant:
        s = (np.round(s * quant) / quant).astype(np.float32)
    return s


def test_noalloc_selection_matches_workspace_selection():
    lens = (100000, 60003, 4000)
    w = W.make_workload(dict(name="noalloc", batch=3, n_q=1, n_heads=32, n_sparse=0,
                             kv_dtype="bf16", lengths=lens, needles=0), seed=3)
    d = W.to_device(w)
    cache = hs2.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, 1, w.n_heads)
    dev = d["k"].device
    ws = torch.empty(hs2.workspace_size(cache), dtype=torch.uint8, device=dev)
    for call, (seed, quant) in enumerate([(11, 0), (12, 8)]):
        s = torch.from_numpy(scores_for(lens, seed, quant)).to(dev)
        idx_a = torch.full((3, 1152), -1, dtype=torch.int32, device=dev)
        cnt_a = torch.zeros(3, dtype=torch.int32, device=dev)
        idx_b = torch.full((3, 1152), -2, dtype=torch.int32, device=dev)
        cnt_b = torch.full((3,), -1, dtype=torch.int32, device=dev)
        hs2.topk_select(cache, s, idx_a, cnt_a, ws)
        hs2.read_device_status(ws)
        hs2.topk_select_noalloc(cache, s, idx_b, cnt_b)
        torch.cuda.synchronize()
        ca, cb = cnt_a.cpu().numpy(), cnt_b.cpu().numpy()
        assert np.array_equal(ca, cb), (call, ca, cb)
        ia, ib = idx_a.cpu().numpy(), idx_b.cpu().numpy()
        for r in range(3):
            assert np.array_equal(ia[r, :ca[r]], ib[r, :cb[r]]), (call, r)
