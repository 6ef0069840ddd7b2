"""hs2_topk_select_noalloc -- the selection step for callers that cannot allocate device memory
(for example a plugin whose host runtime has already reserved the whole device, or a
latency-critical path that must not call cudaMalloc) -- checked through the C ABI against
hs2_topk_select with a caller workspace. Selection is integer work, so the two must agree
exactly, on two calls in a row (the built-in scratch keeps the previous call's contents).
Every way the selection splits its rows is covered: a few rows over a cluster of segments, one
row over more segments than a cluster holds (candidates through the scratch's global buffers),
and many rows of one CTA each. This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import token_level_sparse_hs2_b200 as hs2

pytestmark = pytest.mark.gpu

HS2_ERR_WORKSPACE, HS2_ERR_DEVICE_CHECK = 3, 5


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


def cache_for(lens, n_q=1):
    # the selection reads only the scores and the sequence geometry: every sequence views the
    # same rows of one small cache (rows [0, T_b)), which the view allows
    dev = torch.device("cuda")
    k = torch.zeros((max(lens), 128), dtype=torch.bfloat16, device=dev)
    return hs2.KvCache(k, k, [0] * len(lens), lens, n_q, 32), dev


def compare_twice(lens, draws, n_q=1):
    cache, dev = cache_for(lens, n_q)
    B = len(lens) * n_q
    ws = torch.empty(hs2.workspace_size(cache), dtype=torch.uint8, device=dev)
    for call, (seed, quant) in enumerate(draws):
        s = torch.from_numpy(scores_for(lens * n_q, seed, quant)).to(dev)
        idx_a = torch.full((B, 1152), -1, dtype=torch.int32, device=dev)
        cnt_a = torch.zeros(B, dtype=torch.int32, device=dev)
        idx_b = torch.full((B, 1152), -2, dtype=torch.int32, device=dev)
        cnt_b = torch.full((B,), -1, dtype=torch.int32, device=dev)
        hs2.topk_select(cache, s, idx_a, cnt_a, ws)
        hs2.read_device_status(ws)
        hs2.topk_select_noalloc(cache, s, idx_b, cnt_b)
        hs2.noalloc_read_status()
        ca, cb = cnt_a.cpu().numpy(), cnt_b.cpu().numpy()
        assert np.array_equal(ca, cb), (call, ca, cb)
        ia, ib = idx_a.cpu().numpy(), idx_b.cpu().numpy()
        for r in range(B):
            assert np.array_equal(ia[r, :ca[r]], ib[r, :cb[r]]), (call, r)


def test_noalloc_selection_matches_workspace_selection():
    # three rows, each split over at most 7 segments of one thread-block cluster
    compare_twice((100000, 60003, 4000), [(11, 0), (12, 8)])


def test_noalloc_selection_over_many_segments():
    # one row of about 300k positions: 19 segments, more than a cluster holds, so the
    # candidates go through the scratch's global buffers and arrival counters, which the
    # second call must find reset
    compare_twice((300007,), [(21, 0), (22, 4)])


def test_noalloc_selection_many_rows():
    # 4 sequences x 40 query rows = 160 rows: one CTA per row, no split
    compare_twice((1900, 4999, 3001, 2222), [(31, 0), (32, 16)], n_q=40)


def test_noalloc_rejects_a_plan_above_the_builtin_scratch():
    # 60 rows of 200,000 positions split over many segments need more than 4 MiB: refused on
    # the host with the workspace status, nothing launched, the outputs left as they were
    lens = (200000,) * 60
    cache, dev = cache_for(lens)
    s = torch.zeros((60, 200000), dtype=torch.float32, device=dev)
    idx = torch.full((60, 1152), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((60,), -7, dtype=torch.int32, device=dev)
    with pytest.raises(hs2.HS2Error) as e:
        hs2.topk_select_noalloc(cache, s, idx, cnt)
    assert e.value.status == HS2_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (idx == -7).all() and (cnt == -7).all()


def test_noalloc_reports_a_negative_score_and_clears_it():
    lens = (100000, 4000)
    cache, dev = cache_for(lens)
    s = torch.from_numpy(scores_for(lens, 41, 0)).to(dev)
    s[0, 777] = -1.0          # breaks the bit-pattern order the radix select relies on
    idx = torch.empty((2, 1152), dtype=torch.int32, device=dev)
    cnt = torch.empty(2, dtype=torch.int32, device=dev)
    hs2.topk_select_noalloc(cache, s, idx, cnt)
    with pytest.raises(hs2.HS2Error) as e:
        hs2.noalloc_read_status()
    assert e.value.status == HS2_ERR_DEVICE_CHECK
    hs2.noalloc_read_status()   # the read cleared it
    s[0, 777] = 1.0
    hs2.topk_select_noalloc(cache, s, idx, cnt)
    hs2.noalloc_read_status()   # a clean call reports nothing


def test_noalloc_status_reports_a_bounded_wait_that_ran_out():
    """The built-in array's status word carries a kernel's timeout to hs2_noalloc_read_status
    (the self-test kernel's wait, which nothing satisfies, runs out after 20 ms), the read clears
    it, and a selection afterwards runs and reports nothing."""
    assert hs2.selftest_wait_timeout_noalloc(20000) == 6       # HS2_ERR_TIMEOUT
    hs2.noalloc_read_status()                                  # cleared by the read
    compare_twice((60003,), [(51, 0)])
