"""The roofline numerators of bench.py against the per-token figures of the decode step.

A decode step must move, per cached token, K and V once for the full-attention pass, K again for
the score pass, one fp32 score written and read once by the selection: 3 x 256 + 8 = 776 B for a
bf16 cache, 3 x (128 + 4) + 8 = 404 B for e4m3 rows with their fp32 scales. Each sparse layer
gathers min(T, topk + window) rows of K and V per query plus their indices. Queries, outputs and
lse add well under 1 MB. B_min is the same step with K counted once. These figures are checked here
from the workload shapes alone (no GPU), so that a changed byte count cannot slip into a reported
fraction unnoticed.
"""
import functools

import numpy as np
import pytest

import bench
import workloads as W


@functools.lru_cache(maxsize=None)
def workload(cfg):
    return W.make_workload(cfg)


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_decode_bytes_per_token(cfg):
    w = workload(cfg)
    T = int(w.kv_len.astype(np.int64).sum())
    B, H, L = w.batch, w.n_heads, w.n_sparse
    row = 256 if w.kv_dtype == "bf16" else 132
    per_token = 776 if w.kv_dtype == "bf16" else 404
    sel = sum(min(int(t), w.topk + w.window) for t in w.kv_len)
    q, o, lse = B * H * 128 * 2, B * H * 128 * 4, B * H * 4
    # pass 1 reads q, writes o and lse; pass 2 reads q and lse; the selection writes the indices;
    # each sparse layer reads its q and writes its o
    small = (q + o + lse) + (q + lse) + B * (w.topk + w.window) * 4 + L * (q + o)
    ab = bench.algorithmic_bytes(w)
    expect = T * per_token + L * sel * (2 * row + 4) + small
    assert ab["total"] == expect
    assert ab["total_k_once"] == expect - T * row
    # queries, outputs and indices are a small share for the long workloads (0.14 % for the
    # 8-sequence batch with 32 heads and 3 sparse layers)
    if cfg:
        assert small < 2e-3 * ab["total"]


def test_pass1_bytes_are_the_cache_once():
    for cfg in (1, 2):
        w = workload(cfg)
        ab = bench.algorithmic_bytes(w)
        q_o = w.batch * w.n_heads * (128 * 2 + 128 * 4 + 4)
        assert ab["pass1"] == bench.cache_bytes(w) + q_o


def test_cache_bytes_and_the_l2_rule():
    sizes = {c: bench.cache_bytes(workload(c)) for c in range(5)}
    assert sizes[0] == 4096 * 2 * 256                  # 2 MB: fits in L2, flushed per step
    assert sizes[2] == 1048576 * 2 * (128 + 4)         # e4m3 rows plus fp32 scales
    fits = {c for c, s in sizes.items() if s < bench.L2_BYTES}
    assert fits == {0, 4}                              # the 4k decode and the 32k prefill
