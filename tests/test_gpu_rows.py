"""GPU parity for multi-token query chunks (a short action appended to a long context, and a
causal prefill): every query row gets its own causal attention, scores and selection."""
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


def H():
    from tests import gpu_helpers
    return gpu_helpers


def chunk(**kw):
    cfg = dict(name="chunk_small", batch=2, n_q=40, n_heads=32, n_sparse=2, kv_dtype="bf16",
               lengths=(3000, 5000), needles=6, topk=64, window=16)
    cfg.update(kw)
    return W.make_workload(cfg, seed=kw.pop("seed", 23))


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("heads", [16, 32])
def test_chunk_rows(kv_dtype, heads):
    w = chunk(kv_dtype=kv_dtype, n_heads=heads)
    g = H().run_block(w)
    H().check_block(w, g, topk=64, window=16)


def test_partial_blocks_and_default_budget():
    # 37 queries: the last pass-1 and pass-2 blocks are partial
    w = chunk(n_q=37, lengths=(2000, 1400), topk=1024, window=128)
    g = H().run_block(w)
    H().check_block(w, g)


def test_prefill_small():
    # every position is a query; rows with p < topk + window keep everything
    w = chunk(batch=1, n_q=1500, lengths=(1500,), topk=256, window=32, needles=10)
    rows = W.sample_rows(w, 96, extra=(0, 1, 31, 32, 33, 287, 288, 289, 1499))
    g = H().run_block(w, rows=rows)
    H().check_block(w, g, topk=256, window=32)
    for j, r in enumerate(rows):
        if r < 288:
            assert g["count"][j] == r + 1


def test_chunk_needles_selected():
    w = chunk(n_q=24, lengths=(6000, 4000), needles=8)
    g = H().run_block(w)
    for b in range(w.batch):
        for t, i in zip(w.needle_pos[b], w.needle_row[b]):
            r = b * w.n_q + int(i)
            assert int(t) in set(g["idx"][r, :g["count"][r]].tolist())


@pytest.mark.slow
def test_config3_chunk_full_size():
    w = W.make_workload(3)
    rows = W.sample_rows(w, 12)
    g = H().run_block(w, rows=rows)
    H().check_block(w, g)


@pytest.mark.slow
def test_config4_prefill_full_size():
    w = W.make_workload(4)
    rows = W.sample_rows(w, 320, extra=(0, 1, 126, 127, 128, 129, 1150, 1151, 1152, 1153, 1154,
                                        16383, 16384, 32766, 32767))
    g = H().run_block(w, rows=rows)
    H().check_block(w, g)
    for j, r in enumerate(rows):
        p = int(r)
        assert g["count"][j] == min(p + 1, 1152)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_many_chunked_sequences(kv_dtype):
    """Twelve sequences of 37 queries each (the last blocks of every sequence partial), ragged
    contexts from just above the query count to several thousand tokens."""
    lens = (37, 40, 101, 700, 1300, 2600, 64, 65, 129, 4000, 1153, 900)
    w = chunk(batch=len(lens), n_q=37, lengths=lens, kv_dtype=kv_dtype, n_heads=16,
              topk=128, window=32, needles=1)
    g = H().run_block(w)
    H().check_block(w, g, topk=128, window=32)
