"""The synthetic input recipe (workloads/), checked on CPU.

The recipe: seed 1000 + workload id; sequences packed one after another in the cache; the
ragged decode batch draws its lengths uniformly from 65,536..131,072; every normal draw is
float32 N(0, 1) rounded to bf16; a needle is a key row 2 u sqrt(d) + N(0, 0.1^2) with u the
unit mean of its query row's heads, placed among that row's candidates (before the window);
FP8 caches hold the bf16 rows quantised per row (scale = row max / 448, e4m3 codes).
"""
import numpy as np
import pytest

import workloads as W


def small(kv_dtype="bf16", **kw):
    cfg = dict(name="t", batch=3, n_q=2, n_heads=16, n_sparse=2, kv_dtype=kv_dtype,
               lengths=(3000, 1500, 5000), needles=6)
    cfg.update(kw)
    return W.make_workload(cfg, seed=11)


def test_seeded_and_reproducible():
    a, b = W.make_workload(0), W.make_workload(0)
    assert a.seed == 1000
    for key in ("k", "v", "q_full", "q_sparse", "kv_len", "kv_start"):
        assert np.array_equal(getattr(a, key), getattr(b, key)), key
    c = W.make_workload(0, seed=1001)
    assert not np.array_equal(a.k, c.k)


def test_sequences_are_packed_in_order():
    w = small()
    assert list(w.kv_len) == [3000, 1500, 5000]
    assert list(w.kv_start) == [0, 3000, 4500]
    assert w.kv_rows == 9500
    assert w.position(2, 1) == 4999 and w.position(0, 0) == 2998


def test_ragged_batch_lengths_lie_in_their_range():
    w = W.make_workload(1)
    assert w.batch == 8 and w.seed == 1001
    assert (w.kv_len >= 65536).all() and (w.kv_len <= 131072).all()
    assert len(set(w.kv_len.tolist())) > 1


def test_draws_are_bf16_rounded_standard_normals():
    w = small(needles=0)
    k = W.bf16_bits_to_f32(w.k).astype(np.float64)
    assert np.array_equal(W.f32_to_bf16_bits(k.astype(np.float32)), w.k)   # already bf16
    assert abs(k.mean()) < 0.01 and abs(k.std() - 1.0) < 0.01
    q = W.bf16_bits_to_f32(w.q_sparse).astype(np.float64)
    assert abs(q.std() - 1.0) < 0.02


def test_needles_point_along_their_query_and_sit_before_the_window():
    w = small()
    qf = W.bf16_bits_to_f32(w.q_full).astype(np.float64)
    k = W.bf16_bits_to_f32(w.k).astype(np.float64)
    d = w.head_dim
    for b in range(w.batch):
        pos, row = w.needle_pos[b], w.needle_row[b]
        assert len(pos) == 6 and len(set(pos.tolist())) == 6
        for t, i in zip(pos, row):
            p = w.position(b, int(i))
            assert 0 <= t < p - w.window + 1          # a candidate of its row, not in the window
            m = qf[b, int(i)].mean(axis=0)
            u = m / np.linalg.norm(m)
            key = k[w.kv_start[b] + t]
            assert abs(np.linalg.norm(key) - 2.0 * np.sqrt(d)) < 0.05 * 2.0 * np.sqrt(d)
            assert key @ u / np.linalg.norm(key) > 0.99


@pytest.mark.parametrize("which", ["k", "v"])
def test_fp8_rows_are_the_bf16_rows_quantised(which):
    wb, wf = small("bf16"), small("fp8")
    x = W.bf16_bits_to_f32(getattr(wb, which)).astype(np.float64)
    codes, scale = getattr(wf, which), getattr(wf, which + "_scale")
    amax = np.abs(x).max(axis=1)
    assert np.allclose(scale, (amax / 448.0).astype(np.float32), rtol=2 ** -23, atol=0)
    # decode the OCP e4m3fn codes from the format's definition (bias 7, subnormals at e = 0)
    c = codes.astype(np.int64)
    sgn = np.where(c & 0x80, -1.0, 1.0)
    e, m = (c >> 3) & 0xF, c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7))
    assert not ((e == 15) & (m == 7)).any()          # no NaN code
    y = sgn * mag * scale[:, None].astype(np.float64)
    # round to nearest with 3 mantissa bits: within 2^-4 of each value (relative), plus the
    # subnormal step of the row's scale
    tol = 2.0 ** -4 * np.abs(x) + 2.0 ** -9 * scale[:, None].astype(np.float64) + 1e-30
    assert (np.abs(y - x) <= tol).all()
