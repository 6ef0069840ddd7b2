"""Pins for the oracle's block-level selection (HySparse's 64-token granularity, the variant
HySparse2 replaces with single tokens at the same budget: "HySparse2: How Xiaomi Split the
Transformer to Fix Agent Prefill Costs", section "KV Reuse and Token-Level Sparse Selection").

Each pin checks the oracle against something other than itself: a library sort (block size 1 is
token selection), an exhaustive search over every choice of blocks, hand-computed float32 sums
and the invariants of the definition. Every test runs on the CPU.
"""
import itertools

import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore")


def lexsort_tokens(s, p, k, w):
    nc = max(0, p - w + 1)
    if nc <= k:
        return np.arange(p + 1)
    t = np.arange(nc)
    order = np.lexsort((t, -s[:nc]))
    return np.concatenate([np.sort(order[:k]), np.arange(nc, p + 1)])


@pytest.mark.parametrize("k,win", [(8, 4), (64, 16), (1024, 128)])
def test_block_size_one_is_token_selection(oracle_lib, k, win):
    rng = np.random.default_rng(5)
    for p in list(range(0, 30)) + [200, 1151, 1152, 1153, 3000]:
        for ties in (False, True):
            s = rng.random(p + 1)
            if ties:
                s = np.round(s * 4) / 4
            ref = lexsort_tokens(s, p, k, win)
            assert np.array_equal(oracle_lib.select_blocks_f64(s, p, 1, k, win), ref), (p, ties)
            s32 = s.astype(np.float32)
            ref32 = lexsort_tokens(s32.astype(np.float64), p, k, win)
            assert np.array_equal(oracle_lib.select_blocks_f32(s32, p, 1, k, win), ref32), (p, ties)


@pytest.mark.parametrize("bs,kb,win", [(4, 2, 3), (8, 3, 5), (2, 4, 1), (16, 1, 7)])
def test_selection_captures_the_most_score_mass(oracle_lib, bs, kb, win):
    """Exhaustive search: among every set of kb whole blocks, the selection keeps the one whose
    candidates hold the largest total score (continuous scores make it unique)."""
    rng = np.random.default_rng(bs * 100 + kb)
    k = bs * kb
    for nc in range(k + 1, k + 5 * bs):
        p = nc + win - 1
        s = rng.random(p + 1)
        nb = (nc + bs - 1) // bs
        best, best_mass = None, -1.0
        for comb in itertools.combinations(range(nb), kb):
            pos = [t for j in comb for t in range(j * bs, min((j + 1) * bs, nc))]
            mass = s[pos].sum()
            if mass > best_mass:
                best, best_mass = pos, mass
        ref = np.array(sorted(best) + list(range(nc, p + 1)))
        got = oracle_lib.select_blocks_f64(s, p, bs, k, win)
        assert np.array_equal(got, ref), nc


def test_equal_blocks_go_to_the_lower_index(oracle_lib):
    bs, k, win = 4, 8, 2
    p = 40
    nc = p - win + 1                       # 39 candidates: blocks 0..9, block 9 holds 3
    s = np.full(p + 1, 0.125)
    got = oracle_lib.select_blocks_f64(s, p, bs, k, win)
    assert got.tolist() == list(range(8)) + list(range(nc, p + 1))
    # two blocks with the same (exact, dyadic) sum above the rest: the lower one ranks first
    s = np.full(p + 1, 0.125)
    s[20:24] = [0.5, 0.25, 0.25, 0.5]      # block 5, sum 1.5
    s[8:12] = [0.25, 0.5, 0.5, 0.25]       # block 2, sum 1.5
    s[32:36] = 0.375                       # block 8, sum 1.5
    got = oracle_lib.select_blocks_f64(s, p, bs, k, win)
    assert got.tolist() == list(range(8, 12)) + list(range(20, 24)) + list(range(nc, p + 1))
    got32 = oracle_lib.select_blocks_f32(s.astype(np.float32), p, bs, k, win)
    assert got32.tolist() == got.tolist()


def test_float32_block_score_folds_in_half(oracle_lib):
    e = 2.0 ** -24
    # fold: (1 + e) + (e + e) = 1 + 2^-23, while a left-to-right sum would stay at 1
    s = np.array([1.0, e, e, e], dtype=np.float32)
    assert oracle_lib.block_score_f32(s, 0, 4, 4) == 1.0 + 2.0 ** -23
    # 8 values: ((a0+a4) + (a2+a6)) + ((a1+a5) + (a3+a7)); here a0 = 1 and the other seven are e:
    # 1+e -> 1, e+e -> 2e, then 1 + 2e, 2e + 2e = 4e, finally 1 + 2e + 4e = 1 + 6e (exact)
    s = np.array([1.0] + [e] * 7, dtype=np.float32)
    assert oracle_lib.block_score_f32(s, 0, 8, 8) == 1.0 + 6 * e
    # positions at or past nc count as 0; all-ones blocks sum exactly
    ones = np.ones(300, dtype=np.float32)
    assert oracle_lib.block_score_f32(ones, 64, 300, 64) == 64.0
    assert oracle_lib.block_score_f32(ones, 256, 300, 64) == 44.0
    assert oracle_lib.block_score_f32(ones, 0, 3, 4) == 3.0


def check_block_invariants(S, p, bs, k, win):
    nc = max(0, p - win + 1)
    if nc <= k:
        assert S.tolist() == list(range(p + 1))
        return
    assert np.all(np.diff(S) > 0) and S[0] >= 0 and S[-1] <= p
    assert S[-(p - nc + 1):].tolist() == list(range(nc, p + 1))      # the window, last
    cand = S[S < nc]
    blocks = sorted(set((cand // bs).tolist()))
    assert len(blocks) == k // bs
    expect = [t for j in blocks for t in range(j * bs, min((j + 1) * bs, nc))]
    assert cand.tolist() == expect                                      # whole blocks only
    partial = (nc % bs != 0) and (nc - 1) // bs in blocks
    assert len(S) == k - (bs - nc % bs if partial else 0) + (p - nc + 1)


def test_block_selection_invariants_and_needles(oracle_lib):
    w = W.make_workload(0)            # 4,096-token decode, 16 heads, 8 needles
    _, _, s = oracle_lib.full_attn(w)
    p = w.position(0, 0)
    for bs in (16, 32, 64, 128):
        S = oracle_lib.select_blocks_f64(s[0], p, bs, w.topk, w.window)
        check_block_invariants(S, p, bs, w.topk, w.window)
        assert set(w.needle_pos[0].tolist()) <= set(S.tolist()), bs
        S32 = oracle_lib.select_blocks_f32(s[0].astype(np.float32), p, bs, w.topk, w.window)
        check_block_invariants(S32, p, bs, w.topk, w.window)
    rng = np.random.default_rng(9)
    for p in (1151, 1152, 1153, 1200, 2000, 4095):
        s = rng.random(p + 1)
        for bs in (16, 64, 128):
            check_block_invariants(oracle_lib.select_blocks_f64(s, p, bs, 1024, 128), p, bs,
                                   1024, 128)


def test_rows_wrapper_matches_single_rows(oracle_lib):
    w = W.make_workload(dict(name="blk", batch=2, n_q=3, n_heads=4, n_sparse=1, kv_dtype="bf16",
                             lengths=(700, 1300), needles=3, topk=128, window=32), seed=4)
    rows = np.arange(w.n_rows)
    _, _, s = oracle_lib.full_attn(w, rows=rows)
    for fp32 in (False, True):
        sc = s.astype(np.float32) if fp32 else s
        idx, cnt = oracle_lib.select_blocks_rows(w, rows, sc, 32, fp32=fp32)
        for r in rows:
            p = w.position(r // w.n_q, r % w.n_q)
            one = (oracle_lib.select_blocks_f32 if fp32 else oracle_lib.select_blocks_f64)(
                sc[r], p, 32, w.topk, w.window)
            assert idx[r, :cnt[r]].tolist() == one.tolist()


def test_bad_block_sizes_are_refused(oracle_lib):
    s = np.ones(100)
    for bs in (3, 0, 48):
        with pytest.raises(ValueError):
            oracle_lib.select_blocks_f64(s, 99, bs, 96, 4)
    with pytest.raises(ValueError):
        oracle_lib.select_blocks_f64(s, 99, 64, 96, 4)       # 64 does not divide 96
