"""Pins for the fp64 oracle, each against something other than the oracle itself.

The pages print no worked example, so the pins are: library routines the method reduces to in a
special case (scaled-dot-product attention, a lexicographic sort, torch's FP8 decoding), closed
forms of hand-built cases, and invariants of the definition. Every test runs on the CPU.
Definitions followed: "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs",
section "KV Reuse and Token-Level Sparse Selection" (full layer -> KV cache + token indices;
1,024 tokens + forced window of the 128 most recent; sparse layers reuse both).
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from workloads import Workload, bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.filterwarnings("ignore")


def small(seed=3, **kw):
    cfg = dict(name="small", batch=2, n_q=1, n_heads=4, n_sparse=2, kv_dtype="bf16",
               lengths=(300, 517), needles=4, topk=64, window=16)
    cfg.update(kw)
    return W.make_workload(cfg, seed=seed)


def dense_f64(w, which):
    """Cache K or V widened to float64 through torch's own decoders (bf16 / float8_e4m3fn)."""
    a = w.k if which == "k" else w.v
    if w.kv_dtype == "bf16":
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).double()
    sc = w.k_scale if which == "k" else w.v_scale
    x = torch.from_numpy(a.copy()).view(torch.float8_e4m3fn).double()
    return x * torch.from_numpy(sc).double()[:, None]


def q_f64(q):
    return torch.from_numpy(q.view(np.int16).copy()).view(torch.bfloat16).double()


def sdpa_row(w, q_row, b, idx, scale):
    """torch SDPA (float64, CPU) of one query row's H heads over cache positions idx of seq b."""
    K = dense_f64(w, "k")[w.kv_start[b] + torch.as_tensor(idx)]
    V = dense_f64(w, "v")[w.kv_start[b] + torch.as_tensor(idx)]
    H = q_row.shape[0]
    qq = q_row[None, :, None, :]                       # [1, H, 1, d]
    kk = K[None, None].expand(1, H, -1, -1)
    vv = V[None, None].expand(1, H, -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)[0, :, 0]


# ------------------------------------------------------------------ formats

def test_e4m3_table_matches_torch(oracle_lib):
    tab = oracle_lib.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(tab), nan)
    assert np.array_equal(tab[~nan], ref[~nan])
    assert tab[0x7E] == 448.0 and tab[0x01] == 2.0 ** -9


# ------------------------------------------------------------------ full attention

@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("n_q", [1, 5])
def test_full_attention_matches_sdpa(oracle_lib, kv_dtype, n_q):
    w = small(kv_dtype=kv_dtype, n_q=n_q)
    c = 1.0 / math.sqrt(w.head_dim)
    o, lse, s = oracle_lib.full_attn(w)
    q = q_f64(w.q_full)
    for r in range(w.n_rows):
        b, i = divmod(r, w.n_q)
        p = w.position(b, i)
        ref = sdpa_row(w, q[b, i], b, np.arange(p + 1), c).numpy()
        np.testing.assert_allclose(o[r], ref, rtol=0, atol=1e-12)


def test_single_head_scores_are_softmax_weights(oracle_lib):
    """Hq = 1: s[t] is the softmax weight of t; SDPA with V = identity rows exposes it."""
    w = small(n_heads=1, lengths=(40, 77), needles=0)
    c = 1.0 / math.sqrt(w.head_dim)
    _, lse, s = oracle_lib.full_attn(w)
    q = q_f64(w.q_full)
    for b in range(w.batch):
        p = w.position(b, 0)
        K = dense_f64(w, "k")[w.kv_start[b]:w.kv_start[b] + p + 1]
        eye = torch.eye(p + 1, dtype=torch.float64)
        wts = torch.nn.functional.scaled_dot_product_attention(
            q[b, 0, 0][None, None, None], K[None, None], eye[None, None], scale=c)[0, 0, 0]
        np.testing.assert_allclose(s[b, :p + 1], wts.numpy(), rtol=1e-12, atol=0)


def test_constant_value_rows_give_that_row(oracle_lib):
    w = small(needles=0)
    row = f32_to_bf16_bits(np.linspace(-2, 2, w.head_dim, dtype=np.float32))
    w.v = np.tile(row, (w.kv_rows, 1))
    o, _, _ = oracle_lib.full_attn(w, want_scores=False)
    np.testing.assert_allclose(o, np.broadcast_to(bf16_bits_to_f32(row), o.shape),
                               rtol=1e-13, atol=1e-13)


def hand_case(T=4, H=2):
    """d = 4, so c = 1/2 exactly; q_h = (2, 0, 0, 0) for every head; k_t = (t, 0, 0, 0).
    Logits are l[t] = t, weights e^t / sum_j e^j, lse = log sum_j e^j."""
    d = 4
    k = np.zeros((T, d), np.float32)
    k[:, 0] = np.arange(T)
    v = np.zeros((T, d), np.float32)
    v[:, 1] = np.arange(T) * 0.5
    v[:, 2] = 1.0
    q = np.zeros((1, 1, H, d), np.float32)
    q[..., 0] = 2.0
    return Workload(name="hand", seed=0, batch=1, n_q=1, n_heads=H, head_dim=d, n_sparse=1,
                    kv_dtype="bf16", topk=1, window=1,
                    kv_len=np.array([T], np.int32), kv_start=np.array([0], np.int64),
                    k=f32_to_bf16_bits(k), v=f32_to_bf16_bits(v), k_scale=None, v_scale=None,
                    q_full=f32_to_bf16_bits(q), q_sparse=f32_to_bf16_bits(q[None]),
                    needle_pos=[np.zeros(0, np.int64)], needle_row=[np.zeros(0, np.int64)])


def test_hand_case_closed_form(oracle_lib):
    T, H = 4, 2
    w = hand_case(T, H)
    o, lse, s = oracle_lib.full_attn(w, scale=0.5)
    Z = sum(math.exp(t) for t in range(T))
    wt = np.array([math.exp(t) / Z for t in range(T)])
    assert np.allclose(lse, math.log(Z), rtol=1e-15)
    assert np.allclose(o[0, :, 1], (wt * 0.5 * np.arange(T)).sum(), rtol=1e-15)
    assert np.allclose(o[0, :, 2], 1.0, rtol=1e-15)
    assert np.allclose(o[0, :, [0, 3]], 0.0)
    np.testing.assert_allclose(s[0, :T], H * wt, rtol=1e-14)
    # top-1 of candidates [0, 3) is t = 2; the window of 1 is {3}
    assert oracle_lib.select_f64(s[0, :T], T - 1, 1, 1).tolist() == [2, 3]


def test_identical_keys_give_uniform_scores(oracle_lib):
    w = small(needles=0, n_q=3)
    w.k = np.tile(w.k[:1], (w.kv_rows, 1))
    _, lse, s = oracle_lib.full_attn(w)
    for r in range(w.n_rows):
        p = w.position(*divmod(r, w.n_q))
        np.testing.assert_allclose(s[r, :p + 1], w.n_heads / (p + 1), rtol=1e-13)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_scores_sum_to_heads_and_are_bounded(oracle_lib, kv_dtype):
    w = small(kv_dtype=kv_dtype, n_q=4)
    _, _, s = oracle_lib.full_attn(w)
    for r in range(w.n_rows):
        p = w.position(*divmod(r, w.n_q))
        row = s[r, :p + 1]
        assert abs(row.sum() - w.n_heads) <= 1e-12 * w.n_heads
        assert row.min() >= 0 and row.max() <= w.n_heads


# ------------------------------------------------------------------ selection

def brute_select(s, p, k, w):
    nc = max(0, p - w + 1)
    if nc <= k:
        return np.arange(p + 1)
    t = np.arange(nc)
    order = np.lexsort((t, -s[:nc]))          # score descending, then index ascending
    return np.concatenate([np.sort(order[:k]), np.arange(nc, p + 1)])


@pytest.mark.parametrize("k,win", [(8, 4), (3, 1), (1024, 128), (64, 16)])
def test_selection_matches_lexsort(oracle_lib, k, win):
    rng = np.random.default_rng(11)
    for p in list(range(0, 40)) + [127, 128, 129, 1150, 1151, 1152, 1153, 2047]:
        for kind in ("cont", "ties"):
            s = rng.random(p + 1)
            if kind == "ties":
                s = np.round(s * 4) / 4              # heavy ties
            ref = brute_select(s, p, k, win)
            got = oracle_lib.select_f64(s, p, k, win)
            assert np.array_equal(got, ref), (p, kind)
            got32 = oracle_lib.select_f32(s.astype(np.float32), p, k, win)
            ref32 = brute_select(s.astype(np.float32).astype(np.float64), p, k, win)
            assert np.array_equal(got32, ref32), (p, kind)


def test_selection_all_equal_takes_lowest_indices(oracle_lib):
    p, k, win = 5000, 1024, 128
    got = oracle_lib.select_f64(np.ones(p + 1), p, k, win)
    assert np.array_equal(got, np.concatenate([np.arange(k), np.arange(p - win + 1, p + 1)]))


def test_selection_f32_uses_bit_order(oracle_lib):
    # adjacent floats differ only in the last bit; denormals and +0 are ordered too
    vals = np.array([0.0, 1e-45, 2e-45, 1.0, np.nextafter(np.float32(1), np.float32(2))],
                    dtype=np.float32)
    s = np.concatenate([vals, np.zeros(4, np.float32)])
    got = oracle_lib.select_f32(s, s.size - 1, 2, 4)
    assert got.tolist() == [3, 4, 5, 6, 7, 8]


def check_selection_invariants(idx, count, p, k, win):
    S = idx[:count]
    assert count == min(p + 1, k + win)
    assert np.all(np.diff(S) > 0) and S[0] >= 0 and S[-1] <= p
    wlo = max(0, p - win + 1)
    assert set(range(wlo, p + 1)) <= set(S.tolist())


def test_block_invariants_and_needles(oracle_lib):
    w = W.make_workload(0)            # 4,096-token decode, 16 heads, 8 needles
    out = oracle_lib.block(w)
    p = w.position(0, 0)
    check_selection_invariants(out["idx"][0], out["count"][0], p, w.topk, w.window)
    assert set(w.needle_pos[0].tolist()) <= set(out["idx"][0, :out["count"][0]].tolist())


def test_needles_selected_in_chunk_rows(oracle_lib):
    w = small(n_q=6, lengths=(2000, 2600), needles=6, topk=64, window=16)
    out = oracle_lib.block(w)
    for b in range(w.batch):
        for t, i in zip(w.needle_pos[b], w.needle_row[b]):
            r = b * w.n_q + int(i)
            sel = out["idx"][r, :out["count"][r]]
            assert int(t) in set(sel.tolist())


# ------------------------------------------------------------------ sparse attention

def test_full_budget_sparse_equals_full(oracle_lib):
    """When topk + window covers [0, p], the sparse layer is full causal attention."""
    w = small(n_q=3, topk=600, window=16)
    rows = np.arange(w.n_rows)
    o_full, _, s = oracle_lib.full_attn(w)
    idx, count = oracle_lib.select_rows(w, rows, s)
    for r in rows:
        assert count[r] == w.position(*divmod(r, w.n_q)) + 1
    o_sp = oracle_lib.sparse_attn(w, w.q_full, rows, idx, count)
    assert np.array_equal(o_sp, o_full)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_sparse_matches_sdpa_over_selected_rows(oracle_lib, kv_dtype):
    w = small(kv_dtype=kv_dtype, n_q=2, topk=32, window=8)
    c = 1.0 / math.sqrt(w.head_dim)
    out = oracle_lib.block(w)
    q = q_f64(w.q_sparse[1])
    for r in range(w.n_rows):
        b, i = divmod(r, w.n_q)
        sel = out["idx"][r, :out["count"][r]]
        ref = sdpa_row(w, q[b, i], b, sel, c).numpy()
        np.testing.assert_allclose(out["o_sparse"][1][r], ref, rtol=0, atol=1e-12)


def test_planted_mistake_is_caught(oracle_lib):
    """A plausible slip -- selecting inside the window or dropping the forced window -- must
    fail the lexsort pin; checked by perturbing the oracle's output on the CPU."""
    rng = np.random.default_rng(5)
    p, k, win = 300, 32, 8
    s = rng.random(p + 1)
    ref = brute_select(s, p, k, win)
    got = oracle_lib.select_f64(s, p, k, win)
    assert np.array_equal(got, ref)
    wrong = np.sort(np.lexsort((np.arange(p + 1), -s))[:k + win])   # window not forced
    assert not np.array_equal(wrong, ref)


# ------------------------------------------------------------------ KV append: FP8 quantiser
# "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing", "Inference cost": the shared
# KV cache is FP8; appended rows are quantised per token (scale = max|x| / 448, e4m3 RNE).

def test_e4m3_rne_matches_torch_cast(oracle_lib):
    rng = np.random.default_rng(7)
    ys = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 1e-2, 20000),
                         rng.normal(0, 3e-3, 5000), [0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10]])
    ys = ys.astype(np.float32)
    ref = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_lib.e4m3_rne(float(y)) for y in ys], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_rne_round_trips_every_code_and_ties_go_to_even(oracle_lib):
    table = oracle_lib.e4m3_table()
    finite = [c for c in range(256) if not np.isnan(table[c])]
    for c in finite:
        assert oracle_lib.e4m3_rne(float(table[c])) == c
    pos = sorted(c for c in finite if c < 0x80)           # ascending magnitudes 0 .. 448
    for a, b in zip(pos[:-1], pos[1:]):
        mid = np.float32((table[a] + table[b]) / 2)
        if float(mid) != (table[a] + table[b]) / 2:
            continue                                     # not exactly representable in float32
        even = a if a % 2 == 0 else b
        assert oracle_lib.e4m3_rne(float(mid)) == even
    assert oracle_lib.e4m3_rne(1000.0) == 0x7e and oracle_lib.e4m3_rne(-1000.0) == 0xfe


def test_quantize_rows_scale_codes_and_error_bound(oracle_lib):
    rng = np.random.default_rng(8)
    x = rng.standard_normal((64, 128)).astype(np.float32) * rng.uniform(0.01, 50, (64, 1)).astype(np.float32)
    x[3] = 0.0
    x[5, :] = 0.0
    x[5, 17] = -2.5
    bits = W.f32_to_bf16_bits(x)
    xf = W.bf16_bits_to_f32(bits)
    codes, scale = oracle_lib.quantize_rows(bits)
    amax = np.abs(xf).max(axis=1)
    assert scale[3] == 1.0 and not codes[3].any()
    np.testing.assert_array_equal(scale[amax > 0], (amax[amax > 0] / np.float32(448.0)).astype(np.float32))
    table = oracle_lib.e4m3_table()
    deq = table[codes] * scale[:, None].astype(np.float64)
    # the largest element of each row maps to +-448 exactly; every element within half a step
    big = np.abs(xf).argmax(axis=1)
    assert np.all(np.abs(table[codes[np.arange(64), big]])[amax > 0] == 448.0)
    err = np.abs(deq - xf)
    step = np.maximum(np.abs(xf) / 8.0, 2.0 ** -9 * scale[:, None])    # 3 mantissa bits; subnormal floor
    assert np.all(err <= step * 0.5 + 1e-12)
    assert codes[5, 17] == 0xfe and np.all(codes[5, np.arange(128) != 17] == 0)


def _e4m3_by_torch(y: np.ndarray) -> np.ndarray:
    """torch's float8_e4m3fn cast (round to nearest even) of float32 values clamped to +-448."""
    y = np.clip(y.astype(np.float32), -448.0, 448.0)
    return torch.from_numpy(np.ascontiguousarray(y)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_quantize_rows_codes_are_the_rounded_quotient(oracle_lib):
    """The codes follow value = scale * code: each is the e4m3 rounding of the float32 quotient
    x / scale (numpy's IEEE float32 division), cast by torch -- an implementation independent of
    the oracle's own e4m3 encoder -- on 4,096 random rows whose magnitudes span 2^-20 .. 2^20."""
    rng = np.random.default_rng(81)
    rows = 4096
    mag = np.exp2(rng.uniform(-20, 20, (rows, 1))).astype(np.float32)
    x = rng.standard_normal((rows, 128)).astype(np.float32) * mag
    x[::97] *= rng.uniform(0.0, 1e-3, (x[::97].shape[0], 128)).astype(np.float32)  # tiny tails
    bits = W.f32_to_bf16_bits(x)
    xf = W.bf16_bits_to_f32(bits)
    codes, scale = oracle_lib.quantize_rows(bits)
    amax = np.abs(xf).max(axis=1)
    want_scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    np.testing.assert_array_equal(scale, want_scale)
    quotient = (xf / want_scale[:, None]).astype(np.float32)
    np.testing.assert_array_equal(codes, _e4m3_by_torch(quotient))


def test_quantize_rows_rejects_the_reciprocal_product(oracle_lib):
    """x * rn(1/scale) and rn(x / scale) straddle an e4m3 rounding boundary for some inputs; on
    exactly those the oracle must give the quotient's code (a planted reciprocal form fails)."""
    rng = np.random.default_rng(82)
    found = 0
    for _ in range(64):
        x = (rng.standard_normal((512, 128)) * np.exp2(rng.uniform(-8, 8, (512, 1)))).astype(np.float32)
        bits = W.f32_to_bf16_bits(x)
        xf = W.bf16_bits_to_f32(bits)
        amax = np.abs(xf).max(axis=1)
        sc = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
        q_code = _e4m3_by_torch(xf / sc[:, None])
        r_code = _e4m3_by_torch(xf * (np.float32(1.0) / sc)[:, None])
        rows = np.nonzero((q_code != r_code).any(axis=1))[0]
        if rows.size == 0:
            continue
        codes, _ = oracle_lib.quantize_rows(bits[rows])
        np.testing.assert_array_equal(codes, q_code[rows])
        assert (codes != r_code[rows]).any()
        found += rows.size
        if found >= 8:
            break
    assert found >= 8, "no straddling inputs found"


# ------------------------------------------------------------------ KV Bridging projections

def test_kv_bridge_equals_float64_matmul(oracle_lib):
    """The projections equal a library float64 matmul of the widened bf16 inputs."""
    rng = np.random.default_rng(21)
    m, d = 37, 192
    h = f32_to_bf16_bits(rng.standard_normal((m, d)).astype(np.float32))
    w = f32_to_bf16_bits((rng.standard_normal((256, d)) / np.sqrt(d)).astype(np.float32))
    k, v = oracle_lib.kv_bridge(h, w)
    ref = torch.from_numpy(bf16_bits_to_f32(h).astype(np.float64)) @ \
        torch.from_numpy(bf16_bits_to_f32(w).astype(np.float64)).T
    assert np.allclose(k, ref[:, :128].numpy(), rtol=0, atol=1e-12)
    assert np.allclose(v, ref[:, 128:].numpy(), rtol=0, atol=1e-12)


def test_kv_bridge_selector_weights_copy_features(oracle_lib):
    """One-hot weight rows pick input features: K[:, c] = h[:, 2c], V[:, c] = -h[:, c + 1]."""
    rng = np.random.default_rng(22)
    m, d = 5, 256
    hf = rng.standard_normal((m, d)).astype(np.float32)
    h = f32_to_bf16_bits(hf)
    wf = np.zeros((256, d), dtype=np.float32)
    for c in range(128):
        wf[c, 2 * c] = 1.0
        wf[128 + c, c + 1] = -1.0
    k, v = oracle_lib.kv_bridge(h, f32_to_bf16_bits(wf))
    hb = bf16_bits_to_f32(h).astype(np.float64)
    assert np.array_equal(k, hb[:, 0:256:2])
    assert np.array_equal(v, -hb[:, 1:129])


# ------------------------------------------------------------------ context-parallel decomposition

def test_attention_over_disjoint_shards_merges_to_the_whole(oracle_lib):
    """The reading behind context-parallel decode, pinned in the oracle: softmax attention over a
    union of disjoint position sets is the log-sum-exp merge of the parts (closed form:
    lse = log sum_j e^{lse_j}, O = sum_j e^{lse_j - lse} O_j), and the whole context's scores
    under the merged lse are each shard's scores under that lse."""
    import copy
    w = small(batch=1, lengths=(900,), needles=2, n_heads=4)
    o_ref, lse_ref, s_ref = oracle_lib.full_attn(w)
    parts = []
    for a, b in ((0, 333), (333, 899), (899, 900)):
        ws = copy.copy(w)
        ws.kv_start = np.array([int(w.kv_start[0]) + a], dtype=np.int64)
        ws.kv_len = np.array([b - a], dtype=np.int32)
        o, lse, _ = oracle_lib.full_attn(ws)
        parts.append((o, lse))
    L = np.stack([p[1] for p in parts])                       # [3, 1, H]
    M = L.max(axis=0)
    wgt = np.exp(L - M)
    lse = M + np.log(wgt.sum(axis=0))
    O = sum(wgt[j][..., None] * parts[j][0] for j in range(3)) / wgt.sum(axis=0)[..., None]
    assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)
    assert np.allclose(O, o_ref, rtol=0, atol=1e-12)
    # scores of a shard under the merged lse equal the whole context's scores there
    kd = dense_f64(w, "k").numpy()
    q = q_f64(w.q_full).reshape(w.n_heads, 128)
    logits = (q @ kd[:900].T) / math.sqrt(128)
    s = np.exp(logits - lse.reshape(-1, 1)).sum(axis=0)
    assert np.allclose(s, s_ref[0, :900], rtol=1e-12, atol=0)
