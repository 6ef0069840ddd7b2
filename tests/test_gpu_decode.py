"""GPU parity for the decode hybrid block (one query token per sequence), through the C ABI,
against the fp64 oracle on the same seeded inputs. Tolerances are in tests/gpu_helpers.py."""
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


def decode(**kw):
    cfg = dict(name="decode_small", batch=1, n_q=1, n_heads=32, n_sparse=2, kv_dtype="bf16",
               lengths=(4096,), needles=8)
    cfg.update(kw)
    return W.make_workload(cfg, seed=kw.pop("seed", 17))


def test_config0_decode_4k():
    w = W.make_workload(0)
    g = H().run_block(w)
    H().check_block(w, g)
    sel = set(g["idx"][0, :g["count"][0]].tolist())
    assert set(w.needle_pos[0].tolist()) <= sel


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("heads", [16, 32])
def test_ragged_batch(kv_dtype, heads):
    # several tiles per sequence, ragged tails, tile boundaries shared by two sequences
    w = decode(batch=3, lengths=(3000, 1500, 2701), n_heads=heads, kv_dtype=kv_dtype, needles=5)
    g = H().run_block(w)
    H().check_block(w, g)


def test_short_contexts_keep_everything():
    lens = (1, 2, 127, 128, 129, 1151, 1152, 1153)
    w = decode(batch=len(lens), lengths=lens, n_heads=16, needles=0)
    g = H().run_block(w)
    H().check_block(w, g)
    for b, T in enumerate(lens):
        assert g["count"][b] == min(T, 1152)
        if T <= 1152:
            assert np.array_equal(g["idx"][b, :T], np.arange(T))


@pytest.mark.parametrize("topk,window", [(8, 4), (3, 1), (64, 0), (2048, 256), (2048, 4096)])
def test_budget_variants(topk, window):
    """Budgets up to the largest the C ABI accepts (topk 2,048, window 4,096)."""
    lengths = (700, 3000) if window < 4096 else (7000, 9000)
    w = decode(batch=2, lengths=lengths, topk=topk, window=window, needles=2)
    g = H().run_block(w)
    H().check_block(w, g)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_max_batch(kv_dtype):
    """The largest batch the C ABI accepts (128 sequences), ragged lengths from shorter than the
    budget (every position kept) to several thousand tokens."""
    rng = np.random.default_rng(128)
    lens = tuple(int(x) for x in rng.integers(60, 6000, size=128))
    w = decode(batch=128, lengths=lens, n_heads=16, kv_dtype=kv_dtype, needles=1)
    g = H().run_block(w)
    H().check_block(w, g)


def test_bf16_outputs():
    w = decode(batch=2, lengths=(2000, 900))
    g = H().run_block(w, out_dtype=torch.bfloat16)
    H().check_block(w, g)


def test_workspace_contents_do_not_matter():
    w = decode(batch=2, lengths=(20000, 5000))
    g = H().run_block(w, ws_fill=0xFF)
    H().check_block(w, g)


def test_deterministic():
    w = decode(batch=2, lengths=(40000, 9000), kv_dtype="fp8")
    a = H().run_block(w)
    b = H().run_block(w)
    for key in ("o_full", "lse", "idx", "count"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(np.nan_to_num(a["scores"], nan=-1), np.nan_to_num(b["scores"], nan=-1))
    for x, y in zip(a["o_sparse"], b["o_sparse"]):
        assert np.array_equal(x, y)


def test_all_scores_equal_takes_lowest_indices():
    # identical keys: every score is H/(p+1); the compacted set overflows and the exact
    # fallback must pick [0, topk) plus the window
    w = decode(batch=1, lengths=(20000,), needles=0)
    w.k = np.tile(w.k[:1], (w.kv_rows, 1))
    g = H().run_block(w)
    p = 19999
    nc = p - 127
    assert np.array_equal(g["idx"][0, :1152], np.concatenate([np.arange(1024), np.arange(nc, p + 1)]))
    H().check_block(w, g)


def test_topk_standalone_matches_block():
    import token_level_sparse_hs2_b200 as hs2
    w = decode(batch=2, lengths=(50000, 3000))
    g = H().run_block(w)
    dev = torch.device("cuda")
    scores = torch.from_numpy(g["scores"]).to(dev)
    idx = torch.full_like(torch.from_numpy(g["idx"]), -1).to(dev)
    cnt = torch.zeros(w.n_rows, dtype=torch.int32, device=dev)
    hs2.topk_select(g["cache"], scores, idx, cnt, g["ws"])
    hs2.read_device_status(g["ws"])
    assert np.array_equal(cnt.cpu().numpy(), g["count"])
    for r in range(w.n_rows):
        c = g["count"][r]
        assert np.array_equal(idx[r, :c].cpu().numpy(), g["idx"][r, :c])


@pytest.mark.parametrize("n,quant", [(100000, 0), (100000, 64), (30000, 4), (5000, 0)])
def test_topk_on_synthetic_scores(n, quant):
    """Integer work is bit-exact: arbitrary non-negative scores (heavy ties when quantised,
    denormals and zeros included) against the oracle's fp32 selector."""
    import token_level_sparse_hs2_b200 as hs2
    rng = np.random.default_rng(n + quant)
    lens = (n, n // 2 + 3)
    w = decode(batch=2, lengths=lens, needles=0)
    s = rng.lognormal(0, 2, size=(2, n)).astype(np.float32)
    if quant:
        s = (np.round(s * quant) / quant).astype(np.float32)
    s[:, :50] = np.array([0.0, 1e-45, 3e-39] * 17, dtype=np.float32)[:50]
    d = W.to_device(w)
    cache = hs2.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, 1, w.n_heads)
    dev = torch.device("cuda")
    scores = torch.from_numpy(s).to(dev)
    idx = torch.full((2, 1152), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros(2, dtype=torch.int32, device=dev)
    ws = torch.empty(hs2.workspace_size(cache), dtype=torch.uint8, device=dev)
    hs2.topk_select(cache, scores, idx, cnt, ws)
    hs2.read_device_status(ws)
    ref, rc = oracle.select_rows(w, np.arange(2), s, fp32=True)
    got, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    for r in range(2):
        assert gc[r] == rc[r]
        assert np.array_equal(got[r, :gc[r]], ref[r, :rc[r]])


@pytest.mark.slow
def test_config1_full_size():
    w = W.make_workload(1)
    g = H().run_block(w)
    H().check_block(w, g)
    for b in range(w.batch):
        sel = set(g["idx"][b, :g["count"][b]].tolist())
        assert set(w.needle_pos[b].tolist()) <= sel


@pytest.mark.slow
def test_config2_full_size_fp8():
    w = W.make_workload(2)
    g = H().run_block(w)
    H().check_block(w, g)
    sel = set(g["idx"][0, :g["count"][0]].tolist())
    assert set(w.needle_pos[0].tolist()) <= sel


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_lengths_at_tile_and_budget_edges(kv_dtype):
    """One-token and two-token contexts, lengths at the 64-row tile edges, and the budget edge
    (1,151 keeps everything, 1,152 = budget, 1,153 selects)."""
    lens = (1, 2, 63, 64, 65, 127, 128, 129, 1151, 1152, 1153, 4097)
    w = decode(batch=len(lens), lengths=lens, n_heads=32, kv_dtype=kv_dtype, needles=0)
    g = H().run_block(w)
    H().check_block(w, g)
    for b, T in enumerate(lens):
        assert g["count"][b] == min(T, 1152)


def scatter(w, seed):
    """The same sequences at permuted cache positions with junk rows between and after them,
    so that any read outside a sequence's own rows would change the result."""
    import copy
    from workloads import f32_to_bf16_bits
    rng = np.random.default_rng(seed)
    order = rng.permutation(w.batch)
    gaps = rng.integers(1, 300, size=w.batch)
    rows = int(w.kv_len.astype(np.int64).sum() + gaps.sum() + 77)
    if w.kv_dtype == "bf16":
        junk = lambda: f32_to_bf16_bits((rng.standard_normal((rows, 128)) * 30).astype(np.float32))
    else:
        junk = lambda: rng.integers(0, 0x7e, size=(rows, 128)).astype(np.uint8)
    k, v = junk(), junk()
    ks = vs = None
    if w.kv_dtype == "fp8":
        ks = (rng.random(rows) * 10).astype(np.float32)
        vs = (rng.random(rows) * 10).astype(np.float32)
    start = np.zeros(w.batch, dtype=np.int64)
    pos = 0
    for b in order:
        pos += int(gaps[b])
        start[b] = pos
        s0, n = int(w.kv_start[b]), int(w.kv_len[b])
        k[pos:pos + n], v[pos:pos + n] = w.k[s0:s0 + n], w.v[s0:s0 + n]
        if ks is not None:
            ks[pos:pos + n], vs[pos:pos + n] = w.k_scale[s0:s0 + n], w.v_scale[s0:s0 + n]
        pos += n
    w2 = copy.copy(w)
    w2.k, w2.v, w2.k_scale, w2.v_scale, w2.kv_start = k, v, ks, vs, start
    return w2


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_scattered_sequences_and_custom_scale(kv_dtype):
    """Sequences at permuted, gapped cache positions surrounded by junk rows, and a softmax scale
    other than 1/sqrt(128): decode rows and 9-query chunks."""
    base = decode(batch=5, lengths=(3000, 700, 5000, 129, 2222), kv_dtype=kv_dtype, needles=2)
    w = scatter(base, 5)
    g = H().run_block(w, scale=0.05)
    H().check_block(w, g, scale=0.05)
    base = decode(batch=3, n_q=9, lengths=(900, 2100, 40), kv_dtype=kv_dtype, needles=1,
                  topk=256, window=32)
    w = scatter(base, 6)
    g = H().run_block(w, scale=0.05)
    H().check_block(w, g, scale=0.05)


@pytest.mark.parametrize("kv_dtype,n_q", [("bf16", 1), ("fp8", 1), ("bf16", 40)])
def test_optional_outputs_left_to_the_workspace(kv_dtype, n_q):
    """hs2_block_decode with NULL lse, scores, idx and count (the library keeps them in the
    workspace): the block outputs equal, bit for bit, those of the same call with every output
    given, and that call matches the oracle."""
    import token_level_sparse_hs2_b200 as hs2
    w = decode(batch=3, n_q=n_q, lengths=(5000, 2100, 3333), kv_dtype=kv_dtype, needles=3,
               n_heads=32, n_sparse=2)
    g = H().run_block(w)
    H().check_block(w, g)
    cache, d = g["cache"], g["dev"]
    dev = d["k"].device
    out_full = torch.empty((w.batch, w.n_q, w.n_heads, 128), dtype=torch.float32, device=dev)
    out_sp = [torch.empty_like(out_full) for _ in range(w.n_sparse)]
    nbytes = hs2.workspace_size(cache, flags=hs2.WS_SCORES | hs2.WS_SELECTION)
    assert nbytes > hs2.workspace_size(cache)
    ws = torch.full((nbytes,), 0xff, dtype=torch.uint8, device=dev)
    for _ in range(2):   # twice: the workspace's previous contents must not matter
        hs2.block_decode(cache, d["q_full"], d["q_sparse"], out_full, out_sp, None, None, None,
                         None, ws)
        hs2.read_device_status(ws)
        R = w.n_rows
        np.testing.assert_array_equal(out_full.reshape(R, w.n_heads, 128).cpu().numpy(), g["o_full"])
        for l in range(w.n_sparse):
            np.testing.assert_array_equal(out_sp[l].reshape(R, w.n_heads, 128).cpu().numpy(),
                                          g["o_sparse"][l])
