"""GPU parity for block-level selection (HySparse's 64-token granularity at the token variant's
budget; "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "KV
Reuse and Token-Level Sparse Selection"), through the C ABI, against the oracle.

Selection is integer work: bit-exact against the oracle's fp32 block selector fed the same fp32
scores (the block sums fold each block in half in float32 on both sides). Against the fp64
selector on the oracle's own scores the selected sets agree to >= 99.9 %, differences only at
near-ties of the block scores. Sparse layers over a block selection match the oracle's sparse
attention over the same indices (max-abs 1e-2 bf16 / 3e-2 FP8)."""
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


def hs2():
    import token_level_sparse_hs2_b200 as m
    return m


def workload(**kw):
    cfg = dict(name="blocksel", batch=1, n_q=1, n_heads=16, n_sparse=1, kv_dtype="bf16",
               lengths=(4096,), needles=8)
    seed = kw.pop("seed", 23)
    cfg.update(kw)
    return W.make_workload(cfg, seed=seed)


class Rows:
    """Sequence geometry only, for selection on given scores: the cache rows are never read, so
    the oracle gets a one-row placeholder and the GPU uninitialised K/V of the right size."""

    def __init__(self, lengths, n_q=1, topk=1024, window=128):
        self.batch, self.n_q, self.n_heads, self.head_dim = len(lengths), n_q, 16, 128
        self.kv_dtype, self.topk, self.window = "bf16", topk, window
        self.kv_len = np.asarray(lengths, dtype=np.int32)
        self.kv_start = np.concatenate([[0], np.cumsum(self.kv_len)[:-1]]).astype(np.int64)
        self.k = self.v = np.zeros((1, 128), dtype=np.uint16)
        self.k_scale = self.v_scale = None

    @property
    def n_rows(self):
        return self.batch * self.n_q

    def position(self, b, i):
        return int(self.kv_len[b]) - self.n_q + i


def run_blocks(w, scores_np, bs, topk=None, window=None, ws_fill=None):
    m = hs2()
    topk = w.topk if topk is None else topk
    window = w.window if window is None else window
    if isinstance(w, Rows):
        rows = int(w.kv_len.sum())
        k = torch.empty((rows, 128), dtype=torch.bfloat16, device="cuda")
        d = dict(k=k, v=torch.empty_like(k), k_scale=None, v_scale=None)
    else:
        d = W.to_device(w)
    cache = m.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, w.n_q, w.n_heads, d["k_scale"],
                      d["v_scale"])
    dev = d["k"].device
    scores = torch.from_numpy(np.ascontiguousarray(scores_np, dtype=np.float32)).to(dev)
    cap = min(int(w.kv_len.max()), topk + window)
    idx = torch.full((w.n_rows, cap), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros(w.n_rows, dtype=torch.int32, device=dev)
    ws = torch.empty(m.topk_select_blocks_workspace_size(cache, bs, topk, window),
                     dtype=torch.uint8, device=dev)
    if ws_fill is not None:
        ws.fill_(ws_fill)
    m.topk_select_blocks(cache, scores, idx, cnt, ws, block_size=bs, topk=topk, window=window)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy(), dict(cache=cache, dev=d, idx=idx, cnt=cnt)


def assert_exact(w, s, bs, idx, cnt, topk=None, window=None):
    ref, rc = oracle.select_blocks_rows(w, np.arange(w.n_rows), s, bs, topk, window, fp32=True)
    for r in range(w.n_rows):
        assert cnt[r] == rc[r], (r, cnt[r], rc[r])
        assert np.array_equal(idx[r, :cnt[r]], ref[r, :rc[r]]), r


@pytest.mark.parametrize("bs", [16, 32, 64, 128])
@pytest.mark.parametrize("kind", ["lognormal", "ties", "tiny"])
def test_synthetic_scores_bit_exact(bs, kind):
    """Ragged rows (short rows keep everything; a short last block), every block size, heavy
    ties, zeros and denormals."""
    lens = (100_003, 1_200, 1_151, 1_153, 40_000 + 37, 3_000)
    w = Rows(lens)
    rng = np.random.default_rng(bs * 7 + len(kind))
    n = max(lens)
    s = rng.lognormal(0, 2, size=(len(lens), n)).astype(np.float32)
    if kind == "ties":
        s = (np.round(s * 2) / 2).astype(np.float32)
    elif kind == "tiny":
        s = (s * np.float32(1e-38)).astype(np.float32)        # block sums in the denormal range
        s[:, ::7] = 0.0
    idx, cnt, _ = run_blocks(w, s, bs)
    assert_exact(w, s, bs, idx, cnt)


def test_all_equal_scores_take_the_lowest_blocks():
    w = Rows((9_000, 5_000))
    s = np.ones((2, 9_000), dtype=np.float32)
    idx, cnt, _ = run_blocks(w, s, 64)
    for r, T in enumerate((9_000, 5_000)):
        nc = T - 128
        assert cnt[r] == 1024 + 128
        assert idx[r, :cnt[r]].tolist() == list(range(1024)) + list(range(nc, T))


def test_rows_past_shared_memory_use_the_global_path():
    """Blocks beyond the shared-memory stage (32,768 block scores) are selected from global
    memory with the same result: 16-token blocks over a 600,000-token row."""
    w = Rows((600_000,))
    rng = np.random.default_rng(3)
    s = rng.lognormal(0, 1, size=(1, 600_000)).astype(np.float32)
    idx, cnt, _ = run_blocks(w, s, 16)
    assert_exact(w, s, 16, idx, cnt)


@pytest.mark.parametrize("bs", [16, 64, 128])
def test_many_rows_pool_inside_the_select_kernel(bs):
    """148 rows or more: each CTA pools its own row (one launch); chunk rows of two sequences,
    short rows that keep everything among them."""
    w = Rows((6_000, 1_300), n_q=200)
    rng = np.random.default_rng(bs)
    s = rng.lognormal(0, 1, size=(w.n_rows, 6_000)).astype(np.float32)
    idx, cnt, _ = run_blocks(w, s, bs)
    assert_exact(w, s, bs, idx, cnt)


@pytest.mark.parametrize("topk,window", [(256, 64), (2048, 128), (1024, 0)])
def test_budget_variants(topk, window):
    w = Rows((30_000, 7_777))
    rng = np.random.default_rng(topk + window)
    s = rng.random((2, 30_000)).astype(np.float32)
    for bs in (32, 128):
        idx, cnt, _ = run_blocks(w, s, bs, topk=topk, window=window)
        assert_exact(w, s, bs, idx, cnt, topk, window)


def test_workspace_contents_do_not_matter():
    w = Rows((20_000, 6_000))
    s = np.random.default_rng(1).random((2, 20_000)).astype(np.float32)
    a = run_blocks(w, s, 64, ws_fill=0)[:2]
    b = run_blocks(w, s, 64, ws_fill=0xff)[:2]
    assert np.array_equal(a[1], b[1])
    for r in range(2):
        assert np.array_equal(a[0][r, :a[1][r]], b[0][r, :b[1][r]])


@pytest.mark.parametrize("kv_dtype,n_q", [("bf16", 1), ("fp8", 1), ("bf16", 6), ("bf16", 80)])
def test_block_selection_in_the_hybrid_block(kv_dtype, n_q):
    """Full layer on the GPU, block-level selection of its scores, then a sparse layer over the
    selected blocks: selection bit-exact on the GPU's scores and close to the fp64 selector; the
    sparse output matches the oracle over the same indices; needle blocks are kept."""
    from tests import gpu_helpers as G
    m = hs2()
    lens = (12_000, 5_000) if n_q == 1 else (3_000, 2_500)
    w = workload(batch=2, n_q=n_q, lengths=lens, kv_dtype=kv_dtype, needles=4)
    g = G.run_block(w, n_sparse=0)
    rows = np.arange(w.n_rows)
    s_gpu = g["scores"]
    idx, cnt, ctx = run_blocks(w, s_gpu, 64)
    assert_exact(w, s_gpu, 64, idx, cnt)
    # agreement with the fp64 block selector on the oracle's scores
    _, _, s_ref = oracle.full_attn(w, rows=rows)
    idx64, cnt64 = oracle.select_blocks_rows(w, rows, s_ref, 64)
    inter = tot = 0
    for r in rows:
        a = set(idx[r, :cnt[r]].tolist())
        b = set(idx64[r, :cnt64[r]].tolist())
        inter += len(a & b)
        tot += len(b)
        if a != b:
            p = w.position(*divmod(int(r), w.n_q))
            nc = p - w.window + 1
            blk = np.add.reduceat(s_ref[r, :nc], np.arange(0, nc, 64))
            kth = np.sort(blk)[::-1][w.topk // 64 - 1]
            for t in a ^ b:
                assert abs(blk[t // 64] - kth) <= 1e-3 * kth, (r, t)
    assert inter >= 0.999 * tot
    for b in range(w.batch):
        for t, i in zip(w.needle_pos[b], w.needle_row[b]):
            r = b * w.n_q + int(i)
            assert int(t) in set(idx[r, :cnt[r]].tolist())
    # a sparse layer over the block selection
    d = ctx["dev"]
    out = torch.empty((w.batch, w.n_q, w.n_heads, 128), dtype=torch.float32,
                      device=d["k"].device)
    ws = torch.empty(m.workspace_size(ctx["cache"]), dtype=torch.uint8, device=d["k"].device)
    m.sparse_gather_attn(ctx["cache"], d["q_sparse"][0], ctx["idx"], ctx["cnt"], out, ws)
    m.read_device_status(ws)
    ref = oracle.sparse_attn(w, w.q_sparse[0], rows, idx, cnt)
    err = np.abs(out.reshape(w.n_rows, w.n_heads, 128).cpu().numpy() - ref).max()
    assert err <= G.O_TOL[kv_dtype], err


def test_full_size_decode_block_selection():
    """Block selection at the 8 x 64k-128k decode size and the 1M-token size, on synthetic
    scores of the score pass's shape, bit-exact against the oracle."""
    rng = np.random.default_rng(11)
    lens = tuple(int(x) for x in rng.integers(65_536, 131_073, size=8))
    for lengths in (lens, (1_048_576,)):
        w = Rows(lengths)
        s = rng.lognormal(-12, 1.5, size=(len(lengths), max(lengths))).astype(np.float32)
        idx, cnt, _ = run_blocks(w, s, 64)
        assert_exact(w, s, 64, idx, cnt)
