"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI and compare it
with the fp64 oracle. Tolerances (stated once, used by every test):
  O (bf16 cache)  max-abs 1e-2      O (FP8 cache)  max-abs 3e-2
  scores          |ds| <= 1e-3 * s_ref + 1e-9 * H / (p + 1)
  lse             |dlse| <= 1e-4 + 1e-5 * |lse|
  selection       bit-exact against the oracle's fp32 selector fed the GPU's own scores;
                  >= 99.9 % overlap with the fp64 selector, differences only at near-ties.
"""
import numpy as np
import torch

import oracle
import token_level_sparse_hs2_b200 as hs2
import workloads as W

O_TOL = {"bf16": 1e-2, "fp8": 3e-2}


def run_block(w, out_dtype=torch.float32, topk=None, window=None, ws_fill=None, n_sparse=None,
              stream=None, rows=None, scale=None):
    """Runs the block on the GPU. With `rows`, only those flat query rows are copied back and
    the returned arrays are indexed by position in `rows`."""
    topk = w.topk if topk is None else topk
    window = w.window if window is None else window
    L = w.n_sparse if n_sparse is None else n_sparse
    d = W.to_device(w)
    cache = hs2.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, w.n_q, w.n_heads,
                        d["k_scale"], d["v_scale"])
    dev = d["k"].device
    R, H = w.n_rows, w.n_heads
    stride = int(w.kv_len.max())
    cap = min(stride, topk + window)
    out_full = torch.empty((w.batch, w.n_q, H, 128), dtype=out_dtype, device=dev)
    out_sp = [torch.empty_like(out_full) for _ in range(L)]
    lse = torch.empty((w.batch, w.n_q, H), dtype=torch.float32, device=dev)
    scores = torch.full((R, stride), float("nan"), dtype=torch.float32, device=dev)
    idx = torch.full((R, cap), -1, dtype=torch.int32, device=dev)
    count = torch.zeros(R, dtype=torch.int32, device=dev)
    nbytes = hs2.workspace_size(cache, topk, window)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    if ws_fill is not None:
        ws.fill_(ws_fill)
    hs2.block_decode(cache, d["q_full"], d["q_sparse"][:L], out_full, out_sp, lse, scores, idx,
                     count, ws, topk=topk, window=window, scale=scale, stream=stream)
    hs2.read_device_status(ws, stream)
    torch.cuda.synchronize()
    if rows is None:
        sel = slice(None)
    else:
        sel = torch.as_tensor(np.asarray(rows), device=dev)
    fetch = lambda t: t.reshape(R, *t.shape[2:]) if t.dim() == 4 else t
    return dict(o_full=fetch(out_full)[sel].float().cpu().numpy(),
                lse=lse.reshape(R, H)[sel].cpu().numpy(),
                scores=scores[sel].cpu().numpy(), idx=idx[sel].cpu().numpy(),
                count=count[sel].cpu().numpy(),
                o_sparse=[fetch(o)[sel].float().cpu().numpy() for o in out_sp],
                cache=cache, dev=d, ws=ws, rows=None if rows is None else np.asarray(rows))


def check_scores(w, rows, s_gpu, s_ref):
    for j, r in enumerate(rows):
        p = w.position(*divmod(int(r), w.n_q))
        g = s_gpu[j, :p + 1].astype(np.float64)
        ref = s_ref[j, :p + 1]
        tol = 1e-3 * ref + 1e-9 * w.n_heads / (p + 1)
        bad = np.abs(g - ref) > tol
        assert not bad.any(), (r, int(np.argmax(bad)), g[bad][:4], ref[bad][:4])


def check_block(w, gpu, rows=None, topk=None, window=None, check_sparse=True, scale=None):
    """Full comparison of a GPU block run against the oracle on the listed rows."""
    topk = w.topk if topk is None else topk
    window = w.window if window is None else window
    if gpu.get("rows") is not None:
        rows = gpu["rows"]
        pos = np.arange(len(rows))
    else:
        rows = np.arange(w.n_rows) if rows is None else np.asarray(rows)
        pos = rows
    o_ref, lse_ref, s_ref = oracle.full_attn(w, rows=rows, scale=scale)
    tol = O_TOL[w.kv_dtype]
    err = np.abs(gpu["o_full"][pos] - o_ref).max()
    assert err <= tol, f"O_full max-abs {err}"
    dl = np.abs(gpu["lse"][pos] - lse_ref)
    assert (dl <= 1e-4 + 1e-5 * np.abs(lse_ref)).all(), f"lse max diff {dl.max()}"
    s_gpu = gpu["scores"][pos]
    check_scores(w, rows, s_gpu, s_ref)
    # selection: bit-exact against the fp32 selector on the GPU's own scores
    idx32, cnt32 = oracle.select_rows(w, rows, s_gpu, topk, window, fp32=True)
    for j, r in enumerate(rows):
        c = int(cnt32[j])
        assert int(gpu["count"][pos[j]]) == c, (r, gpu["count"][pos[j]], c)
        assert np.array_equal(gpu["idx"][pos[j], :c], idx32[j, :c]), r
    # agreement with the fp64 selector: >= 99.9 %, differences only at near-ties
    idx64, cnt64 = oracle.select_rows(w, rows, s_ref, topk, window)
    inter = tot = 0
    for j, r in enumerate(rows):
        a = set(gpu["idx"][pos[j], :gpu["count"][pos[j]]].tolist())
        b = set(idx64[j, :cnt64[j]].tolist())
        inter += len(a & b)
        tot += len(b)
        diff = a ^ b
        if diff:
            p = w.position(*divmod(int(r), w.n_q))
            nc = p - window + 1
            kth = np.sort(s_ref[j, :nc])[::-1][topk - 1]
            for t in diff:
                assert abs(s_ref[j, t] - kth) <= 1e-3 * kth, (r, t, s_ref[j, t], kth)
    assert inter >= 0.999 * tot, (inter, tot)
    if check_sparse:
        cnt = gpu["count"][pos]
        for l in range(len(gpu["o_sparse"])):
            ref = oracle.sparse_attn(w, w.q_sparse[l], rows, gpu["idx"][pos], cnt, scale)
            err = np.abs(gpu["o_sparse"][l][pos] - ref).max()
            assert err <= tol, f"sparse layer {l} max-abs {err}"
    return dict(o_ref=o_ref, lse_ref=lse_ref, s_ref=s_ref)
