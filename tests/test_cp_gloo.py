"""The context-parallel decode orchestration on CPU: world sizes 2 and 3 over gloo (127.0.0.1).

cp_block_decode is run unchanged by two or three processes, each holding one token range of a
sequence (one case puts a whole shard inside the forced window, so it offers no candidates),
with its collectives over gloo and its per-shard operations replaced by a float64 CPU stand-in
written here (the oracle's attention and selection on the shard, numpy merges). The merged
results must equal the oracle's single-process block over the whole context: full-layer output
and lse, the selection (exact), and every sparse layer. This checks the exchange steps -- their
order, shapes and the merges they feed -- without a GPU; the GPU kernels behind the same steps
are checked against the oracle in test_gpu_cp.py.
"""
import copy
import math
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W


def workload():
    return W.make_workload(dict(name="cp_cpu", batch=1, n_q=1, n_heads=4, n_sparse=2,
                                kv_dtype="bf16", lengths=(700,), needles=3, topk=64, window=16),
                           seed=44)


class CpuOps:
    """Per-shard operations of the block in float64 on the CPU (test stand-in)."""

    def __init__(self, w):
        import oracle
        self.oracle = oracle
        self.w = w

    def _kv(self, cache, which):
        from tests.test_oracle_pins import dense_f64
        k = np.asarray(dense_f64(self.w, which), dtype=np.float64)
        s = int(cache.kv_start[0])
        return k[s:s + int(cache.kv_len[0])]

    def _q(self, q):
        return torch.from_numpy(W.bf16_bits_to_f32(np.asarray(q)).astype(np.float64)).numpy() \
            .reshape(self.w.n_heads, 128)

    def full_attn(self, cache, q, out, lse, ws, scale=None):
        o, l, _ = self.oracle.full_attn(cache, rows=[0], q=q)
        out.copy_(torch.from_numpy(o.reshape(out.shape)))
        lse.copy_(torch.from_numpy(l.reshape(lse.shape)))

    def lse_merge(self, part_out, part_lse, out, lse=None):
        po, pl = part_out.double().numpy(), part_lse.double().numpy()
        M = pl.max(axis=0)
        wgt = np.where(np.isneginf(pl), 0.0, np.exp(pl - M))
        L = wgt.sum(axis=0)
        o = (wgt[..., None] * po).sum(axis=0) / L[..., None]
        out.copy_(torch.from_numpy(o.reshape(out.shape)))
        if lse is not None:
            lse.copy_(torch.from_numpy((M + np.log(L)).reshape(lse.shape)))

    def score_pass(self, cache, q, lse, scores, ws, scale=None):
        k = self._kv(cache, "k")
        c = 1.0 / math.sqrt(128)
        logits = c * self._q(q) @ k.T                        # [H, T_local]
        s = np.exp(logits - lse.double().numpy().reshape(-1, 1)).sum(axis=0)
        scores.copy_(torch.from_numpy(s.reshape(scores.shape)))

    def topk_select(self, cache, scores, idx, cnt, ws, topk, window):
        i, c = self.oracle.select_rows(cache, [0], scores.numpy(), topk, window, fp32=True)
        idx[0, :c[0]] = torch.from_numpy(i[0, :c[0]])
        cnt[0] = int(c[0])

    def cp_pack_candidates(self, cache, offset, global_len, scores, idx, cnt, keys, topk, window):
        keys.zero_()
        n = 0
        for t in idx[0, :int(cnt[0])].tolist():
            g = offset[0] + t
            if g < global_len[0] - window:
                bits = int(np.float32(scores[0, t]).view(np.uint32))
                key = (bits << 32) | (0xffffffff - g)
                keys[0, n] = key - (1 << 64) if key >= 1 << 63 else key
                n += 1

    def cp_merge_select(self, all_keys, global_len, idx, count, topk, window):
        p = global_len[0] - 1
        nc = max(0, p - window + 1)
        if nc <= topk:
            sel = list(range(p + 1))
        else:
            keys = sorted((k & 0xffffffffffffffff for k in all_keys.flatten().tolist()),
                          reverse=True)[:topk]
            sel = sorted(0xffffffff - (k & 0xffffffff) for k in keys) + list(range(nc, p + 1))
        idx[0, :len(sel)] = torch.tensor(sel, dtype=torch.int32)
        count[0] = len(sel)

    def cp_localize(self, offset, local_len, idx, count, idx_loc, cnt_loc):
        S = np.asarray(idx[0, :int(count[0])])
        mine = S[(S >= offset[0]) & (S < offset[0] + local_len[0])] - offset[0]
        idx_loc[0, :len(mine)] = torch.from_numpy(mine.astype(np.int32))
        cnt_loc[0] = len(mine)

    def sparse_gather_attn_partial(self, cache, q, idx, cnt, out, lse, ws, scale=None):
        n = int(cnt[0])
        if n == 0:
            out.zero_()
            lse.fill_(-math.inf)
            return
        sel = np.asarray(idx[0, :n])
        k, v = self._kv(cache, "k")[sel], self._kv(cache, "v")[sel]
        logits = (1.0 / math.sqrt(128)) * self._q(q) @ k.T   # [H, n]
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        L = e.sum(axis=1, keepdims=True)
        out.copy_(torch.from_numpy(((e / L) @ v).reshape(out.shape)))
        lse.copy_(torch.from_numpy((m + np.log(L)).reshape(lse.shape)))


class ShardCache:
    """The shard as a workload view (rows [start + offset, + T_local) of the same arrays)."""

    def __init__(self, w, offset, local_len):
        self.w = copy.copy(w)
        self.w.kv_start = np.array([int(w.kv_start[0]) + offset], dtype=np.int64)
        self.w.kv_len = np.array([local_len], dtype=np.int32)

    def __getattr__(self, name):
        return getattr(self.w, name)


def _rank(rank, world, port, bounds, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from token_level_sparse_hs2_b200 import cp
        w = workload()
        off, tl = bounds[rank], bounds[rank + 1] - bounds[rank]
        cache = ShardCache(w, off, tl)
        ops = CpuOps(w)

        def gather(x):
            parts = [torch.empty_like(x) for _ in range(world)]
            dist.all_gather(parts, x.contiguous())
            return torch.stack(parts)

        H = w.n_heads
        out = torch.empty((1, 1, H, 128), dtype=torch.float64)
        outs = [torch.empty_like(out) for _ in range(w.n_sparse)]
        q_full = torch.from_numpy(np.asarray(w.q_full, dtype=np.uint16).reshape(-1).copy())
        q_sparse = [torch.from_numpy(np.asarray(w.q_sparse[l], dtype=np.uint16).reshape(-1).copy())
                    for l in range(w.n_sparse)]
        res = cp.cp_block_decode(cache, off, int(w.kv_len[0]), q_full, q_sparse, out, outs,
                                 None, gather, topk=w.topk, window=w.window, ops=ops)
        q.put((rank, out.numpy(), [o.numpy() for o in outs], res["lse"].numpy(),
               res["idx"].numpy(), res["count"].numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [[0, 350, 700], [0, 650, 700], [0, 400, 690, 700]])
def test_cp_decode_over_gloo_equals_the_whole_context(oracle_lib, bounds):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world = len(bounds) - 1
    port = 29700 + os.getpid() % 1000 + bounds[1] % 97 + 101 * (world - 2)
    procs = [ctx.Process(target=_rank, args=(r, world, port, bounds, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = []
    import queue as _queue
    import time
    deadline = time.time() + 300
    while len(got) < len(procs) and time.time() < deadline:
        try:
            got.append(q.get(timeout=2))
        except _queue.Empty:
            if any(p.exitcode not in (None, 0) for p in procs):
                break                       # a rank failed: its traceback is in the output
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    res = sorted(got, key=lambda x: x[0])
    assert len(res) == len(procs)
    w = workload()
    ref = oracle_lib.block(w)
    p = w.position(0, 0)
    nc = p - w.window + 1
    kth = np.sort(ref["scores"][0, :nc])[::-1][w.topk - 1]
    for rank, o, outs, lse, idx, cnt in res:
        # the exchanged partial results are float32 (as on the GPU)
        assert np.allclose(o.reshape(ref["o_full"].shape), ref["o_full"], atol=1e-6)
        assert np.allclose(lse.reshape(ref["lse"].shape), ref["lse"], atol=1e-5)
        c = int(cnt[0])
        assert c == int(ref["count"][0])
        S, R = set(idx[0, :c].tolist()), set(ref["idx"][0, :c].tolist())
        for t in S ^ R:                # only float32 near-ties may differ
            assert abs(ref["scores"][0, t] - kth) <= 1e-5 * kth, t
        assert len(S ^ R) <= 2
        for l in range(w.n_sparse):
            sp = oracle_lib.sparse_attn(w, w.q_sparse[l], [0], idx, cnt)
            assert np.allclose(outs[l].reshape(sp.shape), sp, atol=1e-6)
        if not S ^ R:
            for l in range(w.n_sparse):
                assert np.allclose(outs[l].reshape(ref["o_sparse"][l].shape), ref["o_sparse"][l],
                                   atol=1e-6)
