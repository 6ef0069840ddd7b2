"""Seeded synthetic inputs for the HySparse2 hybrid-block attention path.

The oracle (CPU, fp64) and the CUDA path consume exactly the bytes drawn here. This module holds
none of the method's arithmetic: it draws normal variates, rounds them to the storage formats the
path reads (bf16, or FP8-e4m3 with one fp32 scale per token), and plants "needle" keys, i.e.
keys aligned with a query so that the full-attention layer should select them.

The pages measure on agent trajectories and retrieval suites (RULER, MRCR, GraphWalks) that are
not available here; needle-in-noise inputs with the same context lengths (4k..1M tokens) and
action shapes (1..512 new tokens) stand in for them.

Recipe (one numpy ``default_rng(seed)`` per workload, draws in this order):
  1. context lengths (only where a range is given),
  2. Q of the full-attention layer, 3. K, 4. V, 5. Q of each sparse layer,
  6. for each needle: its keyed query row and its position, 7. needle noise.
All normal draws are float32 N(0,1) rounded to bf16 with round-to-nearest-even.
Needle key: k = 2.0 * u * sqrt(d) + N(0, 0.1^2) per element, with u the unit vector along the
mean over heads of the keyed row's full-layer query; the position is uniform (without
replacement) among the keyed row's non-window positions [0, p - window + 1).
FP8: per cache row, scale = max|x| / 448 (1.0 for an all-zero row), code = e4m3fn(x / scale)
rounded to nearest even (torch's float8_e4m3fn cast) after clamping to [-448, 448].
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch

HEAD_DIM = 128
TOPK = 1024
WINDOW = 128
E4M3_MAX = 448.0

# The five workloads: decode at 4k / ragged 64k-128k / 1M (FP8), a 512-token action chunk at
# 256k, and a 32k causal prefill. Each is 1 full-attention layer plus n_sparse sparse layers.
CONFIGS = {
    0: dict(name="decode_b1_t4k_h16_bf16", batch=1, n_q=1, n_heads=16, n_sparse=2,
            kv_dtype="bf16", lengths=(4096,), needles=8),
    1: dict(name="decode_b8_t64k-128k_h32_bf16", batch=8, n_q=1, n_heads=32, n_sparse=3,
            kv_dtype="bf16", lengths=("uniform", 65536, 131072), needles=64),
    2: dict(name="decode_b1_t1m_h32_fp8", batch=1, n_q=1, n_heads=32, n_sparse=3,
            kv_dtype="fp8", lengths=(1048576,), needles=256),
    3: dict(name="chunk_b2_q512_at256k_h32_bf16", batch=2, n_q=512, n_heads=32, n_sparse=3,
            kv_dtype="bf16", lengths=(262656,), needles=128),
    4: dict(name="prefill_b1_s32k_h32_bf16", batch=1, n_q=32768, n_heads=32, n_sparse=3,
            kv_dtype="bf16", lengths=(32768,), needles=512),
}


@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    batch: int
    n_q: int
    n_heads: int
    head_dim: int
    n_sparse: int
    kv_dtype: str                 # "bf16" or "fp8"
    topk: int
    window: int
    kv_len: np.ndarray            # int32 [B]: tokens in the cache of sequence b (T_b)
    kv_start: np.ndarray          # int64 [B]: first cache row of sequence b
    k: np.ndarray                 # uint16 bf16 bits [rows, d], or uint8 e4m3 codes [rows, d]
    v: np.ndarray
    k_scale: Optional[np.ndarray]  # float32 [rows] (FP8 only)
    v_scale: Optional[np.ndarray]
    q_full: np.ndarray            # uint16 bf16 bits [B, n_q, H, d]
    q_sparse: np.ndarray          # uint16 bf16 bits [L, B, n_q, H, d]
    needle_pos: List[np.ndarray]  # per sequence: positions (within the sequence) of needles
    needle_row: List[np.ndarray]  # per sequence: query index i (0..n_q-1) each needle is keyed to

    @property
    def kv_rows(self) -> int:
        return int(self.k.shape[0])

    @property
    def n_rows(self) -> int:
        return self.batch * self.n_q

    def position(self, b: int, i: int) -> int:
        """Cache position of query i of sequence b (the last n_q tokens are the queries)."""
        return int(self.kv_len[b]) - self.n_q + i


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round-to-nearest-even) and return the raw 16-bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (u.astype(np.uint32) << 16).view(np.float32)


def quantize_e4m3_rows(x: np.ndarray):
    """Per-row FP8-e4m3 storage: returns (codes uint8 [rows, d], scale float32 [rows])."""
    amax = np.abs(x).max(axis=1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = np.clip(x / scale[:, None], -E4M3_MAX, E4M3_MAX).astype(np.float32)
    codes = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def make_workload(config: int | dict, seed: Optional[int] = None, **overrides) -> Workload:
    """Draw one workload.

    ``config`` is a key of CONFIGS or a dict with the same fields; ``overrides`` replace fields
    (e.g. smaller ``lengths`` for parity cases the oracle finishes in seconds).
    """
    if isinstance(config, int):
        cfg = dict(CONFIGS[config])
        if seed is None:
            seed = 1000 + config
    else:
        cfg = dict(config)
    cfg.update(overrides)
    if seed is None:
        seed = 0
    topk = int(cfg.get("topk", TOPK))
    window = int(cfg.get("window", WINDOW))
    d = int(cfg.get("head_dim", HEAD_DIM))
    B, n_q, H, L = int(cfg["batch"]), int(cfg["n_q"]), int(cfg["n_heads"]), int(cfg["n_sparse"])
    rng = np.random.default_rng(seed)

    lens = cfg["lengths"]
    if lens and lens[0] == "uniform":
        kv_len = rng.integers(int(lens[1]), int(lens[2]), size=B, endpoint=True).astype(np.int32)
    elif len(lens) == 1:
        kv_len = np.full(B, int(lens[0]), dtype=np.int32)
    else:
        kv_len = np.asarray(lens, dtype=np.int32)
        assert kv_len.shape == (B,)
    if np.any(kv_len < n_q):
        raise ValueError("every sequence must hold at least n_q tokens")
    kv_start = np.zeros(B, dtype=np.int64)
    kv_start[1:] = np.cumsum(kv_len.astype(np.int64))[:-1]
    rows = int(kv_len.astype(np.int64).sum())

    q_full = _normal(rng, (B, n_q, H, d))
    k = _normal(rng, (rows, d))
    v = _normal(rng, (rows, d))
    q_sparse = _normal(rng, (L, B, n_q, H, d))
    q_full = f32_to_bf16_bits(q_full)
    q_sparse = f32_to_bf16_bits(q_sparse)
    qf = bf16_bits_to_f32(q_full)

    n_needles = int(cfg.get("needles", 0))
    needle_pos, needle_row = [], []
    plan = []
    for b in range(B):
        pos_b, row_b = [], []
        # rows whose candidate range [0, p - window + 1) is non-empty; prefer rows where the
        # candidates outnumber the budget so the needle has to win a real selection
        p = kv_len[b] - n_q + np.arange(n_q)
        ncand = p - window + 1
        eligible = np.nonzero(ncand > topk)[0]
        if eligible.size == 0:
            eligible = np.nonzero(ncand > 0)[0]
        used = set()
        for _ in range(n_needles if eligible.size else 0):
            i = int(eligible[rng.integers(0, eligible.size)])
            hi = int(ncand[i])
            for _try in range(64):
                t = int(rng.integers(0, hi))
                if t not in used:
                    break
            else:
                continue
            used.add(t)
            pos_b.append(t)
            row_b.append(i)
        needle_pos.append(np.asarray(pos_b, dtype=np.int64))
        needle_row.append(np.asarray(row_b, dtype=np.int64))
        plan.append((b, pos_b, row_b))
    k = k.copy()
    for b, pos_b, row_b in plan:
        for t, i in zip(pos_b, row_b):
            m = qf[b, i].mean(axis=0)
            u = m / np.linalg.norm(m)
            noise = (0.1 * rng.standard_normal(size=d)).astype(np.float32)
            k[kv_start[b] + t] = (2.0 * u * np.sqrt(d) + noise).astype(np.float32)

    if cfg["kv_dtype"] == "bf16":
        k_st, v_st, ks, vs = f32_to_bf16_bits(k), f32_to_bf16_bits(v), None, None
    elif cfg["kv_dtype"] == "fp8":
        # the cache holds bf16 values quantised to FP8 per token
        kb = bf16_bits_to_f32(f32_to_bf16_bits(k))
        vb = bf16_bits_to_f32(f32_to_bf16_bits(v))
        k_st, ks = quantize_e4m3_rows(kb)
        v_st, vs = quantize_e4m3_rows(vb)
    else:
        raise ValueError(cfg["kv_dtype"])

    return Workload(name=str(cfg.get("name", "custom")), seed=int(seed), batch=B, n_q=n_q,
                    n_heads=H, head_dim=d, n_sparse=L, kv_dtype=cfg["kv_dtype"], topk=topk,
                    window=window, kv_len=kv_len, kv_start=kv_start, k=k_st, v=v_st,
                    k_scale=ks, v_scale=vs, q_full=q_full, q_sparse=q_sparse,
                    needle_pos=needle_pos, needle_row=needle_row)


def sample_rows(w: Workload, n: int, seed: int = 7, extra=()) -> np.ndarray:
    """Seeded sample of flat query rows (b * n_q + i), always including boundary rows."""
    rng = np.random.default_rng(seed)
    total = w.n_rows
    must = set()
    for b in range(w.batch):
        for i in (0, w.n_q - 1):
            must.add(b * w.n_q + i)
        for p in extra:
            i = p - (int(w.kv_len[b]) - w.n_q)
            if 0 <= i < w.n_q:
                must.add(b * w.n_q + i)
        for i in w.needle_row[b][:4]:
            must.add(b * w.n_q + int(i))
    picks = set(int(x) for x in rng.choice(total, size=min(n, total), replace=False))
    return np.asarray(sorted(must | picks), dtype=np.int64)


def to_device(w: Workload, device="cuda"):
    """Moves a workload's arrays to the device as torch tensors (bf16 / uint8 / fp32)."""
    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    if w.kv_dtype == "bf16":
        k, v = bf16(w.k), bf16(w.v)
        ks = vs = None
    else:
        k = torch.from_numpy(np.ascontiguousarray(w.k)).to(device)
        v = torch.from_numpy(np.ascontiguousarray(w.v)).to(device)
        ks = torch.from_numpy(np.ascontiguousarray(w.k_scale)).to(device)
        vs = torch.from_numpy(np.ascontiguousarray(w.v_scale)).to(device)
    q_full = bf16(w.q_full)
    q_sparse = [bf16(w.q_sparse[l]) for l in range(w.n_sparse)]
    return dict(k=k, v=v, k_scale=ks, v_scale=vs, q_full=q_full, q_sparse=q_sparse)
