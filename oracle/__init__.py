"""fp64 CPU oracle for HySparse2's KV-Reuse hybrid block (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg import this
package; the CUDA library never does, and the two share no code. The arithmetic lives in
``hs2_oracle.c`` (plain C, double precision, sums in index order); this module only marshals
numpy arrays through ctypes and composes the block:

  full layer   -> O_full, lse, s           (``full_attn``)
  selection    -> S (ascending), |S|        (``select_rows_f64`` / ``select_rows_f32``)
  sparse layers-> O^l over S only          (``sparse_attn``)

Sources: "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs"
(originshq.com), section "KV Reuse and Token-Level Sparse Selection"; "HySparse2: Hybrid Sparse
Attention with Two-Level KV Sharing" (academy.dair.ai), bullets "KV Reuse refinements" and
"Inference cost". The scoring rule, tie-break and softmax scale are readings where the pages are
silent; they are listed with the other readings in the design notes.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hs2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/liboracle.so (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _KV(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int32),
                ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("kv_start", ctypes.c_void_p), ("kv_len", ctypes.c_void_p)]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.hs2o_e4m3_table.argtypes = [P]
        L.hs2o_full_attn.argtypes = [P, P, D, P, I64, P, P, P, I64]
        L.hs2o_full_attn.restype = I32
        L.hs2o_select_f64.argtypes = [P, I64, I32, I32, P]
        L.hs2o_select_f64.restype = I64
        L.hs2o_select_f32.argtypes = [P, I64, I32, I32, P]
        L.hs2o_select_f32.restype = I64
        L.hs2o_select_rows_f64.argtypes = [P, P, I64, P, I64, I32, I32, P, I64, P]
        L.hs2o_select_rows_f64.restype = I32
        L.hs2o_select_rows_f32.argtypes = [P, P, I64, P, I64, I32, I32, P, I64, P]
        L.hs2o_select_rows_f32.restype = I32
        L.hs2o_sparse_attn.argtypes = [P, P, D, P, I64, P, I64, P, P]
        L.hs2o_sparse_attn.restype = I32
        L.hs2o_num_threads.restype = I32
        L.hs2o_e4m3_rne.argtypes = [ctypes.c_float]
        L.hs2o_e4m3_rne.restype = ctypes.c_uint8
        L.hs2o_quantize_row.argtypes = [P, I32, P, P]
        L.hs2o_kv_bridge.argtypes = [P, P, I64, I32, P]
        L.hs2o_select_blocks_f64.argtypes = [P, I64, I32, I32, I32, P]
        L.hs2o_select_blocks_f64.restype = I64
        L.hs2o_select_blocks_f32.argtypes = [P, I64, I32, I32, I32, P]
        L.hs2o_select_blocks_f32.restype = I64
        L.hs2o_block_score_f32.argtypes = [P, I64, I64, I32]
        L.hs2o_block_score_f32.restype = ctypes.c_float
        L.hs2o_select_blocks_rows.argtypes = [P, P, I64, P, I64, I32, I32, I32, I32, P, I64, P]
        L.hs2o_select_blocks_rows.restype = I32
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().hs2o_num_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data


class _View:
    """Keeps the arrays referenced by a ctypes KV descriptor alive."""

    def __init__(self, w):
        self.arrays = dict(
            k=np.ascontiguousarray(w.k), v=np.ascontiguousarray(w.v),
            ks=None if w.k_scale is None else np.ascontiguousarray(w.k_scale, dtype=np.float32),
            vs=None if w.v_scale is None else np.ascontiguousarray(w.v_scale, dtype=np.float32),
            start=np.ascontiguousarray(w.kv_start, dtype=np.int64),
            len=np.ascontiguousarray(w.kv_len, dtype=np.int32))
        a = self.arrays
        self.kv = _KV(w.batch, w.n_q, w.n_heads, w.head_dim, 1 if w.kv_dtype == "fp8" else 0,
                      _ptr(a["k"]), _ptr(a["v"]), _ptr(a["ks"]), _ptr(a["vs"]),
                      _ptr(a["start"]), _ptr(a["len"]))
        self.w = w

    @property
    def ref(self):
        return ctypes.byref(self.kv)


def e4m3_table() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    lib().hs2o_e4m3_table(out.ctypes.data)
    return out


def default_scale(head_dim: int) -> float:
    """Softmax scale c = 1/sqrt(d) (the pages give none; the plain transformer default)."""
    return 1.0 / math.sqrt(head_dim)


def positions(w, rows) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.int64)
    b, i = rows // w.n_q, rows % w.n_q
    return w.kv_len[b].astype(np.int64) - w.n_q + i


def full_attn(w, q=None, rows=None, scale=None, want_scores=True):
    """Full-attention layer on listed flat rows: returns (O [n,H,d], lse [n,H], s [n,Tmax])."""
    q = w.q_full if q is None else q
    rows = np.arange(w.n_rows, dtype=np.int64) if rows is None else \
        np.ascontiguousarray(rows, dtype=np.int64)
    scale = default_scale(w.head_dim) if scale is None else scale
    n = rows.size
    out = np.empty((n, w.n_heads, w.head_dim), dtype=np.float64)
    lse = np.empty((n, w.n_heads), dtype=np.float64)
    scores = None
    stride = 0
    if want_scores:
        stride = int(positions(w, rows).max()) + 1 if n else 1
        scores = np.full((n, stride), np.nan, dtype=np.float64)
    view = _View(w)
    qq = np.ascontiguousarray(q, dtype=np.uint16)
    rc = lib().hs2o_full_attn(view.ref, qq.ctypes.data, scale, rows.ctypes.data, n,
                              out.ctypes.data, lse.ctypes.data, _ptr(scores), stride)
    if rc != 0:
        raise RuntimeError("oracle full_attn failed")
    return out, lse, scores


def select_f64(s: np.ndarray, p: int, topk: int, window: int) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float64)
    out = np.empty(max(p + 1, 1), dtype=np.int32)
    c = lib().hs2o_select_f64(s.ctypes.data, p, topk, window, out.ctypes.data)
    return out[:c]


def select_f32(s: np.ndarray, p: int, topk: int, window: int) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float32)
    out = np.empty(max(p + 1, 1), dtype=np.int32)
    c = lib().hs2o_select_f32(s.ctypes.data, p, topk, window, out.ctypes.data)
    return out[:c]


def select_rows(w, rows, scores, topk=None, window=None, fp32=False):
    """Selection for listed rows from a [n, stride] score array; returns (idx [n, cap], count)."""
    topk = w.topk if topk is None else topk
    window = w.window if window is None else window
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.size
    cap = max(int(positions(w, rows).max()) + 1 if n else 1, 1)
    cap = min(cap, topk + window) if cap > topk + window else cap
    out = np.full((n, cap), -1, dtype=np.int32)
    count = np.zeros(n, dtype=np.int32)
    view = _View(w)
    if fp32:
        s = np.ascontiguousarray(scores, dtype=np.float32)
        rc = lib().hs2o_select_rows_f32(view.ref, rows.ctypes.data, n, s.ctypes.data,
                                        s.shape[1], topk, window, out.ctypes.data, cap,
                                        count.ctypes.data)
    else:
        s = np.ascontiguousarray(scores, dtype=np.float64)
        rc = lib().hs2o_select_rows_f64(view.ref, rows.ctypes.data, n, s.ctypes.data,
                                        s.shape[1], topk, window, out.ctypes.data, cap,
                                        count.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle select failed")
    return out, count


def select_blocks_f64(s: np.ndarray, p: int, block: int, topk: int, window: int) -> np.ndarray:
    """Block-level selection (blocks of `block` candidate positions, block score = sum)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    out = np.empty(max(p + 1, 1), dtype=np.int32)
    c = lib().hs2o_select_blocks_f64(s.ctypes.data, p, block, topk, window, out.ctypes.data)
    if c < 0:
        raise ValueError("block size must be a power of two dividing topk")
    return out[:c]


def select_blocks_f32(s: np.ndarray, p: int, block: int, topk: int, window: int) -> np.ndarray:
    """Block-level selection on float32 scores (fold-in-half float32 block sums)."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    out = np.empty(max(p + 1, 1), dtype=np.int32)
    c = lib().hs2o_select_blocks_f32(s.ctypes.data, p, block, topk, window, out.ctypes.data)
    if c < 0:
        raise ValueError("block size must be a power of two dividing topk (at most 4096)")
    return out[:c]


def block_score_f32(s: np.ndarray, t0: int, nc: int, block: int) -> float:
    """float32 score of the block starting at t0 (positions >= nc count as 0)."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    return float(lib().hs2o_block_score_f32(s.ctypes.data, t0, nc, block))


def select_blocks_rows(w, rows, scores, block, topk=None, window=None, fp32=False):
    """Block-level selection for listed rows; returns (idx [n, cap], count) like select_rows."""
    topk = w.topk if topk is None else topk
    window = w.window if window is None else window
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.size
    cap = max(int(positions(w, rows).max()) + 1 if n else 1, 1)
    cap = min(cap, topk + window)
    out = np.full((n, cap), -1, dtype=np.int32)
    count = np.zeros(n, dtype=np.int32)
    view = _View(w)
    s = np.ascontiguousarray(scores, dtype=np.float32 if fp32 else np.float64)
    rc = lib().hs2o_select_blocks_rows(view.ref, rows.ctypes.data, n, s.ctypes.data, s.shape[1],
                                       1 if fp32 else 0, block, topk, window, out.ctypes.data,
                                       cap, count.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle block select failed")
    return out, count


def sparse_attn(w, q, rows, idx, count, scale=None):
    """Sparse layer: attention of q's rows over only their selected positions."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    scale = default_scale(w.head_dim) if scale is None else scale
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    count = np.ascontiguousarray(count, dtype=np.int32)
    n = rows.size
    out = np.empty((n, w.n_heads, w.head_dim), dtype=np.float64)
    view = _View(w)
    qq = np.ascontiguousarray(q, dtype=np.uint16)
    rc = lib().hs2o_sparse_attn(view.ref, qq.ctypes.data, scale, rows.ctypes.data, n,
                                idx.ctypes.data, idx.shape[1], count.ctypes.data,
                                out.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle sparse_attn failed")
    return out


def block(w, rows=None, scale=None):
    """The whole hybrid block on listed rows: full layer, selection, and every sparse layer."""
    rows = np.arange(w.n_rows, dtype=np.int64) if rows is None else \
        np.ascontiguousarray(rows, dtype=np.int64)
    o_full, lse, s = full_attn(w, rows=rows, scale=scale)
    idx, count = select_rows(w, rows, s)
    o_sparse = [sparse_attn(w, w.q_sparse[l], rows, idx, count, scale)
                for l in range(w.n_sparse)]
    return dict(rows=rows, o_full=o_full, lse=lse, scores=s, idx=idx, count=count,
                o_sparse=o_sparse)


def kv_bridge(hidden_bits: np.ndarray, w_bits: np.ndarray):
    """KV Bridging projections: hidden bf16 bits [m, d], w bf16 bits [256, d] (K rows 0..127,
    V rows 128..255) -> (K [m, 128], V [m, 128]) in float64."""
    h = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    m, d = h.shape
    if w.shape != (256, d):
        raise ValueError("w must be [256, d]")
    out = np.empty((m, 256), dtype=np.float64)
    lib().hs2o_kv_bridge(h.ctypes.data, w.ctypes.data, m, d, out.ctypes.data)
    return out[:, :128], out[:, 128:]


def e4m3_rne(y: float) -> int:
    """OCP e4m3fn code nearest to the float32 value y (ties to even, saturating at 448)."""
    return int(lib().hs2o_e4m3_rne(float(y)))


def quantize_rows(x_bf16_bits: np.ndarray):
    """FP8 cache rows for appended tokens: x as bf16 bits [rows, d] -> (codes uint8 [rows, d],
    scale float32 [rows]); scale = max|x| / 448 (1 for a zero row), codes = e4m3 RNE of the float32 quotient x / scale."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    rows, d = x.shape
    codes = np.zeros((rows, d), dtype=np.uint8)
    scale = np.zeros(rows, dtype=np.float32)
    for r in range(rows):
        lib().hs2o_quantize_row(x[r].ctypes.data, d, codes[r].ctypes.data, scale[r:].ctypes.data)
    return codes, scale
