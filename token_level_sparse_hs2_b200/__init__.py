"""token_level_sparse_hs2_b200 -- HySparse2 KV-Reuse token-sparse attention on NVIDIA B200.

A thin ctypes binding over ``libhs2.so`` (C ABI in ``include/hs2.h``). The functions here only
marshal arguments: every step of the hybrid block runs in the library's CUDA kernels. PyTorch
provides device memory and streams. There is no CPU fallback: if the library is missing the
first call raises.

The hybrid block ("HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs",
section "KV Reuse and Token-Level Sparse Selection"):
  1. ``full_attn_scores``   -- full-attention MQA layer over the shared K/V cache, plus the
                               per-position importance score s[t] = sum_h softmax_h[t];
  2. ``topk_select``        -- top-1,024 tokens outside the 128-token forced window, plus the
                               window, ascending;
  3. ``sparse_gather_attn`` -- a sparse layer: its own queries over the selected rows only;
  ``block_decode`` chains 1, 2 and n_sparse x 3 on one stream.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

__all__ = ["HS2Error", "KvCache", "lib", "workspace_size", "WS_SCORES", "WS_SELECTION", "full_attn_scores", "topk_select",
           "sparse_gather_attn", "block_decode", "read_device_status", "default_scale",
           "KV_BF16", "KV_FP8_E4M3", "OUT_BF16", "OUT_F32", "TOPK", "WINDOW"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs2.so")

KV_BF16, KV_FP8_E4M3 = 0, 1
OUT_BF16, OUT_F32 = 0, 1
TOPK, WINDOW = 1024, 128
HEAD_DIM = 128
_STATUS = {0: "HS2_OK", 1: "HS2_ERR_INVALID_ARG", 2: "HS2_ERR_UNSUPPORTED",
           3: "HS2_ERR_WORKSPACE", 4: "HS2_ERR_CUDA", 5: "HS2_ERR_DEVICE_CHECK",
           6: "HS2_ERR_TIMEOUT"}


class HS2Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


class _KvView(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("kv_rows", ctypes.c_int64),
                ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("kv_start", ctypes.POINTER(ctypes.c_int64)),
                ("kv_len", ctypes.POINTER(ctypes.c_int32))]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libhs2.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m token_level_sparse_hs2_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, F, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                              ctypes.c_size_t)
        V = ctypes.POINTER(_KvView)
        L.hs2_workspace_size.argtypes = [V, I32, I32, ctypes.c_uint32, ctypes.POINTER(SZ)]
        L.hs2_full_attn_scores.argtypes = [V, P, F, P, I32, P, P, I64, P, SZ, P]
        L.hs2_topk_select.argtypes = [V, P, I64, I32, I32, P, I32, P, P, SZ, P]
        L.hs2_sparse_gather_attn.argtypes = [V, P, P, I32, P, F, P, I32, P, SZ, P]
        L.hs2_block_decode.argtypes = [V, P, P, I32, I32, I32, F, P, P, I32, P, P, I64, P, I32,
                                       P, P, SZ, P]
        L.hs2_block_decode_traced.argtypes = [V, P, P, I32, I32, I32, F, P, P, I32, P, P, I64, P,
                                              I32, P, P, SZ, P, I32, P]
        L.hs2_topk_select_noalloc.argtypes = [V, P, I64, I32, I32, P, I32, P, P]
        L.hs2_noalloc_read_status.argtypes = [P]
        L.hs2_noalloc_read_status.restype = ctypes.c_int
        L.hs2_topk_select_blocks_workspace_size.argtypes = [V, I32, I32, I32, ctypes.POINTER(SZ)]
        L.hs2_topk_select_blocks.argtypes = [V, P, I64, I32, I32, I32, P, I32, P, P, SZ, P]
        L.hs2_read_device_status.argtypes = [P, P]
        L.hs2_last_error.restype = ctypes.c_char_p
        L.hs2_status_string.restype = ctypes.c_char_p
        L.hs2_status_string.argtypes = [ctypes.c_int]
        L.hs2_version.restype = I32
        L.hs2_launch_count.restype = ctypes.c_uint64
        L.hs2_selftest_wait_timeout.argtypes = [ctypes.c_uint32, P, SZ, P]
        L.hs2_selftest_exp2.argtypes = [P, P, I64, P]
        L.hs2_selftest_exp2.restype = ctypes.c_int
        L.hs2_kv_append.argtypes = [V, P, P, P]
        L.hs2_kv_bridge.argtypes = [V, P, I32, P, P, SZ, P]
        L.hs2_kv_bridge.restype = ctypes.c_int
        L.hs2_full_attn.argtypes = [V, P, F, P, I32, P, P, SZ, P]
        L.hs2_score_pass.argtypes = [V, P, F, P, P, I64, P, SZ, P]
        L.hs2_sparse_gather_attn_partial.argtypes = [V, P, P, I32, P, F, P, P, P, SZ, P]
        L.hs2_lse_merge.argtypes = [I32, I64, I32, P, P, P, I32, P, P]
        L.hs2_cp_pack_candidates.argtypes = [V, P, P, P, I64, P, I32, P, I32, I32, P, P]
        L.hs2_cp_merge_select.argtypes = [I32, I32, P, P, I32, I32, P, I32, P, P]
        L.hs2_cp_localize.argtypes = [I32, P, P, P, I32, P, P, I32, P, P]
        for name in ("hs2_full_attn", "hs2_score_pass", "hs2_sparse_gather_attn_partial",
                     "hs2_lse_merge", "hs2_cp_pack_candidates", "hs2_cp_merge_select",
                     "hs2_cp_localize"):
            getattr(L, name).restype = ctypes.c_int
        L.hs2_kv_append.restype = ctypes.c_int
        L.hs2_selftest_wait_timeout.restype = ctypes.c_int
        for name in ("hs2_workspace_size", "hs2_full_attn_scores", "hs2_topk_select",
                     "hs2_sparse_gather_attn", "hs2_block_decode", "hs2_block_decode_traced",
                     "hs2_topk_select_noalloc", "hs2_read_device_status",
                     "hs2_topk_select_blocks_workspace_size", "hs2_topk_select_blocks"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise HS2Error(status, lib().hs2_last_error().decode())


def default_scale(head_dim: int = HEAD_DIM) -> float:
    return 1.0 / math.sqrt(head_dim)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class KvCache:
    """The shared single-head K/V cache of one full-attention layer (device tensors) plus the
    host-side sequence geometry. Sequence b owns rows [kv_start[b], kv_start[b] + kv_len[b]);
    its n_q queries are its last n_q tokens."""

    def __init__(self, k: torch.Tensor, v: torch.Tensor, kv_start, kv_len, n_q: int,
                 n_heads: int, k_scale: Optional[torch.Tensor] = None,
                 v_scale: Optional[torch.Tensor] = None):
        if k.dtype == torch.bfloat16:
            self.kv_dtype = KV_BF16
        elif k.dtype in (torch.uint8, torch.float8_e4m3fn):
            self.kv_dtype = KV_FP8_E4M3
        else:
            raise TypeError(f"unsupported cache dtype {k.dtype}")
        if not (k.is_contiguous() and v.is_contiguous()) or k.shape != v.shape or k.dim() != 2:
            raise ValueError("k and v must be contiguous [rows, 128] tensors of one shape")
        self.k, self.v, self.k_scale, self.v_scale = k, v, k_scale, v_scale
        self.kv_start = (ctypes.c_int64 * len(kv_start))(*[int(x) for x in kv_start])
        self.kv_len = (ctypes.c_int32 * len(kv_len))(*[int(x) for x in kv_len])
        self.batch, self.n_q, self.n_heads = len(kv_len), int(n_q), int(n_heads)
        self.view = _KvView(self.batch, self.n_q, self.n_heads, int(k.shape[1]), self.kv_dtype,
                            0, int(k.shape[0]), k.data_ptr(), v.data_ptr(),
                            None if k_scale is None else k_scale.data_ptr(),
                            None if v_scale is None else v_scale.data_ptr(),
                            self.kv_start, self.kv_len)

    @property
    def n_rows(self) -> int:
        return self.batch * self.n_q

    @property
    def max_len(self) -> int:
        return max(self.kv_len)

    def ref(self):
        return ctypes.byref(self.view)


WS_SCORES, WS_SELECTION = 1, 2


def workspace_size(cache: KvCache, topk: int = TOPK, window: int = WINDOW, flags: int = 0) -> int:
    """Workspace bytes; flags WS_SCORES / WS_SELECTION reserve room for the block outputs that
    block_decode is given as None."""
    n = ctypes.c_size_t(0)
    _check(lib().hs2_workspace_size(cache.ref(), topk, window, flags, ctypes.byref(n)))
    return int(n.value)


def _stride0(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.stride(0)


def _out_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return OUT_BF16
    if t.dtype == torch.float32:
        return OUT_F32
    raise TypeError(f"output dtype {t.dtype}")


def full_attn_scores(cache: KvCache, q, out, lse, scores, workspace, scale=None, stream=None):
    scale = default_scale() if scale is None else scale
    _check(lib().hs2_full_attn_scores(cache.ref(), _ptr(q), scale, _ptr(out), _out_dtype(out),
                                      _ptr(lse), _ptr(scores), scores.stride(0), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream)))


def topk_select(cache: KvCache, scores, idx, count, workspace, topk=TOPK, window=WINDOW,
                stream=None):
    _check(lib().hs2_topk_select(cache.ref(), _ptr(scores), scores.stride(0), topk, window,
                                 _ptr(idx), idx.stride(0), _ptr(count), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))


def topk_select_noalloc(cache: KvCache, scores, idx, count, topk=TOPK, window=WINDOW,
                        stream=None):
    """topk_select for callers that cannot allocate: uses the library's built-in 4 MiB device
    scratch instead of a workspace (see hs2_topk_select_noalloc in include/hs2.h)."""
    _check(lib().hs2_topk_select_noalloc(cache.ref(), _ptr(scores), scores.stride(0), topk,
                                         window, _ptr(idx), idx.stride(0), _ptr(count),
                                         _stream(stream)))


def noalloc_read_status(stream=None):
    """Synchronises and raises HS2Error if the last topk_select_noalloc recorded a problem in
    the built-in scratch (hs2_noalloc_read_status; the word is cleared by the read)."""
    _check(lib().hs2_noalloc_read_status(_stream(stream)))


def topk_select_blocks_workspace_size(cache: KvCache, block_size: int = 64, topk: int = TOPK,
                                      window: int = WINDOW) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().hs2_topk_select_blocks_workspace_size(cache.ref(), block_size, topk, window,
                                                       ctypes.byref(n)))
    return int(n.value)


def topk_select_blocks(cache: KvCache, scores, idx, count, workspace, block_size: int = 64,
                       topk=TOPK, window=WINDOW, stream=None):
    """Block-level selection (topk / block_size whole blocks plus the window); same outputs as
    topk_select (see hs2_topk_select_blocks in include/hs2.h)."""
    _check(lib().hs2_topk_select_blocks(cache.ref(), _ptr(scores), scores.stride(0), block_size,
                                        topk, window, _ptr(idx), idx.stride(0), _ptr(count),
                                        _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)))


def sparse_gather_attn(cache: KvCache, q, idx, count, out, workspace, scale=None, stream=None):
    scale = default_scale() if scale is None else scale
    _check(lib().hs2_sparse_gather_attn(cache.ref(), _ptr(q), _ptr(idx), idx.stride(0),
                                        _ptr(count), scale, _ptr(out), _out_dtype(out),
                                        _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)))


def block_decode(cache: KvCache, q_full, q_sparse: Sequence[torch.Tensor], out_full,
                 out_sparse: Sequence[torch.Tensor], lse, scores, idx, count, workspace,
                 topk=TOPK, window=WINDOW, scale=None, stream=None):
    """The hybrid block (hs2_block_decode). lse, scores and idx + count may be None: the library
    keeps them in the workspace, sized by workspace_size(..., flags=WS_SCORES | WS_SELECTION)."""
    scale = default_scale() if scale is None else scale
    L = len(q_sparse)
    if len(out_sparse) != L:
        raise ValueError("one output per sparse layer")
    qs = (ctypes.c_void_p * max(L, 1))(*[t.data_ptr() for t in q_sparse])
    os_ = (ctypes.c_void_p * max(L, 1))(*[t.data_ptr() for t in out_sparse])
    _check(lib().hs2_block_decode(cache.ref(), _ptr(q_full), qs, L, topk, window, scale,
                                  _ptr(out_full), os_, _out_dtype(out_full), _ptr(lse),
                                  _ptr(scores), _stride0(scores), _ptr(idx), _stride0(idx),
                                  _ptr(count), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  _stream(stream)))


def block_decode_traced(cache: KvCache, q_full, q_sparse: Sequence[torch.Tensor], out_full,
                        out_sparse: Sequence[torch.Tensor], lse, scores, idx, count, workspace,
                        events: Sequence[torch.cuda.Event], topk=TOPK, window=WINDOW,
                        scale=None, stream=None):
    """block_decode that also records `events` (6 + n_sparse torch.cuda.Event) around each
    step on the launch stream: before the clear, then after the clear, the pass 1 kernel, the
    pass 1 merge, pass 2, the selection and each sparse layer."""
    scale = default_scale() if scale is None else scale
    L = len(q_sparse)
    qs = (ctypes.c_void_p * max(L, 1))(*[t.data_ptr() for t in q_sparse])
    os_ = (ctypes.c_void_p * max(L, 1))(*[t.data_ptr() for t in out_sparse])
    ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib().hs2_block_decode_traced(cache.ref(), _ptr(q_full), qs, L, topk, window, scale,
                                         _ptr(out_full), os_, _out_dtype(out_full), _ptr(lse),
                                         _ptr(scores), _stride0(scores), _ptr(idx),
                                         _stride0(idx), _ptr(count), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), ev,
                                         len(events), _stream(stream)))


def read_device_status(workspace, stream=None):
    """Synchronises and raises HS2Error if a kernel of the last call recorded a problem."""
    _check(lib().hs2_read_device_status(_ptr(workspace), _stream(stream)))


def launch_count() -> int:
    """Kernels the library has launched in this process so far (hs2_launch_count)."""
    return int(lib().hs2_launch_count())


def selftest_wait_timeout(workspace, limit_us: int = 20000, stream=None):
    """Runs hs2_selftest_wait_timeout: a kernel whose bounded wait must run out; returns the
    status hs2_read_device_status then reports (an int, HS2_ERR_TIMEOUT = 6 expected)."""
    _check(lib().hs2_selftest_wait_timeout(limit_us, _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(stream)))
    return int(lib().hs2_read_device_status(_ptr(workspace), _stream(stream)))


def selftest_exp2(x: torch.Tensor, y: torch.Tensor, stream=None):
    """y = the FMA-pipe 2^x of the tensor-core score passes (hs2_selftest_exp2); fp32 tensors."""
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel():
        raise ValueError("x and y must be float32 tensors of one size")
    _check(lib().hs2_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream)))


def selftest_wait_timeout_noalloc(limit_us: int = 20000, stream=None) -> int:
    """hs2_selftest_wait_timeout on the no-allocation selection's built-in status word; returns
    the status hs2_noalloc_read_status then reports (HS2_ERR_TIMEOUT = 6 expected)."""
    _check(lib().hs2_selftest_wait_timeout(limit_us, None, 0, _stream(stream)))
    return int(lib().hs2_noalloc_read_status(_stream(stream)))


def kv_append(cache: KvCache, new_k, new_v, stream=None):
    """Writes the n_q new tokens of every sequence (bf16 [batch, n_q, 128] each) into the last
    n_q rows of each sequence of the cache (e4m3 caches: quantised with per-row scales)."""
    _check(lib().hs2_kv_append(cache.ref(), _ptr(new_k), _ptr(new_v), _stream(stream)))


def kv_bridge(cache: KvCache, hidden, w_kv, workspace, stream=None):
    """KV Bridging: cache rows of each sequence's last n_q tokens = hidden . [W_K; W_V]^T
    (hidden bf16 [batch, n_q, d_model], w_kv bf16 [256, d_model]); see hs2_kv_bridge."""
    if hidden.dtype != torch.bfloat16 or w_kv.dtype != torch.bfloat16:
        raise TypeError("hidden and w_kv must be bfloat16")
    if not (hidden.is_contiguous() and w_kv.is_contiguous()):
        raise ValueError("hidden and w_kv must be contiguous")
    d_model = int(hidden.shape[-1])
    if hidden.numel() != cache.n_rows * d_model or tuple(w_kv.shape) != (256, d_model):
        raise ValueError("hidden must be [batch, n_q, d_model] and w_kv [256, d_model]")
    _check(lib().hs2_kv_bridge(cache.ref(), _ptr(hidden), d_model, _ptr(w_kv), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)))


# ---------------------------------------------------------------- context-parallel pieces

def _host_i64(xs):
    return (ctypes.c_int64 * len(xs))(*[int(x) for x in xs])


def _host_i32(xs):
    return (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])


def full_attn(cache: KvCache, q, out, lse, workspace, scale=None, stream=None):
    """Full-attention output and lse only (decode), see hs2_full_attn."""
    scale = default_scale() if scale is None else scale
    _check(lib().hs2_full_attn(cache.ref(), _ptr(q), scale, _ptr(out), _out_dtype(out), _ptr(lse),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream)))


def score_pass(cache: KvCache, q, lse, scores, workspace, scale=None, stream=None):
    """Importance scores with a given lse (decode), see hs2_score_pass."""
    scale = default_scale() if scale is None else scale
    _check(lib().hs2_score_pass(cache.ref(), _ptr(q), scale, _ptr(lse), _ptr(scores),
                                scores.stride(0), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)))


def sparse_gather_attn_partial(cache: KvCache, q, idx, count, out, lse, workspace, scale=None,
                               stream=None):
    """A sparse layer's fp32 output and lse over the given (possibly empty) selection."""
    scale = default_scale() if scale is None else scale
    _check(lib().hs2_sparse_gather_attn_partial(cache.ref(), _ptr(q), _ptr(idx), idx.stride(0),
                                                _ptr(count), scale, _ptr(out), _ptr(lse),
                                                _ptr(workspace),
                                                workspace.numel() * workspace.element_size(),
                                                _stream(stream)))


def lse_merge(part_out, part_lse, out, lse=None, stream=None):
    """Log-sum-exp merge of [n_parts, rows, H, 128] outputs with [n_parts, rows, H] lse."""
    if not (part_out.is_contiguous() and part_lse.is_contiguous() and out.is_contiguous()):
        raise ValueError("lse_merge needs contiguous tensors")
    n_parts, rows, heads = part_lse.shape[0], part_lse.shape[1], part_lse.shape[2]
    _check(lib().hs2_lse_merge(n_parts, rows, heads, _ptr(part_out), _ptr(part_lse), _ptr(out),
                               _out_dtype(out), _ptr(lse), _stream(stream)))


def cp_pack_candidates(cache: KvCache, global_offset, global_len, scores, idx, count, keys,
                       topk=TOPK, window=WINDOW, stream=None):
    _check(lib().hs2_cp_pack_candidates(cache.ref(), _host_i64(global_offset),
                                        _host_i32(global_len), _ptr(scores), scores.stride(0),
                                        _ptr(idx), idx.stride(0), _ptr(count), topk, window,
                                        _ptr(keys), _stream(stream)))


def cp_merge_select(keys, global_len, idx, count, topk=TOPK, window=WINDOW, stream=None):
    """keys: int64 [n_parts, batch, topk] (the u64 keys of every shard)."""
    n_parts, batch = keys.shape[0], keys.shape[1]
    _check(lib().hs2_cp_merge_select(n_parts, batch, _host_i32(global_len), _ptr(keys), topk,
                                     window, _ptr(idx), idx.stride(0), _ptr(count),
                                     _stream(stream)))


def cp_localize(global_offset, local_len, idx, count, idx_local, count_local, stream=None):
    _check(lib().hs2_cp_localize(len(local_len), _host_i64(global_offset), _host_i32(local_len),
                                 _ptr(idx), idx.stride(0), _ptr(count), _ptr(idx_local),
                                 idx_local.stride(0), _ptr(count_local), _stream(stream)))
