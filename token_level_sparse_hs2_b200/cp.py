"""Context-parallel decode of one long sequence: its cache is split by token range over the
ranks of a process group, every rank runs the hybrid block's kernels on its own shard, and three
small all-gathers per block join the shards (the LSE-merge of the full layer, the shards' top-k
candidates, the LSE-merge of each sparse layer).

Why a split by position composes exactly ("HySparse2: How Xiaomi Split the Transformer to Fix
Agent Prefill Costs", section "KV Reuse and Token-Level Sparse Selection", for what each layer
computes; "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing", bullet "Inference
cost", for the 1M-token contexts this is for): attention over disjoint position sets merges by
log-sum-exp; the score of a position needs only the merged lse; the top-k of the whole context
lies in the union of the shards' own top-k. The kernels are the library's (see hs2.h, section
"Context-parallel decode"); the collectives are torch.distributed all-gathers (NCCL on GPUs).

Shapes: one sequence (batch 1), one decode query (n_q 1). Rank r holds global positions
[offset, offset + T_local) as a KvCache of T_local rows; T_global is the whole context.
The shards follow the ranks' order: rank r's positions all precede rank r + 1's (the merged
selection is laid out shard by shard, so rank order is position order).
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch

HEAD_DIM = 128


def local_window(offset: int, local_len: int, global_len: int, window: int) -> int:
    """How many of the shard's positions fall in the global forced window [T - window, T)."""
    first_window = global_len - window
    local_candidates = min(max(first_window - offset, 0), local_len)
    return local_len - local_candidates


def nccl_all_gather(group=None) -> Callable[[torch.Tensor], torch.Tensor]:
    """all_gather(x) -> [world, *x.shape] over `group` (torch.distributed, e.g. NCCL)."""
    import torch.distributed as dist

    def gather(x: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        out = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(out, x.contiguous(), group=group)
        return out
    return gather


def _split(parts: torch.Tensor, H: int):
    """[world, H * 128 + H] gathered buffers -> contiguous ([world, 1, H, 128], [world, 1, H])."""
    world = parts.shape[0]
    return (parts[:, :H * HEAD_DIM].contiguous().view(world, 1, H, HEAD_DIM),
            parts[:, H * HEAD_DIM:].contiguous().view(world, 1, H))


def _default_ops():
    import token_level_sparse_hs2_b200 as ops
    return ops


def cp_block_decode(cache_local, offset: int, global_len: int, q_full, q_sparse: Sequence,
                    out_full, out_sparse: Sequence, workspace, all_gather: Callable,
                    topk: int = 1024, window: int = 128, scale: Optional[float] = None, ops=None):
    """One hybrid-block decode step of this rank's shard; every rank calls it with its own
    shard and the same queries, in the same order. Writes out_full ([1, 1, H, 128]) and each
    out_sparse[l]; returns dict(lse [1, H], idx [1, cap] global selection, count [1],
    scores [1, T_local] this shard's scores)."""
    ops = _default_ops() if ops is None else ops
    if cache_local.batch != 1 or cache_local.n_q != 1:
        raise ValueError("context-parallel decode takes one sequence and one query")
    H = cache_local.n_heads
    T_local = int(cache_local.kv_len[0])
    dev = q_full.device
    f32 = dict(dtype=torch.float32, device=dev)
    i32 = dict(dtype=torch.int32, device=dev)

    # 1. full layer: local (O, lse), all-gather, log-sum-exp merge
    part = torch.empty(H * HEAD_DIM + H, **f32)
    o_r = part[:H * HEAD_DIM].view(1, H, HEAD_DIM)
    lse_r = part[H * HEAD_DIM:].view(1, H)
    ops.full_attn(cache_local, q_full, o_r, lse_r, workspace, scale=scale)
    parts = all_gather(part)
    lse = torch.empty((1, H), **f32)
    ops.lse_merge(*_split(parts, H), out_full, lse)

    # 2. the shard's scores under the merged lse, its own top-k, all-gather, global merge
    scores = torch.empty((1, T_local), **f32)
    ops.score_pass(cache_local, q_full, lse, scores, workspace, scale=scale)
    wl = local_window(offset, T_local, global_len, window)
    idx_l = torch.empty((1, max(1, min(T_local, topk + wl))), **i32)
    cnt_l = torch.empty(1, **i32)
    ops.topk_select(cache_local, scores, idx_l, cnt_l, workspace, topk=topk, window=wl)
    keys = torch.empty((1, topk), dtype=torch.int64, device=dev)
    ops.cp_pack_candidates(cache_local, [offset], [global_len], scores, idx_l, cnt_l, keys,
                           topk=topk, window=window)
    all_keys = all_gather(keys)
    cap = min(global_len, topk + window)
    idx = torch.empty((1, cap), **i32)
    count = torch.empty(1, **i32)
    ops.cp_merge_select(all_keys, [global_len], idx, count, topk=topk, window=window)

    # 3. sparse layers: attention over the shard's part of the selection, merged the same way
    idx_loc = torch.empty((1, cap), **i32)
    cnt_loc = torch.empty(1, **i32)
    ops.cp_localize([offset], [T_local], idx, count, idx_loc, cnt_loc)
    for l, q in enumerate(q_sparse):
        ops.sparse_gather_attn_partial(cache_local, q, idx_loc, cnt_loc, o_r, lse_r, workspace,
                                       scale=scale)
        parts = all_gather(part)
        ops.lse_merge(*_split(parts, H), out_sparse[l])
    return dict(lse=lse, idx=idx, count=count, scores=scores)
