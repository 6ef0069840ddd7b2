"""Full-row parity of the 2 x 512-query action chunk at a 256k context: every one of the 1,024
query rows of the full-size workload, through the C ABI, against the fp64 oracle (O, lse,
scores, the selection bit for bit on the GPU's scores, the sparse layers). Every query row
selects its own set ("HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs",
section "KV Reuse and Token-Level Sparse Selection"), so sampled rows do not stand for the rest.

Marked `fullparity`, not `gpu`: it takes minutes of oracle time on the host and runs on request
(`pytest -m fullparity`)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.fullparity


def test_config3_chunk_every_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from token_level_sparse_hs2_b200 import build
    build.build()
    oracle.build()
    from tests import gpu_helpers as H
    w = W.make_workload(3)
    g = H.run_block(w)
    R = w.n_rows
    assert R == 1024
    checked = 0
    for r0 in range(0, R, 128):   # 128 rows at a time keeps the fp64 score rows in bounds
        rows = np.arange(r0, min(R, r0 + 128))
        part = dict(g)
        part["rows"] = rows
        for key in ("o_full", "lse", "scores", "idx", "count"):
            part[key] = g[key][rows]
        part["o_sparse"] = [o[rows] for o in g["o_sparse"]]
        H.check_block(w, part)
        checked += len(rows)
    assert checked == R
