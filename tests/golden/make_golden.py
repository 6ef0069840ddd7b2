"""Writes tests/golden/tiny_block.json from the fp64 oracle alone.

The pages print no worked example of the hybrid block, so this fixture is a regression pin: it
freezes the oracle's output on two tiny seeded workloads (bf16 and FP8-e4m3 caches). The
independent pins (SDPA, lexsort, closed forms, invariants) live in tests/test_oracle_pins.py;
this file only guards the oracle against unintended change. Run from the repo root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

CASES = {
    "bf16": dict(name="tiny_bf16", batch=2, n_q=2, n_heads=2, n_sparse=1, kv_dtype="bf16",
                 lengths=(40, 70), needles=2, topk=8, window=4),
    "fp8": dict(name="tiny_fp8", batch=1, n_q=3, n_heads=2, n_sparse=1, kv_dtype="fp8",
                lengths=(60,), needles=2, topk=8, window=4),
}
SEED = 20260922


def compute(case):
    w = workloads.make_workload(CASES[case], seed=SEED)
    out = oracle.block(w)
    return dict(config=CASES[case], seed=SEED,
                lse=out["lse"].tolist(),
                o_full_row0_head0=out["o_full"][0, 0].tolist(),
                scores=[row[:w.position(*divmod(r, w.n_q)) + 1].tolist()
                        for r, row in enumerate(out["scores"])],
                idx=[out["idx"][r, :out["count"][r]].tolist() for r in range(w.n_rows)],
                o_sparse_row_last=out["o_sparse"][0][-1].tolist())


if __name__ == "__main__":
    data = {case: compute(case) for case in CASES}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_block.json"),
              "w") as f:
        json.dump(data, f, indent=1)
