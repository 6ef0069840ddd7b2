"""Regression pin: the oracle still reproduces tests/golden/tiny_block.json."""
import json
import os

import numpy as np

from tests.golden import make_golden

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_frozen_fixture(oracle_lib):
    with open(os.path.join(HERE, "golden", "tiny_block.json")) as f:
        gold = json.load(f)
    for case, ref in gold.items():
        got = make_golden.compute(case)
        assert got["idx"] == ref["idx"], case
        for key in ("lse", "o_full_row0_head0", "o_sparse_row_last"):
            np.testing.assert_allclose(np.array(got[key]), np.array(ref[key]), rtol=1e-12,
                                       atol=1e-14, err_msg=f"{case}:{key}")
        for a, b in zip(got["scores"], ref["scores"]):
            np.testing.assert_allclose(a, b, rtol=1e-12, atol=0)
