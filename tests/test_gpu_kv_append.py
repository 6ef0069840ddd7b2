"""KV append (the step before the block): bit-exact against the oracle's quantiser.

"HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing", "Inference cost": the shared
single-head cache is FP8; every new token's K/V row is written (quantised per token) before the
full-attention layer and the window read it.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_hs2_b200 as hs2
import workloads as W
from tests.gpu_helpers import check_block, run_block

pytestmark = pytest.mark.gpu


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _new_rows(rng, B, n_q):
    x = rng.standard_normal((B, n_q, 128)).astype(np.float32)
    x *= rng.uniform(1e-3, 300.0, (B, n_q, 1)).astype(np.float32)
    x.reshape(-1, 128)[0] = 0.0                          # an all-zero row
    if B * n_q > 2:
        r = x.reshape(-1, 128)[1]
        r[:] = 0.0
        r[5] = -7.25                                      # one nonzero
        x.reshape(-1, 128)[2] *= 1e-30                    # tiny values (subnormal codes)
    return W.f32_to_bf16_bits(x)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("lengths,n_q", [([700], 1), ([300, 1000, 97], 1), ([512, 260], 9)])
def test_append_matches_oracle(kv_dtype, lengths, n_q):
    w = W.make_workload(0, lengths=lengths, batch=len(lengths), n_q=n_q, n_sparse=1, kv_dtype=kv_dtype,
                        n_heads=16)
    d = W.to_device(w, "cuda")
    cache = hs2.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, w.n_q, w.n_heads, d["k_scale"], d["v_scale"])
    rng = np.random.default_rng(11)
    nk, nv = _new_rows(rng, w.batch, n_q), _new_rows(rng, w.batch, n_q)
    k0 = d["k"].clone()
    hs2.kv_append(cache, _bf16(nk), _bf16(nv))
    torch.cuda.synchronize()
    rows = np.concatenate([w.kv_start[b] + w.kv_len[b] - n_q + np.arange(n_q) for b in range(w.batch)])
    others = np.setdiff1d(np.arange(w.k.shape[0]), rows)
    for new, dev, host_scale, dev_scale in ((nk, d["k"], w.k_scale, d["k_scale"]), (nv, d["v"], w.v_scale, d["v_scale"])):
        got = dev.cpu()
        if kv_dtype == "bf16":
            got_bits = got.view(torch.int16).numpy().view(np.uint16)
            np.testing.assert_array_equal(got_bits[rows], new.reshape(-1, 128))
        else:
            codes, scale = oracle.quantize_rows(new.reshape(-1, 128))
            np.testing.assert_array_equal(got.numpy()[rows], codes)
            np.testing.assert_array_equal(dev_scale.cpu().numpy()[rows], scale)
            np.testing.assert_array_equal(dev_scale.cpu().numpy()[others], host_scale[others])
    # rows of the cache that were not appended are untouched
    if kv_dtype == "bf16":
        assert torch.equal(d["k"].cpu()[others], k0.cpu()[others])
    else:
        assert torch.equal(d["k"].cpu()[others], k0.cpu()[others])


def test_decode_step_after_append_matches_oracle():
    # append the step's token, then run the block on the updated cache: both sides see the same bytes
    w = W.make_workload(0, lengths=[900, 1400], batch=2, n_sparse=2, kv_dtype="fp8", n_heads=16)
    rng = np.random.default_rng(12)
    nk, nv = _new_rows(rng, w.batch, 1), _new_rows(rng, w.batch, 1)
    d = W.to_device(w, "cuda")
    cache = hs2.KvCache(d["k"], d["v"], w.kv_start, w.kv_len, w.n_q, w.n_heads, d["k_scale"], d["v_scale"])
    hs2.kv_append(cache, _bf16(nk), _bf16(nv))
    torch.cuda.synchronize()
    w2 = dataclasses.replace(w, k=d["k"].cpu().numpy(), v=d["v"].cpu().numpy(),
                             k_scale=d["k_scale"].cpu().numpy(), v_scale=d["v_scale"].cpu().numpy())
    check_block(w2, run_block(w2))
