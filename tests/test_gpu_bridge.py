"""GPU parity for KV Bridging (the cross-decoder cache projected from self-decoder hidden states:
"HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section "The
Self-Decoder and Cross-Decoder Split"), through the C ABI, against the oracle.

bf16 cache rows: each element within half a bf16 ulp of the exact product plus the float32
accumulation bound d_model * 2^-24 * sum_d |h_d w_d|. e4m3 cache rows: codes and scales bit for
bit equal to the oracle's quantiser applied to the GPU's own bf16 rows (the same kernel run into
a bf16 cache), since the float32 accumulation decides those integers. Rows outside the written
ones stay untouched."""
import numpy as np
import pytest
import torch

import oracle
from workloads import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from token_level_sparse_hs2_b200 import build
    build.build()
    oracle.build()


def hs2():
    import token_level_sparse_hs2_b200 as m
    return m


def inputs(batch, n_q, d, seed):
    rng = np.random.default_rng(seed)
    h = f32_to_bf16_bits(rng.standard_normal((batch * n_q, d)).astype(np.float32))
    w = f32_to_bf16_bits((rng.standard_normal((256, d)) / np.sqrt(d)).astype(np.float32))
    return h, w


def bf16_tensor(bits, shape, dev="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16) \
        .reshape(shape).to(dev)


def run(lengths, n_q, h, w, fp8):
    m = hs2()
    d = h.shape[1]
    lengths = np.asarray(lengths)
    start = np.concatenate([[0], np.cumsum(lengths)[:-1]])
    rows = int(lengths.sum())
    dev = torch.device("cuda")
    if fp8:
        k = torch.full((rows, 128), 0x5a, dtype=torch.uint8, device=dev)
        ks = torch.full((rows,), -1.0, dtype=torch.float32, device=dev)
        vs = ks.clone()
    else:
        k = torch.full((rows, 128), 0x5a5a, dtype=torch.int16, device=dev).view(torch.bfloat16)
        ks = vs = None
    v = k.clone()
    cache = m.KvCache(k, v, start, lengths, n_q, 32, ks, vs)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    m.kv_bridge(cache, bf16_tensor(h, (len(lengths), n_q, d)), bf16_tensor(w, (256, d)), ws)
    m.read_device_status(ws)             # raises on a recorded device error
    torch.cuda.synchronize()
    out = dict(start=start, lengths=lengths)
    if fp8:
        out.update(k=k.cpu().numpy(), v=v.cpu().numpy(), ks=ks.cpu().numpy(), vs=vs.cpu().numpy())
    else:
        out.update(k=k.view(torch.int16).cpu().numpy().view(np.uint16),
                   v=v.view(torch.int16).cpu().numpy().view(np.uint16))
    return out


def written_rows(o, n_q):
    return np.concatenate([np.arange(s + L - n_q, s + L) for s, L in zip(o["start"], o["lengths"])])


def check_bf16(o, h, w, n_q, sample=None):
    d = h.shape[1]
    rows = written_rows(o, n_q)
    sel = np.arange(len(rows)) if sample is None else np.asarray(sample)
    k_ref, v_ref = oracle.kv_bridge(h[sel], w)
    ka, va = oracle.kv_bridge(h[sel] & 0x7fff, w & 0x7fff)        # sum_d |h_d w_d|
    for got_bits, ref, mag in ((o["k"][rows[sel]], k_ref, ka), (o["v"][rows[sel]], v_ref, va)):
        got = bf16_bits_to_f32(got_bits).astype(np.float64)
        err = d * 2.0 ** -24 * mag
        top = np.abs(ref) + err
        ulp = np.where(top > 0, 2.0 ** (np.floor(np.log2(np.maximum(top, 1e-300))) - 7), 0)
        bad = np.abs(got - ref) > 0.5 * ulp + err + 1e-30
        assert not bad.any(), (np.argwhere(bad)[:4], got[bad][:4], ref[bad][:4])


@pytest.mark.parametrize("d,n_q,lengths", [(512, 300, (1000, 700)), (4096, 77, (500, 77, 90)),
                                           (64, 129, (129,)), (1024, 1, (33, 4096))])
def test_bf16_rows_match_the_exact_projection(d, n_q, lengths):
    h, w = inputs(len(lengths), n_q, d, seed=d + n_q)
    o = run(lengths, n_q, h, w, fp8=False)
    check_bf16(o, h, w, n_q)
    keep = np.setdiff1d(np.arange(int(np.sum(lengths))), written_rows(o, n_q))
    assert (o["k"][keep] == 0x5a5a).all() and (o["v"][keep] == 0x5a5a).all()


@pytest.mark.parametrize("d,n_q,lengths", [(512, 300, (1000, 700)), (4096, 77, (500, 77, 90))])
def test_fp8_rows_are_the_quantised_bf16_rows(d, n_q, lengths):
    h, w = inputs(len(lengths), n_q, d, seed=7 * d + n_q)
    ob = run(lengths, n_q, h, w, fp8=False)
    of = run(lengths, n_q, h, w, fp8=True)
    rows = written_rows(ob, n_q)
    for mat, sc in (("k", "ks"), ("v", "vs")):
        codes, scale = oracle.quantize_rows(ob[mat][rows])
        assert np.array_equal(of[mat][rows], codes), mat
        assert np.array_equal(of[sc][rows].view(np.uint32), scale.view(np.uint32)), mat
    keep = np.setdiff1d(np.arange(int(np.sum(lengths))), rows)
    assert (of["k"][keep] == 0x5a).all() and (of["ks"][keep] == -1.0).all()


def test_full_size_prefill_bridge_sampled():
    """32,768 prompt tokens, d_model 4096 (the prefill workload): sampled rows, both ends and a
    spread of interior rows, against the exact projection."""
    n_q, d = 32768, 4096
    h, w = inputs(1, n_q, d, seed=5)
    o = run((n_q,), n_q, h, w, fp8=False)
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, 1, 127, 128, n_q - 1], rng.integers(0, n_q, 250)]))
    check_bf16(o, h, w, n_q, sample=sample)
