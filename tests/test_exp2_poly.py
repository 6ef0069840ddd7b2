"""exp2_poly2, the 2^x that the tensor-core score passes evaluate on the FMA pipe for part of
their exponentials (the special-function unit does the rest): its cubic is the Remez minimax fit
of tests/exp2_poly_fit.py, and its relative error stays within the stated 7.5e-5.

CPU: the coefficients in the kernel source equal the fit's, rounded to float32, and the fit's
levelled error (and its float32 evaluation) is below the bound. GPU: the device function, run
through hs2_selftest_exp2 on every float32 step of a dense grid of [-125, 0] plus the points
where the Cody-Waite split changes, against 2^x in float64."""
import os
import re

import numpy as np
import pytest
import torch

from tests import exp2_poly_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUND = 7.5e-5


def kernel_coefficients():
    src = open(os.path.join(ROOT, "token_level_sparse_hs2_b200", "csrc", "attn_tile.cuh")).read()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    c3, c2, c1, c0 = vals[:4]   # Horner order in the source
    return [c0, c1, c2, c3]


def test_kernel_cubic_is_the_remez_fit():
    c, E = exp2_poly_fit.fit()
    assert E < BOUND
    fit32 = [float(np.float32(v)) for v in c]
    src = [float(np.float32(v)) for v in kernel_coefficients()]
    assert src == fit32, (src, fit32)
    assert exp2_poly_fit.kernel_error(src) < BOUND


def test_remez_error_is_levelled():
    """The error curve of the fit equioscillates: five extrema of equal size and alternating
    sign, the Chebyshev alternation that characterises the minimax polynomial."""
    c, E = exp2_poly_fit.fit()
    xs = np.linspace(-0.5, 0.5, 200001)
    e = np.polyval(np.asarray(c)[::-1], xs) / np.exp2(xs) - 1.0
    assert abs(np.abs(e).max() - E) < 1e-3 * E
    runs = np.split(np.arange(xs.size), np.nonzero(np.diff(np.sign(e)) != 0)[0] + 1)
    peaks = np.array([e[r][np.argmax(np.abs(e[r]))] for r in runs])
    assert peaks.size == 5
    assert np.all(np.sign(peaks[1:]) == -np.sign(peaks[:-1]))
    assert np.allclose(np.abs(peaks), E, rtol=1e-3)


@pytest.mark.gpu
def test_device_exp2_within_bound():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import token_level_sparse_hs2_b200 as hs2
    from token_level_sparse_hs2_b200 import build
    build.build()
    grid = np.linspace(-125.0, 0.0, 4_000_001, dtype=np.float64).astype(np.float32)
    j = np.arange(-125, 1, dtype=np.float64)
    edges = np.concatenate([j, j + 0.5, j - 0.5]).astype(np.float32)
    edges = np.concatenate([edges, np.nextafter(edges, np.float32(1)), np.nextafter(edges, np.float32(-1))])
    x = np.concatenate([grid, edges[(edges >= -125.0) & (edges <= 0.0)]]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    hs2.selftest_exp2(xd, yd)
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND, (float(rel.max()), float(x[np.argmax(rel)]))
