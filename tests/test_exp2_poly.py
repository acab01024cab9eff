"""The FMA-pipe exp2 used for part of the softmax: the fitted cubic meets its
stated error bound (CPU, float32 Horner as the kernel evaluates it) and the
device version matches 2^x within that bound (GPU)."""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUH = os.path.join(ROOT, "streaming_frame_causal_b200", "csrc", "exp2_poly.cuh")


def _coeffs():
    text = open(CUH).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f", text).group(1))) for i in range(4)]


def test_cubic_relative_error_bound():
    c0, c1, c2, c3 = _coeffs()
    f = np.linspace(0, 1, 1 << 20, endpoint=False).astype(np.float32)
    p = ((c3 * f + c2) * f + c1) * f + c0
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
    assert rel.max() < 8e-5
    # far below the 2^-9 relative rounding of the bf16 probabilities it feeds
    assert rel.max() < 2.0 ** -9 / 20


@pytest.mark.gpu
def test_device_poly_matches_exp2():
    import torch
    import streaming_frame_causal_b200 as swa
    x = torch.cat([torch.linspace(-125, 8, 1_000_001), torch.tensor([-126.0, -200.0, -float("inf"), 0.0, 7.5])])
    xd = x.cuda()
    y = torch.empty_like(xd)
    swa.swa_debug_exp2_poly(xd, y)
    torch.cuda.synchronize()
    got = y.cpu().double().numpy()
    ref = np.exp2(x.double().numpy())
    ok = x.numpy() >= -125
    rel = np.abs(got[ok] / ref[ok] - 1)
    assert rel.max() < 8e-5, rel.max()
    # at and below -126 the result may be denormal or clamped: tiny, never NaN
    assert np.all(np.isfinite(got)) and np.all(got[~ok] <= 2.0 ** -125)
