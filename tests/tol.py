"""Parity tolerances (element by element against the float64 oracle).

bf16 path: max-abs <= 2e-2 and relative RMS <= 5e-3; f32 path: max-abs <= 1e-4.
The bf16 bound comes from the arithmetic: P is rounded to bf16 (relative error
<= 2^-9 per probability) before the PV product and the output is rounded to
bf16 (2^-9 relative), everything else accumulates in float32.
"""
import numpy as np

BF16_MAX_ABS = 2e-2
BF16_REL_RMS = 5e-3
F32_MAX_ABS = 1e-4


def check_bf16(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    rel = np.sqrt(np.mean(err ** 2)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30)
    assert err.max() <= BF16_MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert rel <= BF16_REL_RMS, f"{what}: rel-RMS {rel:.3e}"
    return float(err.max()), float(rel)


def check_f32(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref).max()
    assert err <= F32_MAX_ABS, f"{what}: max-abs {err:.3e}"
    return float(err)
