"""Shared parity helpers: tolerances and comparison against the oracle."""
import numpy as np

# Per-element tolerance, written out: FP32 K/V -> max |gpu - oracle| <= 1e-5;
# 16-bit and FP8 K/V -> |err| <= 2e-3, or |err| <= 2e-3 * |oracle|.
FP32_ABS = 1e-5
LOWP_TOL = 2e-3


def assert_close(got, want, dtype, what="out"):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU values"
    err = np.abs(got - want)
    if dtype == "f32":
        worst = float(err.max(initial=0.0))
        assert worst <= FP32_ABS, f"{what}: max abs error {worst:.3e} > {FP32_ABS}"
    else:
        ok = (err <= LOWP_TOL) | (err <= LOWP_TOL * np.abs(want))
        if not ok.all():
            i = np.unravel_index(np.argmax(np.where(ok, 0, err)), err.shape)
            raise AssertionError(f"{what}: {int((~ok).sum())} elements out of tolerance, "
                                 f"worst at {i}: gpu {got[i]:.6g} oracle {want[i]:.6g}")
    return float(err.max(initial=0.0))


def lse_tol(dtype):
    return FP32_ABS if dtype == "f32" else LOWP_TOL
