"""Helpers shared by the GPU parity tests: error statistics and the tolerance gates.

Tolerances (bf16 outputs and gradients): max-abs <= 2e-2 and mean-abs <= 2e-3 against the
fp64 oracle, plus relative L2 <= 1e-2 so that a real error cannot hide under the loose
absolute gates; fp32 problems: max-abs <= 1e-5.  LSE: 1e-3 (bf16 inputs) / 1e-5 (fp32).
"""
import numpy as np

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
BF16_REL_L2 = 1e-2
F32_MAX_ABS = 1e-5
LSE_BF16 = 1e-3
LSE_F32 = 1e-5


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    return float(err.max()), float(err.mean()), rel


def assert_close(got, ref, dtype: str, what: str):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    mx, mean, rel = errors(got, ref)
    if dtype == "f32":
        assert mx <= F32_MAX_ABS, f"{what}: max-abs {mx:.3e} > {F32_MAX_ABS}"
    else:
        assert mx <= BF16_MAX_ABS, f"{what}: max-abs {mx:.3e} > {BF16_MAX_ABS}"
        assert mean <= BF16_MEAN_ABS, f"{what}: mean-abs {mean:.3e} > {BF16_MEAN_ABS}"
        assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e} > {BF16_REL_L2}"
    return mx, mean, rel


def assert_lse_close(got, ref, dtype: str, what: str = "lse"):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    tol = LSE_F32 if dtype == "f32" else LSE_BF16
    mx = float(np.abs(got - np.asarray(ref, dtype=np.float64)).max())
    assert mx <= tol, f"{what}: max-abs {mx:.3e} > {tol}"
    return mx
