"""Shared comparison helpers for the GPU parity tests (no attention arithmetic here)."""
from __future__ import annotations

import numpy as np

# Tolerances of the parity bar: bf16 inputs -> max-abs 2e-2 and mean-abs 2e-3 on outputs;
# fp32 inputs -> 1e-4; LSE (natural log) -> 1e-3 absolute.
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
F32_ABS = 1e-4
LSE_ABS = 1e-3


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got) == np.isfinite(ref)), "non-finite pattern differs"
    fin = np.isfinite(ref)
    if not np.all(np.isinf(ref[~fin]) == np.isinf(got[~fin])) or not np.array_equal(ref[~fin], got[~fin]):
        raise AssertionError("infinite entries differ")
    d = np.abs(got[fin] - ref[fin])
    return (float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0,
            float(np.abs(ref[fin]).max()) if d.size else 0.0)


def assert_close_bf16(got, ref, what="o", max_abs=BF16_MAX_ABS, mean_abs=BF16_MEAN_ABS):
    mx, mean, ref_max = errors(got, ref)
    # the bf16 output grid: half an ulp at |x| in [8, 16) is already 0.031 > 2e-2
    assert ref_max < 8.0, f"{what}: |ref| reaches {ref_max:.3g}; the 2e-2 bar is below bf16 resolution there"
    assert mx <= max_abs, f"{what}: max-abs {mx:.3e} > {max_abs:.1e} (mean {mean:.3e}, |ref|max {ref_max:.3g})"
    assert mean <= mean_abs, f"{what}: mean-abs {mean:.3e} > {mean_abs:.1e} (max {mx:.3e})"
    return mx, mean


def assert_close_f32(got, ref, what="o", tol=F32_ABS):
    mx, mean, _ = errors(got, ref)
    assert mx <= tol, f"{what}: max-abs {mx:.3e} > {tol:.1e}"
    return mx, mean


def assert_lse(got, ref, tol=LSE_ABS):
    mx, mean, _ = errors(got, ref)
    assert mx <= tol, f"lse: max-abs {mx:.3e} > {tol:.1e}"
    return mx
