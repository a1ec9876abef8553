"""Shared helpers for the GPU parity tests: tolerances and comparisons.

Tolerances (fixed for every workload): bf16 outputs O, dQ, dK, dV must be
within max-abs 2e-2 AND relative L2 1e-2 of the fp64 oracle; fp32 LSE
within 1e-4 absolute; fp32 Delta within 1e-4 relative to its scale.
"""

from __future__ import annotations

import numpy as np

MAX_ABS = 2e-2
REL_L2 = 1e-2
LSE_ABS = 1e-4


def errors(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), "non-finite values in GPU output"
    diff = gpu - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    nrm = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff)) / nrm if nrm > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def check_bf16(name, gpu, ref, max_abs=MAX_ABS, rel_l2=REL_L2):
    ma, rl = errors(gpu, ref)
    assert ma <= max_abs and rl <= rel_l2, (
        f"{name}: max-abs {ma:.3e} (tol {max_abs}), rel-L2 {rl:.3e} (tol {rel_l2})")
    return ma, rl


def check_bf16_beyond_rounding(name, gpu, ref, max_abs=MAX_ABS, rel_l2=REL_L2):
    """For cases outside the five workloads whose values are so large that
    bf16's own rounding (half an ulp, up to 2^-8 |x|) exceeds max_abs: the
    error beyond that rounding must stay within max_abs, and rel-L2 within
    rel_l2."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    excess = float((np.abs(gpu - ref) - 2.0 ** -8 * np.abs(ref)).max())
    _, rl = errors(gpu, ref)
    assert excess <= max_abs and rl <= rel_l2, (
        f"{name}: error beyond bf16 rounding {excess:.3e} (tol {max_abs}), "
        f"rel-L2 {rl:.3e} (tol {rel_l2})")
    return excess, rl


def check_lse(gpu, ref, tol=LSE_ABS):
    ma, _ = errors(gpu, ref)
    assert ma <= tol, f"lse: max-abs {ma:.3e} (tol {tol})"
    return ma
