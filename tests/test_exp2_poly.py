"""The polynomial exp2 that the kernels evaluate on the FMA pipes.

Part of the softmax exponentials (forward and backward) are computed as
2^x = 2^round(x) * p(x - round(x)) with a degree-4 minimax polynomial p and
the integer part added into the exponent bits.  These CPU tests pin that
helper without a GPU:

* the coefficients in the device header are the ones the committed Remez
  generator prints (so the header cannot drift from its derivation);
* a bit-level float32 emulation of the device sequence (round by the
  1.5 * 2^23 shift, Horner, exponent-field add) stays within 4e-6 relative
  error of exp2 over the whole range the kernels use, x in [-126, 8];
* the generator's polynomial is a minimax fit: its error equioscillates
  (degree + 2 alternating extrema of equal size).
"""

from __future__ import annotations

import re
import subprocess
import sys
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parents[1]
CSRC = ROOT / "causal_self_attention_flash_b200" / "csrc"


def header_coefficients():
    text = (CSRC / "sm100.cuh").read_text()
    found = dict(re.findall(r"constexpr float kExp2C(\d) = ([-0-9.e]+)f;", text))
    return [float(found[str(i)]) for i in range(5)]


def generator_output(degree: int) -> str:
    out = subprocess.run([sys.executable, str(CSRC / "gen_exp2_poly.py"), str(degree)],
                         capture_output=True, text=True, check=True)
    return out.stdout


def emulate(x: np.ndarray, coef) -> np.ndarray:
    """The device sequence in float32, step by step (separate multiply and
    add in place of the fused multiply-add: a rounding difference of one
    float32 ulp per step, far below the tolerance checked)."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    f = (x - (t - magic).astype(f32)).astype(f32)
    c = [f32(v) for v in coef]
    p = (c[4] * f + c[3]).astype(f32)
    p = (p * f + c[2]).astype(f32)
    p = (p * f + c[1]).astype(f32)
    p = (p * f + c[0]).astype(f32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_header_matches_generator():
    out = generator_output(4)
    gen = [float(v) for v in re.findall(r"constexpr float kExp2C\d = ([-0-9.e]+)f;", out)]
    assert gen == header_coefficients()


def test_relative_error_over_kernel_range():
    coef = header_coefficients()
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-126.0, 8.0, 400001, dtype=np.float32),
        rng.uniform(-30.0, 8.0, 200000).astype(np.float32),
        np.arange(-126, 9, dtype=np.float32),             # integers: f = 0
        np.arange(-126, 8, dtype=np.float32) + np.float32(0.5),  # round-half cases
    ])
    got = emulate(x, coef).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 4e-6, rel.max()
    assert np.all(got > 0)


def test_clamp_below_range():
    coef = header_coefficients()
    x = np.array([-np.inf, -1000.0, -127.5, -126.0], dtype=np.float32)
    got = emulate(x, coef).astype(np.float64)
    np.testing.assert_allclose(got, 2.0 ** -126, rtol=4e-6)


def test_minimax_equioscillation():
    sys.path.insert(0, str(CSRC))
    try:
        import gen_exp2_poly as g
    finally:
        sys.path.pop(0)
    for degree in (4, 5):
        coef = g.remez(degree)
        grid = np.linspace(-0.5, 0.5, 200001)
        err = np.polyval(np.asarray(coef)[::-1], grid) / np.exp2(grid) - 1.0
        emax = np.abs(err).max()
        # alternating extrema of the error, each within 1% of the maximum
        sign = np.sign(err)
        runs = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[runs[-1]]:
                runs.append(i)
            elif abs(err[i]) > abs(err[runs[-1]]):
                runs[-1] = i
        peaks = np.abs(err[runs])
        assert len(runs) >= degree + 2
        assert np.sum(peaks > 0.99 * emax) >= degree + 2
