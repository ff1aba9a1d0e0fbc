"""The erf of the tensor-core forward's GELU: Abramowitz & Stegun, Handbook of
Mathematical Functions, formula 7.1.28, erf(u) = 1 - (1 + a1 u + ... + a6
u^6)^-16 with a published |error| <= 3e-7.  Evaluated here in fp32 in the
kernel's order (Horner, then four squarings, then the reciprocal); the
coefficients are read from the kernel source, so a mistyped one fails."""
import math
import pathlib
import re

import numpy as np

SRC = pathlib.Path(__file__).resolve().parents[1] / "spatiotemporal_neural_field_b200" / "csrc" / "decode_heads.cu"


def _coefficients():
    body = SRC.read_text().split("float gelu_fast(float x) {", 1)[1].split("}", 1)[0]
    lits = [float(v) for v in re.findall(r"fmaf\([^;]*?, ([0-9.]+)f\)", body)]
    # Horner from a6: fmaf(u, a6, a5), then a4, a3, a2, a1, 1
    a6 = float(re.search(r"fmaf\(u, ([0-9.]+)f, ([0-9.]+)f\)", body).group(1))
    return a6, lits


def test_rational_erf_meets_the_published_bound():
    a6, lits = _coefficients()
    a5, a4, a3, a2, a1, one = lits
    assert one == 1.0
    u64 = np.linspace(0.0, 8.0, 100001)
    p = 1 + a1 * u64 + a2 * u64**2 + a3 * u64**3 + a4 * u64**4 + a5 * u64**5 + a6 * u64**6
    exact = np.array([math.erf(x) for x in u64])
    assert np.abs((1 - p**-16) - exact).max() <= 3e-7          # the bound, exact arithmetic
    u = u64.astype(np.float32)
    q = np.float32(a6) * u + np.float32(a5)
    for c in (a4, a3, a2, a1, 1.0):
        q = q * u + np.float32(c)
    with np.errstate(over="ignore"):
        for _ in range(4):
            q = q * q
        e = np.float32(1.0) / q
    # fp32: the squarings amplify rounding to ~2e-6, still far below fp16's 4.9e-4
    assert np.abs((1 - e.astype(np.float64)) - exact).max() <= 2e-6


def test_gelu_from_the_rational_erf():
    a6, (a5, a4, a3, a2, a1, _) = _coefficients()
    x = np.linspace(-12.0, 12.0, 4801)
    u = np.abs(x) / math.sqrt(2.0)
    e = (1 + a1 * u + a2 * u**2 + a3 * u**3 + a4 * u**4 + a5 * u**5 + a6 * u**6) ** -16
    g = np.where(x >= 0, x - 0.5 * x * e, 0.5 * x * e)
    exact = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2.0))) for v in x])
    assert np.abs(g - exact).max() <= 0.5 * 12.0 * 3e-7
