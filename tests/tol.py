"""Tolerances for GPU-vs-oracle parity, derived from the arithmetic.

* fp32 path (fp32 tables/weights, fp32 arithmetic): "max relative error
  <= 1e-5", read per Gaussian row: |g - o| <= 1e-5 * max_j |o_row|.  Every
  output is a short fp32 sum (16-term interpolation, <= 128-term dot products)
  or a well-conditioned function of one; such a sum's rounding error is a few
  ulp (6e-8) of the magnitude of its terms, which the row maximum bounds.
* fp16 path (fp16 tables/weights, fp32 accumulate): |g - o| <= 2e-3 on the
  attributes and Sigma.
* gradients: normwise per tensor, |g - o| <= rtol * max|o| with rtol 1e-5
  (fp32 path) or 1e-2 (fp16 path); atomics make the summation order vary, so
  only a normwise bound is meaningful for entries that receive many terms.
* integer results (corner indices): bit-exact.
* rendering (fp32 projection and blending): on pixels where no decision lies
  near its threshold, |C - C_oracle| <= 2e-3 (and the same on the final
  transmittance).  The projected mean carries fp32 rounding of the image
  coordinate (ulp 6e-5 at x = 640, a few roundings: ~2e-4 pixel); for the
  narrowest footprint the filter allows (sigma ~0.55 px) at the 3-sigma edge
  that moves d^2 by ~1e-3 and alpha by ~5e-4 relative, and the blended sum
  is a convex combination of colours of order 1.  Gradients: normwise 1e-2
  -- per-Gaussian sums over many pixels, some of whose decisions sit near a
  threshold and may go the other way in fp32.
"""
import numpy as np

FP32_RTOL = 1e-5
FP16_ATOL = 2e-3
FP32_GRAD_RTOL = 1e-5
FP16_GRAD_RTOL = 1e-2


def rowwise(got, want, rtol=FP32_RTOL, name=""):
    g = np.asarray(got, np.float64).reshape(len(got), -1)
    o = np.asarray(want, np.float64).reshape(len(want), -1)
    assert g.shape == o.shape, (name, g.shape, o.shape)
    assert np.all(np.isfinite(g)), name + ": non-finite values"
    scale = np.maximum(np.max(np.abs(o), axis=1, keepdims=True), 1e-30)
    rel = np.abs(g - o) / scale
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= rtol, "%s: max row-relative error %.3e > %.1e at %s" % (
        name, worst, rtol, np.unravel_index(np.argmax(rel), rel.shape))
    return worst


def absolute(got, want, atol=FP16_ATOL, name=""):
    g = np.asarray(got, np.float64)
    o = np.asarray(want, np.float64)
    assert g.shape == o.shape, (name, g.shape, o.shape)
    assert np.all(np.isfinite(g)), name + ": non-finite values"
    err = float(np.max(np.abs(g - o))) if g.size else 0.0
    assert err <= atol, "%s: max abs error %.3e > %.1e" % (name, err, atol)
    return err


def normwise(got, want, rtol, name=""):
    g = np.asarray(got, np.float64)
    o = np.asarray(want, np.float64)
    assert g.shape == o.shape, (name, g.shape, o.shape)
    assert np.all(np.isfinite(g)), name + ": non-finite values"
    ref = max(float(np.max(np.abs(o))), 1e-30)
    err = float(np.max(np.abs(g - o)))
    assert err <= rtol * ref, "%s: normwise error %.3e > %.1e (max|o| %.3e)" % (name, err / ref, rtol, ref)
    return err / ref


RENDER_ATOL = 2e-3
RENDER_GRAD_RTOL = 1e-2
