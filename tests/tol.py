"""Tolerances for GPU-vs-oracle parity, derived from the arithmetic.

The parity bound is element-wise with a floor:

    |g - o| <= rtol * max(|o|, floor * max|o|_group)

taken separately over each *group* of a result: each hash-table level, each
HexPlane plane, each weight matrix and each bias vector, each output
attribute.  A small entry is then held to its own size (down to the floor),
not to the largest entry of the whole tensor, so a mistake confined to the
fine hashed levels or to one block of weights cannot hide behind the coarse
levels' large sums.  floor = 1e-3.

* fp32 path (fp32 tables/weights, fp32 arithmetic): rtol 1e-5 on every output
  and every gradient.
* fp16 path (fp16 tables/weights, fp32 accumulate): |g - o| <= 2e-3 absolute
  on the attributes and Sigma; gradients rtol 1e-2.
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

GPU-vs-GPU consistency checks (the same arithmetic with another fp32
accumulation order) use ``normwise`` per group: they compare two results
of the library, not the library with the oracle.

Every check prints its worst ratio |g - o| / bound per group (visible with
``pytest -s``), then asserts that none exceeds 1.
"""
import numpy as np

FP32_RTOL = 1e-5
FP16_ATOL = 2e-3
FP32_GRAD_RTOL = 1e-5
FP16_GRAD_RTOL = 1e-2
FLOOR = 1e-3


def _pair(got, want, name):
    g = np.asarray(got, np.float64)
    o = np.asarray(want, np.float64)
    assert g.shape == o.shape, (name, g.shape, o.shape)
    assert np.all(np.isfinite(g)), name + ": non-finite values"
    return g, o


def elementwise_ratio(got, want, rtol, floor=FLOOR, rho=None):
    """(worst ratio, flat index) of |g - o| / (rtol * max(|o|, floor * max|o|[, rho]))."""
    g = np.asarray(got, np.float64).reshape(-1)
    o = np.asarray(want, np.float64).reshape(-1)
    if g.size == 0:
        return 0.0, -1
    err = np.abs(g - o)
    ref = np.max(np.abs(o))
    scale = np.maximum(np.abs(o), floor * ref)
    if rho is not None:
        scale = np.maximum(scale, np.asarray(rho, np.float64).reshape(-1))
    bound = rtol * scale
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / np.where(bound > 0, bound, 1.0), np.where(err > 0, np.inf, 0.0))
    i = int(np.argmax(ratio))
    return float(ratio[i]), i


def elementwise(got, want, rtol, name="", groups=None, floor=FLOOR, rho=None):
    """Element-wise check with a floor, per group.

    ``groups``: None (the whole array is one group), or a list of
    (label, index) where index selects the group's entries of the flattened
    array (a slice or an index array).  ``rho``: the root-sum-square of the
    terms of each entry's sum (``tests/magnitude.py``), or None where the
    entries are not cancelling sums.  Prints one line per group with its
    worst ratio (and, with ``rho``, the worst ratio without it and how many
    entries only ``rho`` admits); asserts every ratio <= 1 after all groups
    are reported."""
    g, o = _pair(got, want, name)
    gf, of = g.reshape(-1), o.reshape(-1)
    rf = None if rho is None else np.asarray(rho, np.float64).reshape(-1)
    assert rf is None or rf.shape == of.shape, (name, "rho shape")
    if groups is None:
        groups = [("", slice(None))]
    worst, bad = 0.0, []
    for label, sel in groups:
        rs = None if rf is None else rf[sel]
        r, i = elementwise_ratio(gf[sel], of[sel], rtol, floor, rs)
        tag = name + ("[" + label + "]" if label else "")
        if i >= 0:
            line = "  %-34s worst %.3f (g %.6e o %.6e max|o| %.3e)" % (
                tag, r, gf[sel][i], of[sel][i], float(np.max(np.abs(of[sel]))))
            if rs is not None:
                r0, _ = elementwise_ratio(gf[sel], of[sel], rtol, floor)
                e = np.abs(gf[sel] - of[sel])
                b0 = rtol * np.maximum(np.abs(of[sel]), floor * np.max(np.abs(of[sel])))
                line += " | without rho %.3f, %d of %d entries need rho" % (r0, int(np.sum(e > b0)), e.size)
            print(line)
        worst = max(worst, r)
        if r > 1.0:
            bad.append("%s ratio %.3g" % (tag, r))
    assert not bad, "element-wise bound (rtol %.1e, floor %.0e) exceeded: %s" % (rtol, floor, "; ".join(bad))
    return worst


def rowwise(got, want, rtol=FP32_RTOL, name=""):
    """Per-row relative bound |g - o| <= rtol * max_j |o_row|: used only where
    a row is one sum whose terms the row maximum bounds (see callers)."""
    g, o = _pair(got, want, name)
    g = g.reshape(len(g), -1)
    o = o.reshape(len(o), -1)
    scale = np.maximum(np.max(np.abs(o), axis=1, keepdims=True), 1e-30)
    rel = np.abs(g - o) / scale
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= rtol, "%s: max row-relative error %.3e > %.1e at %s" % (
        name, worst, rtol, np.unravel_index(np.argmax(rel), rel.shape))
    return worst


def absolute(got, want, atol=FP16_ATOL, name=""):
    g, o = _pair(got, want, name)
    err = float(np.max(np.abs(g - o))) if g.size else 0.0
    print("  %-40s max |g-o| %.3e (bound %.1e)" % (name, err, atol))
    assert err <= atol, "%s: max abs error %.3e > %.1e" % (name, err, atol)
    return err


def normwise(got, want, rtol, name="", groups=None):
    """|g - o| <= rtol * max|o|, per group: GPU-vs-GPU consistency only."""
    g, o = _pair(got, want, name)
    gf, of = g.reshape(-1), o.reshape(-1)
    if groups is None:
        groups = [("", slice(None))]
    bad = []
    worst = 0.0
    for label, sel in groups:
        ref = max(float(np.max(np.abs(of[sel]))) if of[sel].size else 0.0, 1e-30)
        err = float(np.max(np.abs(gf[sel] - of[sel]))) if of[sel].size else 0.0
        worst = max(worst, err / ref)
        if err > rtol * ref:
            bad.append("%s%s normwise error %.3e > %.1e (max|o| %.3e)"
                       % (name, "[" + label + "]" if label else "", err / ref, rtol, ref))
    assert not bad, "; ".join(bad)
    return worst


# ---------------------------------------------------------------------------
# Groups
# ---------------------------------------------------------------------------
def table_levels(L, T, F):
    """One group per hash-table level of an L x T x F gradient."""
    n = T * F
    return [("level %d" % l, slice(l * n, (l + 1) * n)) for l in range(L)]


def weight_blocks(shapes, prefix="", offset=0):
    """One group per weight matrix and per bias vector of a packed
    [W0 b0 W1 b1 ...] vector (W row-major [out][in])."""
    out, o = [], offset
    for j, (m, k) in enumerate(shapes):
        out.append(("%sW%d %dx%d" % (prefix, j, m, k), slice(o, o + m * k)))
        o += m * k
        out.append(("%sb%d %d" % (prefix, j, m), slice(o, o + m)))
        o += m
    return out


def plane_groups(hx):
    """One group per HexPlane plane (scale-major, XY XZ YZ XT YT ZT)."""
    names = ("XY", "XZ", "YZ", "XT", "YT", "ZT")
    out, o = [], 0
    for i, (rows, cols) in enumerate(hx.plane_shapes()):
        n = rows * cols * hx.channels
        out.append(("%d %s" % (hx.scales[i // 6], names[i % 6]), slice(o, o + n)))
        o += n
    return out


def column_groups(ncols, labels=None):
    """One group per column of an N x ncols array (flattened row-major)."""
    labels = labels or ["col %d" % c for c in range(ncols)]
    return [(labels[c], slice(c, None, ncols)) for c in range(ncols)]


RENDER_ATOL = 2e-3
RENDER_GRAD_RTOL = 1e-2
# A pixel with decisions within fp32 reach of their thresholds may take any
# of them the other way; the oracle bounds each single change
# (oracle/render.py pixel_flip_bound) and several together change the pixel
# by the sum of their changes up to products of two of the (small) alphas
# involved, which this factor covers.
RENDER_FLIP_SLACK = 1.5


def absolute_with_bound(got, want, bound, atol, name=""):
    """|g - o| <= atol + RENDER_FLIP_SLACK * bound element-wise; prints the
    worst ratio and the number of entries that needed their bound."""
    g, o = _pair(got, want, name)
    b = np.asarray(bound, np.float64).reshape(g.shape)
    err = np.abs(g - o)
    lim = atol + RENDER_FLIP_SLACK * b
    ratio = float(np.max(err / lim)) if g.size else 0.0
    needed = int(np.count_nonzero(err > atol))
    print("  %-40s worst |g-o|/bound %.3f, %d of %d entries beyond %.1e (within their flip bound)"
          % (name, ratio, needed, g.size, atol))
    assert ratio <= 1.0, "%s: |g-o| exceeds its bound by %.3fx" % (name, ratio)
    return ratio
