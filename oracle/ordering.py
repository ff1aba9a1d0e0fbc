"""Oracle: Z-order (Morton) ordering of Gaussians for gather locality.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: the KineticGS notes, "overall kinetic synchronisation": particle
coordinates are serialised onto a Z-order (or Hilbert) space-filling curve,
whose locality keeps spatial neighbours close in the 1D order.  Here the
curve orders the Gaussians themselves, so that consecutive positions (one
tile of the decoder) read neighbouring hash-table entries.

Readings: the curve runs over the normalised spatial coordinates mu_bar of
Eq. 7 (the same fp32 values the decoder interpolates at, so a whole scene,
contracted, fits the unit cube); each axis is quantised to 10 bits,
q = min(floor(mu_bar * 1024), 1023); the key interleaves the bits as
x0 y0 z0 x1 y1 z1 ... (x in the lowest bit), a 30-bit code.  Time is left
out: every Gaussian is decoded at every frame, so the order is per scene.
Equal keys keep their input order (a stable sort).
"""
from __future__ import annotations

import numpy as np

from . import hashgrid

BITS = 10


def quantise(mu_bar: np.ndarray) -> np.ndarray:
    """N x 3 fp32 in [0, 1] -> N x 3 integer cells in [0, 2^BITS)."""
    scaled = np.asarray(mu_bar, np.float32) * np.float32(1 << BITS)     # exact: power of two
    return np.minimum(np.floor(scaled).astype(np.int64), (1 << BITS) - 1)


def interleave(q: np.ndarray) -> np.ndarray:
    """Bit b of axis d goes to bit 3b + d of the key (pure-Python loop)."""
    q = np.asarray(q, np.int64)
    key = np.zeros(q.shape[0], np.int64)
    for b in range(BITS):
        for d in range(3):
            key |= ((q[:, d] >> b) & 1) << (3 * b + d)
    return key.astype(np.uint32)


def morton_keys(pos: np.ndarray, t_min: float, t_max: float, normalised_input: bool = False) -> np.ndarray:
    if normalised_input:
        xt = hashgrid._clamp01(np.asarray(pos, np.float32))
    else:
        xt = hashgrid.normalise(pos, t_min, t_max)
    return interleave(quantise(xt[:, :3]))


def morton_order(keys: np.ndarray) -> np.ndarray:
    """The permutation that sorts the keys, equal keys in input order."""
    return np.argsort(np.asarray(keys, np.uint32), kind="stable").astype(np.uint32)
