"""Oracle: input normalisation and the 4D multiresolution hash encoder.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources, on *Implicit 4D Gaussian Splatting for Fast Motion with Large
Inter-Frame Displacements* (SPIN-4DGS):

* section 3.3 "input position normalisation", Eq. 7 (Mip-NeRF scene
  contraction, then mu_bar = contract(mu)/4 + 1/2) and Eq. 8 (time divided by
  the total duration, x~ = [mu_bar, t_norm] in [0,1]^4);
* section 3.3 "encoder architecture", Eq. 9: Instant-NGP's multiresolution
  hash grid extended to 4D by adding the time axis; the features of all L
  levels (F channels each) are concatenated into z in R^{LF}.

Details the page leaves open, and the reading taken here:

* hash: xor of (coordinate x prime) over the four axes with primes
  (1, 2654435761, 805459861, 3674653429), products wrapped to 32 bits, then
  reduced mod T = 2^log2_T; a level is indexed densely (x fastest, then y, z,
  t) when the product of its per-axis resolutions is at most T;
* resolution = number of grid vertices along an axis, so a coordinate in
  [0,1] is scaled by (res - 1); per level, res_l = floor(Nmin * b^l) with
  b = exp((ln Nmax - ln Nmin)/(L - 1)) (Instant-NGP's geometric growth),
  computed separately for the three spatial axes and the time axis;
* the cell index floor(p) is clamped to [0, res-2] so that x~ = 1 falls in
  the last cell with weight 1; normalised coordinates are clamped to [0,1]
  and a NaN coordinate is treated as 0;
* normalisation runs in fp32 with a fixed operation order and no fused
  multiply-add: n = sqrt((x*x + y*y) + z*z); inside if n <= 1, else
  c_i = (2 - 1/n) * (mu_i / n); mu_bar_i = c_i*0.25 + 0.5;
  t_norm = clamp((t - t_min)/(t_max - t_min), 0, 1).
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

PRIMES = (1, 2654435761, 805459861, 3674653429)
F32 = np.float32


def level_resolutions(L: int, nmin: int, nmax: int) -> List[int]:
    """Per-level vertex counts along one axis, geometric growth Nmin -> Nmax."""
    if L == 1:
        return [int(nmin)]
    b = math.exp((math.log(nmax) - math.log(nmin)) / (L - 1))
    return [int(math.floor(nmin * b ** l + 1e-9)) for l in range(L)]


def grid_resolutions(L: int, nmin_s: int, nmax_s: int, nmin_t: int, nmax_t: int) -> np.ndarray:
    """L x 4 vertex counts (x, y, z, t); the three spatial axes are equal."""
    rs = level_resolutions(L, nmin_s, nmax_s)
    rt = level_resolutions(L, nmin_t, nmax_t)
    return np.array([[rs[l], rs[l], rs[l], rt[l]] for l in range(L)], dtype=np.int64)


def _clamp01(v: np.ndarray) -> np.ndarray:
    v = np.where(np.isnan(v), F32(0), v)
    return np.minimum(np.maximum(v, F32(0)), F32(1)).astype(F32)


def normalise(pos: np.ndarray, t_min: float, t_max: float) -> np.ndarray:
    """Eq. 7 + Eq. 8 in fp32: N x 4 (x,y,z,t) -> N x 4 x~ in [0,1]^4."""
    pos = np.asarray(pos, dtype=F32)
    mu = pos[:, :3]
    x, y, z = mu[:, 0], mu[:, 1], mu[:, 2]
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        n2 = (x * x + y * y) + z * z
        n = np.sqrt(n2)
        inside = n <= F32(1)
        k = F32(2) - F32(1) / n
        outside = k[:, None] * (mu / n[:, None])
        c = np.where(inside[:, None], mu, outside).astype(F32)
        mu_bar = c * F32(0.25) + F32(0.5)
        span = F32(t_max) - F32(t_min)
        t_norm = (pos[:, 3] - F32(t_min)) / span
    out = np.empty_like(pos)
    out[:, :3] = _clamp01(mu_bar)
    out[:, 3] = _clamp01(t_norm)
    return out


def is_dense(res_l: Sequence[int], log2_T: int) -> bool:
    return int(np.prod([int(r) for r in res_l])) <= (1 << log2_T)


def corner_select(xt: np.ndarray, res: np.ndarray, log2_T: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Per level: the cell of each position and the 16 corner table indices.

    Returns (base, frac, idx):
      base  N x L x 4 int64   lower cell vertex per axis,
      frac  N x L x 4 float32 position inside the cell per axis (p - base),
      idx   N x L x 16 uint32 table index of corner c, where bit d of c
            (d = 0 x, 1 y, 2 z, 3 t) selects vertex base_d + 1.
    """
    xt = np.asarray(xt, dtype=F32)
    N = xt.shape[0]
    L = res.shape[0]
    T = 1 << log2_T
    base = np.empty((N, L, 4), np.int64)
    frac = np.empty((N, L, 4), F32)
    idx = np.empty((N, L, 16), np.uint32)
    for l in range(L):
        for d in range(4):
            r = int(res[l, d])
            p = xt[:, d] * F32(r - 1)                     # fp32 product
            i = np.clip(np.floor(p).astype(np.int64), 0, r - 2)
            base[:, l, d] = i
            frac[:, l, d] = p - i.astype(F32)             # exact
        dense = is_dense(res[l], log2_T)
        for c in range(16):
            v = [base[:, l, d] + ((c >> d) & 1) for d in range(4)]
            if dense:
                rx, ry, rz = (int(res[l, 0]), int(res[l, 1]), int(res[l, 2]))
                e = v[0] + rx * (v[1] + ry * (v[2] + rz * v[3]))
            else:
                h = np.zeros(N, np.uint64)
                for d in range(4):
                    prod = (v[d].astype(np.uint64) * np.uint64(PRIMES[d])) & np.uint64(0xFFFFFFFF)
                    h ^= prod
                e = h & np.uint64(T - 1)
            idx[:, l, c] = e.astype(np.uint32)
    return base, frac, idx


def corner_weights(frac: np.ndarray) -> np.ndarray:
    """N x L x 16 fp64 quadrilinear weights: prod_d (bit_d ? w_d : 1 - w_d)."""
    w = frac.astype(np.float64)
    out = np.ones(frac.shape[:2] + (16,), np.float64)
    for c in range(16):
        for d in range(4):
            out[:, :, c] *= w[:, :, d] if (c >> d) & 1 else (1.0 - w[:, :, d])
    return out


def encode(xt: np.ndarray, tables: np.ndarray, res: np.ndarray, log2_T: int) -> np.ndarray:
    """Eq. 9: z[n, l*F + f] = sum_c weight_c * table[l, idx_c, f]  (fp64).

    ``tables`` is L x T x F (fp32 or fp16 storage); values are read exactly."""
    L, T, F = tables.shape
    assert T == 1 << log2_T
    _, frac, idx = corner_select(xt, res, log2_T)
    wts = corner_weights(frac)
    N = xt.shape[0]
    z = np.zeros((N, L * F), np.float64)
    for l in range(L):
        for f in range(F):
            col = np.ascontiguousarray(tables[l, :, f]).astype(np.float64)
            acc = np.zeros(N, np.float64)
            for c in range(16):
                acc += wts[:, l, c] * np.take(col, idx[:, l, c].astype(np.int64))
            z[:, l * F + f] = acc
    return z


def scatter_table_grad_level(dz: np.ndarray, xt: np.ndarray, res: np.ndarray, log2_T: int, l: int,
                             F: int) -> np.ndarray:
    """Level l of the adjoint of ``encode`` w.r.t. the tables, T x F:
    grad[idx_c, f] += weight_c * dz[:, l*F + f] (for tables too large to hold
    every level's fp64 gradient at once)."""
    T = 1 << log2_T
    _, frac, idx = corner_select(xt, res, log2_T)
    wts = corner_weights(frac)
    grad = np.zeros((T, F), np.float64)
    for f in range(F):
        g = dz[:, l * F + f]
        # all 16 corners of every position in one serial histogram
        grad[:, f] = np.bincount(idx[:, l, :].astype(np.int64).reshape(-1),
                                 weights=(wts[:, l, :] * g[:, None]).reshape(-1), minlength=T)
    return grad


def scatter_table_grad(dz: np.ndarray, xt: np.ndarray, res: np.ndarray, log2_T: int,
                       L: int, F: int) -> np.ndarray:
    """Adjoint of ``encode`` w.r.t. the tables: grad[l, idx_c, f] += weight_c * dz."""
    grad = np.zeros((L, 1 << log2_T, F), np.float64)
    for l in range(L):
        grad[l] = scatter_table_grad_level(dz, xt, res, log2_T, l, F)
    return grad


# ---------------------------------------------------------------------------
# Position gradient (trainable Gaussian means, SPIN-4DGS section 3.3: the
# positions are optimised jointly with the decoder)
# ---------------------------------------------------------------------------
def contraction_jacobian(pos: np.ndarray) -> np.ndarray:
    """d mu_bar / d mu of Eq. 7, N x 3 x 3 fp64, at the fp32 positions.

    Inside the unit ball mu_bar = mu/4 + 1/2, so the Jacobian is I/4.
    Outside, c = (2 - 1/n) mu / n = (2/n - 1/n^2) mu with n = |mu|, so
    dc/dmu = (2/n - 1/n^2) I + (2/n^4 - 2/n^3) mu mu^T, and mu_bar = c/4 + 1/2.
    The branch is the one the fp32 normalisation takes (n <= 1 in fp32)."""
    mu32 = np.asarray(pos, F32)[:, :3]
    x, y, z = mu32[:, 0], mu32[:, 1], mu32[:, 2]
    inside = np.sqrt((x * x + y * y) + z * z) <= F32(1)
    mu = mu32.astype(np.float64)
    n = np.sqrt(np.sum(mu * mu, axis=1))
    eye = np.broadcast_to(np.eye(3), (mu.shape[0], 3, 3))
    with np.errstate(divide="ignore", invalid="ignore"):
        g = 2.0 / n - 1.0 / n ** 2
        h = 2.0 / n ** 4 - 2.0 / n ** 3
        out = g[:, None, None] * eye + h[:, None, None] * mu[:, :, None] * mu[:, None, :]
    out = np.where(inside[:, None, None], eye, out)
    return 0.25 * out


def clamp_passes(v: np.ndarray) -> np.ndarray:
    """Mask of the clamp to [0, 1]: 1 where the value passes unchanged."""
    v = np.asarray(v)
    return ((v >= 0) & (v <= 1)).astype(np.float64)


def encode_position_grad(dz: np.ndarray, xt: np.ndarray, tables: np.ndarray, res: np.ndarray,
                         log2_T: int) -> np.ndarray:
    """Adjoint of ``encode`` w.r.t. the normalised position, N x 4 fp64.

    z_l = sum_c W_c e_c with W_c = prod_d (bit_d ? w_d : 1 - w_d) and
    w_d = x~_d (res_d - 1) - base_d, so
    d<dz_l, z_l>/dx~_d = (res_d - 1) sum_c (dz_l . e_c) dW_c/dw_d,
    dW_c/dw_d = (bit_d ? 1 : -1) prod_{e != d} (bit_e ? w_e : 1 - w_e)
    (the derivative inside the cell; the interpolant is continuous across
    cells, its derivative is taken from the cell the position falls in)."""
    L, T, F = tables.shape
    _, frac, idx = corner_select(xt, res, log2_T)
    w = frac.astype(np.float64)
    N = xt.shape[0]
    g = np.zeros((N, 4), np.float64)
    for l in range(L):
        s = np.zeros((N, 16), np.float64)          # dz_l . e_c per corner
        for f in range(F):
            col = np.ascontiguousarray(tables[l, :, f]).astype(np.float64)
            s += dz[:, l * F + f][:, None] * np.take(col, idx[:, l, :].astype(np.int64))
        for d in range(4):
            acc = np.zeros(N, np.float64)
            for c in range(16):
                dw = np.ones(N, np.float64) if (c >> d) & 1 else -np.ones(N, np.float64)
                for e in range(4):
                    if e != d:
                        dw = dw * (w[:, l, e] if (c >> e) & 1 else 1.0 - w[:, l, e])
                acc += s[:, c] * dw
            g[:, d] += (int(res[l, d]) - 1) * acc
    return g
