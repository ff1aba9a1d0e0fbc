"""Oracle: EWA projection and alpha compositing of the decoded Gaussians.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: *Implicit 4D Gaussian Splatting for Fast Motion with Large
Inter-Frame Displacements* (SPIN-4DGS), section 3.1: a Gaussian is
exp(-(x-mu)^T Sigma^-1 (x-mu) / 2) (Eq. 1) with colour from spherical-harmonic
coefficients and an opacity o; it is projected to the image plane with the
view transform W and the Jacobian J of the projection (Zwicker et al. 2001):
Sigma_2D = J W Sigma W^T J^T (Eq. 3); each pixel's colour is the front-to-back
alpha blend C = sum_i c_i a_i prod_{j<i} (1 - a_j) with a_i = o_i G_2D,i(x)
(Eq. 4).  The pages stop there; the readings below fill in the rest and the
CUDA path implements the same readings.

Readings (where the pages are silent):
  * Camera: pinhole, world -> camera x_c = R mu + t (R, t from a 3x4 view
    matrix, W = R in Eq. 3), the camera looks along +z; the image point of x_c
    is (fx x/z + cx, fy y/z + cy) and J is that map's Jacobian at x_c.  The
    image spans [0, width] x [0, height]; pixel (i, j) (column i, row j) is
    evaluated at (i + 1/2, j + 1/2).
  * A Gaussian with camera depth z <= z_near is culled.  ``lowpass`` (in
    pixels^2) is added to the diagonal of Sigma_2D -- the screen-space
    filter of EWA splatting; lowpass = 0 is Eq. 3 exactly.  A Gaussian whose
    filtered Sigma_2D has a determinant <= 0 is culled.
  * Support: a Gaussian covers a pixel when the pixel's Mahalanobis distance
    d^2 = (x - mu_2D)^T Sigma_2D^-1 (x - mu_2D) is at most 9 (its 3-sigma
    ellipse).  a = min(alpha_max, o exp(-d^2/2)); a covered pixel with
    a < alpha_min is skipped.
  * Order: by camera depth z ascending, equal depths by Gaussian index.
  * Termination: blending stops before the first Gaussian that would bring
    the transmittance below t_stop (t_stop = 0: never; all N terms of Eq. 4).
  * Background: C += T_final * background (the pages' Eq. 4 has none:
    background 0).
  * Colour: ``sh_degree`` -1 takes RGB as given; degree D in 0..3 takes
    (D+1)^2 coefficients per channel, stored coefficient-major
    (k[n, 3*(l*l + l + m) + channel]), evaluates the real spherical harmonics
    Y_lm (no Condon-Shortley phase) in the viewing direction
    (mu - camera centre) / |mu - camera centre| and clamps the sum at 0.

Everything is fp64.  Each pixel also gets a margin flag: False when any
decision taken at that pixel (the 3-sigma test, alpha_min, the alpha_max clamp,
termination, the depth order of two contributors) lies so close to its
threshold that fp32 rounding may take it the other way.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np
from numpy.polynomial import legendre as npleg

SUPPORT_D2 = 9.0            # 3-sigma ellipse
PACK3 = ((0, 0), (0, 1), (0, 2), (1, 1), (1, 2), (2, 2))

# margins below which a decision is called ambiguous (see module docstring)
D2_MARGIN = 2.5e-3          # absolute, on d^2 near 9 (fp32 error <= 1.3e-3 at the narrowest filtered footprint)
REL_MARGIN = 2e-3           # relative, on alpha vs alpha_min / alpha_max and T vs t_stop
DEPTH_MARGIN = 1e-6         # relative gap between two contributors' depths (fp32 depth: <= 3e-7)


@dataclass
class Camera:
    view: np.ndarray        # 3 x 4 [R | t]
    fx: float
    fy: float
    cx: float
    cy: float
    width: int
    height: int
    z_near: float = 0.2

    @property
    def R(self) -> np.ndarray:
        return np.asarray(self.view, np.float64)[:, :3]

    @property
    def t(self) -> np.ndarray:
        return np.asarray(self.view, np.float64)[:, 3]

    @property
    def centre(self) -> np.ndarray:
        """Camera centre in world coordinates: x_c = 0  <=>  mu = -R^T t."""
        return -self.R.T @ self.t


@dataclass
class Settings:
    sh_degree: int = 3
    lowpass: float = 0.3
    alpha_max: float = 0.99
    alpha_min: float = 1.0 / 255.0
    t_stop: float = 1e-4
    background: np.ndarray = field(default_factory=lambda: np.zeros(3))


# ---------------------------------------------------------------------------
# real spherical harmonics, from their definition
# ---------------------------------------------------------------------------
def _sh_terms(l: int, m: int):
    """Y_lm on the unit sphere as K * Q(z) * {Re, Im}((x + i y)^|m|) with
    Q = d^|m| P_l / dz^|m| (Legendre P_l), K = sqrt((2l+1)/(4 pi) (l-|m|)!/(l+|m|)!),
    times sqrt 2 for m != 0: cos(m phi) sin^m(theta) = Re((x+iy)^m) on the
    sphere and P_l^m(cos theta) = sin^m(theta) Q(cos theta) without the
    Condon-Shortley phase."""
    am = abs(m)
    K = math.sqrt((2 * l + 1) / (4 * math.pi) * math.factorial(l - am) / math.factorial(l + am))
    if m != 0:
        K *= math.sqrt(2.0)
    Q = npleg.Legendre.basis(l).deriv(am).convert(kind=np.polynomial.Polynomial)
    return K, Q, am, (m >= 0)


def sh_basis(d: np.ndarray, degree: int) -> np.ndarray:
    """(n, (degree+1)^2) values of Y_lm at unit directions d (n x 3), index l*l + l + m."""
    d = np.asarray(d, np.float64)
    w = d[:, 0] + 1j * d[:, 1]
    out = []
    for l in range(degree + 1):
        for m in range(-l, l + 1):
            K, Q, am, real = _sh_terms(l, m)
            p = w ** am
            out.append(K * Q(d[:, 2]) * (p.real if real else p.imag))
    return np.stack(out, axis=1)


def sh_basis_grad(d: np.ndarray, degree: int) -> np.ndarray:
    """(n, (degree+1)^2, 3): gradient in R^3 of the polynomial extension
    K Q(z) {Re,Im}((x+iy)^m) used by ``sh_basis`` (equal to Y_lm on the sphere)."""
    d = np.asarray(d, np.float64)
    w = d[:, 0] + 1j * d[:, 1]
    out = []
    for l in range(degree + 1):
        for m in range(-l, l + 1):
            K, Q, am, real = _sh_terms(l, m)
            p = w ** am
            dp = am * w ** (am - 1) if am > 0 else np.zeros_like(w)   # d/dx (x+iy)^m; d/dy = i * that
            q, dq = Q(d[:, 2]), Q.deriv()(d[:, 2])
            if real:
                gx, gy, f = dp.real, -dp.imag, p.real
            else:
                gx, gy, f = dp.imag, dp.real, p.imag
            out.append(np.stack([K * q * gx, K * q * gy, K * dq * f], axis=1))
    return np.stack(out, axis=1)


def sh_colour(mu: np.ndarray, coeffs: np.ndarray, degree: int, campos: np.ndarray):
    """RGB from SH in the viewing direction; returns (rgb clamped at 0, pre-clamp sum, direction, |v|)."""
    v = np.asarray(mu, np.float64) - campos[None, :]
    nv = np.linalg.norm(v, axis=1)
    d = v / nv[:, None]
    K = (degree + 1) ** 2
    k = np.asarray(coeffs, np.float64).reshape(-1, K, 3)
    pre = np.einsum("nk,nkc->nc", sh_basis(d, degree), k)
    return np.maximum(pre, 0.0), pre, d, nv


# ---------------------------------------------------------------------------
# projection (Eq. 3)
# ---------------------------------------------------------------------------
def unpack_cov(cov6: np.ndarray) -> np.ndarray:
    c = np.asarray(cov6, np.float64)
    S = np.zeros((c.shape[0], 3, 3))
    for k, (i, j) in enumerate(PACK3):
        S[:, i, j] = c[:, k]
        S[:, j, i] = c[:, k]
    return S


def project(cam: Camera, st: Settings, mu, cov6, opacity, colours) -> Dict[str, np.ndarray]:
    """Per-Gaussian screen-space quantities (fp64)."""
    mu = np.asarray(mu, np.float64)[:, :3]
    R, t = cam.R, cam.t
    xc = mu @ R.T + t
    x, y, z = xc[:, 0], xc[:, 1], xc[:, 2]
    n = mu.shape[0]
    visible = z > cam.z_near
    zs = np.where(visible, z, 1.0)
    J = np.zeros((n, 2, 3))
    J[:, 0, 0] = cam.fx / zs
    J[:, 0, 2] = -cam.fx * x / zs ** 2
    J[:, 1, 1] = cam.fy / zs
    J[:, 1, 2] = -cam.fy * y / zs ** 2
    T = J @ R                                            # J W, W = R
    S2 = T @ unpack_cov(cov6) @ np.transpose(T, (0, 2, 1))
    A = S2[:, 0, 0] + st.lowpass
    B = S2[:, 0, 1]
    C = S2[:, 1, 1] + st.lowpass
    det = A * C - B * B
    visible &= det > 0
    dets = np.where(visible, det, 1.0)
    conic = np.stack([C / dets, -B / dets, A / dets], axis=1)
    mean2d = np.stack([cam.fx * x / zs + cam.cx, cam.fy * y / zs + cam.cy], axis=1)
    if st.sh_degree < 0:
        rgb = np.asarray(colours, np.float64).reshape(n, 3).copy()
        pre = rgb.copy()
    else:
        rgb, pre, _, _ = sh_colour(mu, colours, st.sh_degree, cam.centre)
    return dict(visible=visible, depth=z, mean2d=mean2d, conic=conic, cov2d=np.stack([A, B, C], axis=1),
                opacity=np.asarray(opacity, np.float64).reshape(n), rgb=rgb, rgb_pre=pre, xc=xc, J=J, T=T)


# ---------------------------------------------------------------------------
# compositing (Eq. 4)
# ---------------------------------------------------------------------------
def _depth_order(pr) -> np.ndarray:
    idx = np.flatnonzero(pr["visible"])
    return idx[np.lexsort((idx, pr["depth"][idx]))]


def composite_pixel(px: float, py: float, pr, order, st: Settings):
    """One pixel: returns (rgb, T_final, contributors in order, their alphas,
    the transmittance before each, margin_ok, grad_margin_ok).

    A margin counts only where the decision can change the result: Gaussians
    up to the one that ends the blending, the 3-sigma edge only where alpha
    there would still reach alpha_min."""
    m = pr["mean2d"][order]
    q = pr["conic"][order]
    o = pr["opacity"][order]
    dx, dy = px - m[:, 0], py - m[:, 1]
    d2 = q[:, 0] * dx * dx + 2.0 * q[:, 1] * dx * dy + q[:, 2] * dy * dy
    cover = d2 <= SUPPORT_D2
    a_raw = o * np.exp(-0.5 * d2)
    a = np.minimum(a_raw, st.alpha_max)
    blend = cover & (a >= st.alpha_min)
    pos = np.flatnonzero(blend)                           # positions in `order` that blend
    ab = a[pos]
    Tb = np.concatenate([[1.0], np.cumprod(1.0 - ab)])   # T before each, then after the last
    n_eval = len(order)
    k = len(pos)
    if st.t_stop > 0:
        stop = np.flatnonzero(Tb[1:] < st.t_stop)
        if stop.size:
            k = int(stop[0])
            n_eval = int(pos[k]) + 1                      # the ending Gaussian was evaluated
    ev = slice(0, n_eval)
    ok = True
    edge_matters = o[ev] * math.exp(-0.5 * SUPPORT_D2) >= st.alpha_min * (1.0 - REL_MARGIN)
    if np.any((np.abs(d2[ev] - SUPPORT_D2) < D2_MARGIN) & edge_matters):
        ok = False
    if st.alpha_min > 0 and np.any(cover[ev] & (np.abs(a[ev] - st.alpha_min) < REL_MARGIN * st.alpha_min)):
        ok = False
    if st.t_stop > 0 and np.any(np.abs(Tb[1:min(k + 1, len(pos)) + 1] - st.t_stop) < REL_MARGIN * st.t_stop):
        ok = False
    sel = pos[:k]
    idx = order[sel]
    a_k, Tb_k = ab[:k], Tb[:k + 1]
    z = pr["depth"][idx]
    if z.size > 1 and np.any(np.diff(z) < DEPTH_MARGIN * z[1:]):
        ok = False
    gok = not np.any(np.abs(a_raw[sel] - st.alpha_max) < REL_MARGIN * st.alpha_max)
    rgb = (pr["rgb"][idx] * (a_k * Tb_k[:-1])[:, None]).sum(axis=0) + Tb_k[-1] * np.asarray(st.background, np.float64)
    return rgb, Tb_k[-1], idx, a_k, Tb_k[:-1], ok, ok and gok


def _blend(px: float, py: float, pr, order, st: Settings, flip_cover=None, flip_alpha_min=None, stop_at=None,
           swap=None):
    """Colour and final transmittance of one pixel, decided as in
    composite_pixel except for one forced change: the 3-sigma test
    (flip_cover) or the alpha_min test (flip_alpha_min) of the Gaussian at that
    position of ``order`` taken the other way; blending that stops after
    exactly ``stop_at`` blending Gaussians; or the Gaussians at the two
    positions ``swap`` of ``order`` exchanged."""
    if swap is not None:
        order = np.array(order, copy=True)
        order[swap[0]], order[swap[1]] = order[swap[1]], order[swap[0]]
    m = pr["mean2d"][order]
    q = pr["conic"][order]
    o = pr["opacity"][order]
    dx, dy = px - m[:, 0], py - m[:, 1]
    d2 = q[:, 0] * dx * dx + 2.0 * q[:, 1] * dx * dy + q[:, 2] * dy * dy
    cover = d2 <= SUPPORT_D2
    a = np.minimum(o * np.exp(-0.5 * d2), st.alpha_max)
    passes = a >= st.alpha_min
    if flip_cover is not None:
        cover[flip_cover] = not cover[flip_cover]
    if flip_alpha_min is not None:
        passes[flip_alpha_min] = not passes[flip_alpha_min]
    pos = np.flatnonzero(cover & passes)
    ab = a[pos]
    Tb = np.concatenate([[1.0], np.cumprod(1.0 - ab)])
    k = len(pos)
    if stop_at is not None:
        k = min(stop_at, len(pos))
    elif st.t_stop > 0:
        stop = np.flatnonzero(Tb[1:] < st.t_stop)
        if stop.size:
            k = int(stop[0])
    idx = order[pos[:k]]
    rgb = (pr["rgb"][idx] * (ab[:k] * Tb[:k])[:, None]).sum(axis=0) + Tb[k] * np.asarray(st.background, np.float64)
    return rgb, Tb[k]


def pixel_flip_bound(px: float, py: float, pr, order, st: Settings):
    """How far fp32 rounding can move one pixel: the sum, over the decisions
    that composite_pixel finds within their margins, of the change in colour
    (3) and final transmittance that taking that one decision the other way
    makes (each computed by _blend).  Zero for a pixel clear of every margin.
    Two decisions taken the other way together change the pixel by the sum of
    their changes up to a product of two of the (small) alphas involved."""
    base_rgb, base_T, _, _, _, ok, _ = composite_pixel(px, py, pr, order, st)
    if ok:
        return np.zeros(3), 0.0
    m = pr["mean2d"][order]
    q = pr["conic"][order]
    o = pr["opacity"][order]
    dx, dy = px - m[:, 0], py - m[:, 1]
    d2 = q[:, 0] * dx * dx + 2.0 * q[:, 1] * dx * dy + q[:, 2] * dy * dy
    cover = d2 <= SUPPORT_D2
    a = np.minimum(o * np.exp(-0.5 * d2), st.alpha_max)
    pos = np.flatnonzero(cover & (a >= st.alpha_min))
    Tb = np.concatenate([[1.0], np.cumprod(1.0 - a[pos])])
    k, n_eval = len(pos), len(order)
    if st.t_stop > 0:
        stop = np.flatnonzero(Tb[1:] < st.t_stop)
        if stop.size:
            k = int(stop[0])
            n_eval = int(pos[k]) + 1
    alts = []
    edge_matters = o * math.exp(-0.5 * SUPPORT_D2) >= st.alpha_min * (1.0 - REL_MARGIN)
    for g in np.flatnonzero((np.abs(d2[:n_eval] - SUPPORT_D2) < D2_MARGIN) & edge_matters[:n_eval]):
        alts.append(_blend(px, py, pr, order, st, flip_cover=int(g)))
    if st.alpha_min > 0:
        near = cover[:n_eval] & (np.abs(a[:n_eval] - st.alpha_min) < REL_MARGIN * st.alpha_min)
        for g in np.flatnonzero(near):
            alts.append(_blend(px, py, pr, order, st, flip_alpha_min=int(g)))
    if st.t_stop > 0:
        for i in range(min(k + 1, len(pos))):
            if abs(Tb[i + 1] - st.t_stop) < REL_MARGIN * st.t_stop:
                # stopping before blending Gaussian i, or blending it too
                alts.append(_blend(px, py, pr, order, st, stop_at=i if i < k else k + 1))
    z = pr["depth"][order[pos[:k]]]
    for i in np.flatnonzero(np.diff(z) < DEPTH_MARGIN * z[1:]) if z.size > 1 else []:
        alts.append(_blend(px, py, pr, order, st, swap=(int(pos[i]), int(pos[i + 1]))))
    rgb_b, T_b = np.zeros(3), 0.0
    for rgb, T in alts:
        rgb_b += np.abs(rgb - base_rgb)
        T_b += abs(T - base_T)
    return rgb_b, T_b


def render_flip_bounds(cam: Camera, st: Settings, mu, cov6, opacity, colours, pixels: np.ndarray):
    """pixel_flip_bound for the listed pixels (k x 2 integer (column, row)):
    (k x 3 colour bounds, k transmittance bounds)."""
    pr = project(cam, st, mu, cov6, opacity, colours)
    order = _depth_order(pr)
    rgb = np.zeros((len(pixels), 3))
    T = np.zeros(len(pixels))
    for k, (i, j) in enumerate(np.asarray(pixels)):
        rgb[k], T[k] = pixel_flip_bound(i + 0.5, j + 0.5, pr, order, st)
    return rgb, T


def render_pixels(cam: Camera, st: Settings, mu, cov6, opacity, colours, pixels: np.ndarray):
    """Colour (k x 3), final transmittance (k) and margin flags (k) of the
    listed pixels (k x 2 integer (column, row))."""
    pr = project(cam, st, mu, cov6, opacity, colours)
    order = _depth_order(pr)
    out = np.zeros((len(pixels), 3))
    T = np.zeros(len(pixels))
    ok = np.zeros(len(pixels), bool)
    for k, (i, j) in enumerate(np.asarray(pixels)):
        c, t, _, _, _, o, _ = composite_pixel(i + 0.5, j + 0.5, pr, order, st)
        out[k], T[k], ok[k] = c, t, o
    return out, T, ok


def render(cam: Camera, st: Settings, mu, cov6, opacity, colours):
    """Whole image: (3 x H x W colour, H x W final transmittance, H x W margin flags)."""
    jj, ii = np.mgrid[0:cam.height, 0:cam.width]
    pix = np.stack([ii.reshape(-1), jj.reshape(-1)], axis=1)
    c, T, ok = render_pixels(cam, st, mu, cov6, opacity, colours, pix)
    H, W = cam.height, cam.width
    return c.T.reshape(3, H, W), T.reshape(H, W), ok.reshape(H, W)


def back_to_front(rgbs: np.ndarray, alphas: np.ndarray, background) -> np.ndarray:
    """Painter's recursion C <- c_i a_i + (1 - a_i) C from the background,
    farthest first: the same value as Eq. 4's front-to-back sum."""
    C = np.asarray(background, np.float64).copy()
    for c, a in zip(rgbs[::-1], alphas[::-1]):
        C = c * a + (1.0 - a) * C
    return C


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------
def render_backward(cam: Camera, st: Settings, mu, cov6, opacity, colours, grad_image: np.ndarray):
    """Gradients of L = sum(grad_image * image) (grad_image 3 x H x W) w.r.t.
    mu (n x 3), the packed covariance (n x 6), the opacity (n) and the colour
    inputs (n x 3 RGB, or n x 3(D+1)^2 SH coefficients), plus the per-pixel
    gradient margin flags (H x W).  Decisions (culling, support, alpha_min,
    termination) are held fixed; where a > alpha_max the clamp makes the
    alpha's derivative zero."""
    mu = np.asarray(mu, np.float64)[:, :3]
    n = mu.shape[0]
    pr = project(cam, st, mu, cov6, opacity, colours)
    order = _depth_order(pr)
    g_mean2d = np.zeros((n, 2))
    g_conic = np.zeros((n, 3))
    g_op = np.zeros(n)
    g_rgb = np.zeros((n, 3))
    bg = np.asarray(st.background, np.float64)
    gok = np.ones((cam.height, cam.width), bool)
    for j in range(cam.height):
        for i in range(cam.width):
            if not np.any(grad_image[:, j, i]):
                continue                                          # contributes nothing
            px, py = i + 0.5, j + 0.5
            _, Tf, idx, a, Tb, _, ok = composite_pixel(px, py, pr, order, st)
            gok[j, i] = ok
            if idx.size == 0:
                continue
            g = grad_image[:, j, i].astype(np.float64)
            gc = pr["rgb"][idx] @ g                               # g . c_i
            g_rgb[idx] += np.outer(a * Tb, g)
            # everything behind i: sum_{k>i} (g.c_k) a_k T_k + T_final (g.bg)
            term = gc * a * Tb
            behind = np.concatenate([np.cumsum(term[::-1])[::-1][1:], [0.0]]) + Tf * (g @ bg)
            g_a = Tb * gc - behind / (1.0 - a)
            m = pr["mean2d"][idx]
            q = pr["conic"][idx]
            dx, dy = px - m[:, 0], py - m[:, 1]
            d2 = q[:, 0] * dx * dx + 2.0 * q[:, 1] * dx * dy + q[:, 2] * dy * dy
            G = np.exp(-0.5 * d2)
            o = pr["opacity"][idx]
            live = o * G <= st.alpha_max                          # clamp inactive
            g_a = np.where(live, g_a, 0.0)
            g_op[idx] += g_a * G
            g_d2 = -0.5 * g_a * o * G
            g_conic[idx] += np.stack([g_d2 * dx * dx, g_d2 * 2.0 * dx * dy, g_d2 * dy * dy], axis=1)
            # d d2 / d mean2d = -2 (conic delta)
            g_mean2d[idx, 0] += g_d2 * -2.0 * (q[:, 0] * dx + q[:, 1] * dy)
            g_mean2d[idx, 1] += g_d2 * -2.0 * (q[:, 1] * dx + q[:, 2] * dy)
    g_mu, g_cov, g_col = project_backward(cam, st, mu, cov6, colours, pr, g_mean2d, g_conic, g_rgb)
    return dict(mu=g_mu, cov=g_cov, opacity=g_op, colours=g_col, mean2d=g_mean2d, conic=g_conic, rgb=g_rgb,
                grad_ok=gok)


def project_backward(cam: Camera, st: Settings, mu, cov6, colours, pr, g_mean2d, g_conic, g_rgb):
    """Chain rule through ``project``: screen-space gradients -> (mu, packed
    covariance, colour inputs).  Culled Gaussians get zero."""
    n = mu.shape[0]
    vis = pr["visible"]
    R = cam.R
    x, y, z = pr["xc"][:, 0], pr["xc"][:, 1], np.where(vis, pr["xc"][:, 2], 1.0)
    fx, fy = cam.fx, cam.fy
    A, B, C = pr["cov2d"][:, 0], pr["cov2d"][:, 1], pr["cov2d"][:, 2]
    det = np.where(vis, A * C - B * B, 1.0)
    ga, gb, gc = g_conic[:, 0], g_conic[:, 1], g_conic[:, 2]
    # conic (a, b, c) = (C, -B, A) / det, det = A C - B^2
    ddet_A, ddet_B, ddet_C = C, -2.0 * B, A
    inv2 = 1.0 / det ** 2
    gA = ga * (-C * ddet_A * inv2) + gb * (B * ddet_A * inv2) + gc * (1.0 / det - A * ddet_A * inv2)
    gB = ga * (-C * ddet_B * inv2) + gb * (-1.0 / det + B * ddet_B * inv2) + gc * (-A * ddet_B * inv2)
    gC = ga * (1.0 / det - C * ddet_C * inv2) + gb * (B * ddet_C * inv2) + gc * (-A * ddet_C * inv2)
    # symmetric full-matrix gradient of Sigma_2D (lowpass is a constant shift)
    G2 = np.zeros((n, 2, 2))
    G2[:, 0, 0], G2[:, 1, 1] = gA, gC
    G2[:, 0, 1] = G2[:, 1, 0] = 0.5 * gB
    T = pr["T"]
    Sig = unpack_cov(cov6)
    G3 = np.transpose(T, (0, 2, 1)) @ G2 @ T                 # dL/dSigma (full, symmetric)
    g_cov = np.stack([G3[:, i, j] * (1.0 if i == j else 2.0) for i, j in PACK3], axis=1)
    gT = 2.0 * G2 @ T @ Sig                                    # dL/d(J W)
    gJ = gT @ R.T
    gxc = np.zeros((n, 3))
    # J entries: J00 = fx/z, J02 = -fx x/z^2, J11 = fy/z, J12 = -fy y/z^2
    gxc[:, 0] += gJ[:, 0, 2] * (-fx / z ** 2)
    gxc[:, 1] += gJ[:, 1, 2] * (-fy / z ** 2)
    gxc[:, 2] += (gJ[:, 0, 0] * (-fx / z ** 2) + gJ[:, 0, 2] * (2.0 * fx * x / z ** 3)
                  + gJ[:, 1, 1] * (-fy / z ** 2) + gJ[:, 1, 2] * (2.0 * fy * y / z ** 3))
    # mean2d = (fx x/z + cx, fy y/z + cy)
    gxc[:, 0] += g_mean2d[:, 0] * fx / z
    gxc[:, 1] += g_mean2d[:, 1] * fy / z
    gxc[:, 2] += -g_mean2d[:, 0] * fx * x / z ** 2 - g_mean2d[:, 1] * fy * y / z ** 2
    g_mu = gxc @ R                                             # x_c = R mu + t
    if st.sh_degree < 0:
        g_col = g_rgb.copy()
    else:
        D = st.sh_degree
        K = (D + 1) ** 2
        _, pre, d, nv = sh_colour(mu, colours, D, cam.centre)
        gpre = np.where(pre >= 0.0, g_rgb, 0.0)
        Y = sh_basis(d, D)
        g_col = np.einsum("nk,nc->nkc", Y, gpre).reshape(n, 3 * K)
        k = np.asarray(colours, np.float64).reshape(n, K, 3)
        gd = np.einsum("nc,nkc,nki->ni", gpre, k, sh_basis_grad(d, D))   # dL/d(direction)
        gv = (gd - d * np.sum(gd * d, axis=1, keepdims=True)) / nv[:, None]
        g_mu = g_mu + gv
    g_mu[~vis] = 0.0
    g_cov[~vis] = 0.0
    g_col[~vis] = 0.0
    return g_mu, g_cov, g_col
