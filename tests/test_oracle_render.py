"""Pins of the projection and compositing oracle (SPIN-4DGS section 3.1,
Eqs. 1, 3, 4).

Against what mathematics fixes, not against the oracle itself: the real
spherical harmonics' orthonormality (exact quadrature), Unsold's theorem and
harmonicity; the projected covariance of an isotropic Gaussian on the optical
axis and, for any Gaussian, the sample covariance of Monte Carlo points pushed
through the exact pinhole map; the 2D Gaussian's integral over the image;
closed forms for one, two and three stacked Gaussians; the painter's
back-to-front recursion; invariance to the input order and to a joint
rotation of scene and camera; and central differences for every gradient.
"""
import math

import numpy as np
import pytest

from oracle import render as rd
from spatiotemporal_neural_field_b200 import synthetic as S


def _cam(spec: S.CameraSpec) -> rd.Camera:
    return rd.Camera(view=np.array(spec.view, np.float64), fx=spec.fx, fy=spec.fy, cx=spec.cx, cy=spec.cy,
                     width=spec.width, height=spec.height, z_near=spec.z_near)


def _axis_cam(w=64, h=48, f=80.0, z_near=0.2):
    """Camera at the origin looking along +z (identity view)."""
    view = np.concatenate([np.eye(3), np.zeros((3, 1))], axis=1)
    return rd.Camera(view=view, fx=f, fy=f, cx=w / 2, cy=h / 2, width=w, height=h, z_near=z_near)


def _iso(n, s):
    c = np.zeros((n, 6))
    c[:, 0] = c[:, 3] = c[:, 5] = s * s
    return c


# ---------------------------------------------------------------------------
# spherical harmonics
# ---------------------------------------------------------------------------
def _sphere_quadrature(nz=16, nphi=32):
    z, wz = np.polynomial.legendre.leggauss(nz)
    phi = 2 * np.pi * np.arange(nphi) / nphi
    Z, P = np.meshgrid(z, phi, indexing="ij")
    r = np.sqrt(1 - Z ** 2)
    d = np.stack([r * np.cos(P), r * np.sin(P), Z], axis=-1).reshape(-1, 3)
    w = (wz[:, None] * np.full(nphi, 2 * np.pi / nphi)[None, :]).reshape(-1)
    return d, w


def test_sh_orthonormal():
    d, w = _sphere_quadrature()
    Y = rd.sh_basis(d, 3)
    gram = (Y * w[:, None]).T @ Y
    np.testing.assert_allclose(gram, np.eye(16), atol=1e-13)


def test_sh_closed_values_and_unsold():
    d = np.array([[0.0, 0.0, 1.0], [1.0, 0.0, 0.0], [0.0, 1.0, 0.0]])
    Y = rd.sh_basis(d, 3)
    assert abs(Y[0, 0] - 1 / (2 * math.sqrt(math.pi))) < 1e-15
    c1 = math.sqrt(3 / (4 * math.pi))
    # degree 1: (y, z, x) scaled by sqrt(3/4pi) in index order m = -1, 0, 1
    np.testing.assert_allclose(Y[0, 1:4], [0, c1, 0], atol=1e-15)
    np.testing.assert_allclose(Y[1, 1:4], [0, 0, c1], atol=1e-15)
    np.testing.assert_allclose(Y[2, 1:4], [c1, 0, 0], atol=1e-15)
    # Unsold: sum_m Y_lm(d)^2 = (2l+1)/(4pi) for every unit d
    rng = np.random.default_rng(0)
    v = rng.normal(size=(50, 3))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    Y = rd.sh_basis(v, 3)
    for l in range(4):
        np.testing.assert_allclose((Y[:, l * l:(l + 1) ** 2] ** 2).sum(axis=1), (2 * l + 1) / (4 * math.pi),
                                   rtol=1e-13)


def test_sh_harmonic():
    """r^l Y_lm(v/r) is a harmonic polynomial: its Laplacian vanishes."""
    rng = np.random.default_rng(1)
    v = rng.normal(size=(6, 3))
    h = 1e-3

    def f(p):
        r = np.linalg.norm(p, axis=1)
        Y = rd.sh_basis(p / r[:, None], 3)
        ls = np.array([l for l in range(4) for _ in range(2 * l + 1)])
        return Y * r[:, None] ** ls[None, :]

    lap = -6 * f(v)
    for k in range(3):
        e = np.zeros(3)
        e[k] = h
        lap += f(v + e) + f(v - e)
    lap /= h * h
    # the second difference of a cubic is exact up to rounding
    assert np.abs(lap).max() < 1e-7 * np.abs(f(v)).max()


def test_sh_gradient_is_tangent_derivative():
    rng = np.random.default_rng(2)
    d = rng.normal(size=(10, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    G = rd.sh_basis_grad(d, 3)
    t = rng.normal(size=(10, 3))
    t -= d * np.sum(t * d, axis=1, keepdims=True)         # tangent direction
    h = 1e-6

    def on_sphere(e):
        p = d + e
        return rd.sh_basis(p / np.linalg.norm(p, axis=1, keepdims=True), 3)

    fd = (on_sphere(h * t) - on_sphere(-h * t)) / (2 * h)
    np.testing.assert_allclose(np.einsum("nki,ni->nk", G, t), fd, atol=1e-8)


# ---------------------------------------------------------------------------
# projection
# ---------------------------------------------------------------------------
def test_isotropic_on_axis():
    cam = _axis_cam()
    st = rd.Settings(sh_degree=-1, lowpass=0.3)
    mu = np.array([[0.0, 0.0, 2.0]])
    pr = rd.project(cam, st, mu, _iso(1, 0.05), [0.5], [[1, 1, 1]])
    s2 = (80.0 * 0.05 / 2.0) ** 2
    np.testing.assert_allclose(pr["cov2d"][0], [s2 + 0.3, 0.0, s2 + 0.3], atol=1e-12)
    np.testing.assert_allclose(pr["mean2d"][0], [32.0, 24.0], atol=1e-12)
    np.testing.assert_allclose(pr["conic"][0], [1 / (s2 + 0.3), 0.0, 1 / (s2 + 0.3)], rtol=1e-12)


def test_projection_matches_monte_carlo():
    """Eq. 3 is the first-order covariance of the projected points."""
    cam = _cam(S.orbit_camera(320, 240, focal=300.0))
    st = rd.Settings(sh_degree=-1, lowpass=0.0)
    rng = np.random.default_rng(3)
    mu = np.array([[0.3, -0.2, 0.4]])
    sig = np.array([0.004, 0.002, 0.001])
    cov = S.random_spd(1, sig[None, :], rng)
    pr = rd.project(cam, st, mu, cov, [0.5], [[1, 1, 1]])
    Sig = rd.unpack_cov(cov)[0]
    pts = rng.multivariate_normal(mu[0], Sig, size=400_000)
    xc = pts @ cam.R.T + cam.t
    uv = np.stack([cam.fx * xc[:, 0] / xc[:, 2] + cam.cx, cam.fy * xc[:, 1] / xc[:, 2] + cam.cy], axis=1)
    emp = np.cov(uv.T)
    A, B, C = pr["cov2d"][0]
    np.testing.assert_allclose([emp[0, 0], emp[0, 1], emp[1, 1]], [A, B, C], rtol=1.5e-2, atol=2e-2 * max(A, C))
    np.testing.assert_allclose(uv.mean(axis=0), pr["mean2d"][0], atol=0.01)


def test_near_plane_and_behind_are_culled():
    cam = _axis_cam(z_near=0.5)
    st = rd.Settings(sh_degree=-1)
    mu = np.array([[0.0, 0.0, 0.49], [0.0, 0.0, -3.0], [0.0, 0.0, 0.51]])
    pr = rd.project(cam, st, mu, _iso(3, 0.01), [0.5] * 3, np.ones((3, 3)))
    assert list(pr["visible"]) == [False, False, True]


def test_joint_rotation_invariance():
    rng = np.random.default_rng(4)
    spec = S.orbit_camera(48, 32, focal=40.0)
    cam = _cam(spec)
    sc = S.render_scene(60, seed=4, positions=rng.uniform(-0.6, 0.6, size=(60, 3)).astype(np.float32),
                        sh_degree=2, scale_factor=1.0)
    st = rd.Settings(sh_degree=2)
    img, T, _ = rd.render(cam, st, sc["mu"], sc["cov"], sc["opacity"], sc["colours"])
    # rotate the world by Q: mu -> Q mu, Sigma -> Q Sigma Q^T, view R -> R Q^T.
    # SH colour is view-dependent through the world direction, so rotate its
    # argument too by using degree 0 only for this check
    Q, _ = np.linalg.qr(rng.normal(size=(3, 3)))
    if np.linalg.det(Q) < 0:
        Q[:, 0] = -Q[:, 0]
    st0 = rd.Settings(sh_degree=0)
    col0 = sc["colours"].reshape(60, 9, 3)[:, :1, :].reshape(60, 3)
    img0, T0, _ = rd.render(cam, st0, sc["mu"], sc["cov"], sc["opacity"], col0)
    mu2 = sc["mu"].astype(np.float64) @ Q.T
    Sg = Q @ rd.unpack_cov(sc["cov"]) @ Q.T
    cov2 = np.stack([Sg[:, i, j] for i, j in rd.PACK3], axis=1)
    view2 = np.concatenate([cam.R @ Q.T, cam.t[:, None]], axis=1)
    cam2 = rd.Camera(view=view2, fx=cam.fx, fy=cam.fy, cx=cam.cx, cy=cam.cy, width=cam.width, height=cam.height)
    img2, T2, _ = rd.render(cam2, st0, mu2, cov2, sc["opacity"], col0)
    np.testing.assert_allclose(img2, img0, atol=1e-10)
    np.testing.assert_allclose(T2, T0, atol=1e-12)
    assert img.shape == (3, 32, 48)


# ---------------------------------------------------------------------------
# compositing
# ---------------------------------------------------------------------------
def test_single_gaussian_at_its_centre():
    cam = _axis_cam()
    st = rd.Settings(sh_degree=-1, background=np.array([0.2, 0.3, 0.4]))
    # mean exactly on pixel (10, 7)'s sample point (10.5, 7.5)
    z = 2.0
    mu = np.array([[(10.5 - 32) * z / 80, (7.5 - 24) * z / 80, z]])
    c = np.array([[0.9, 0.5, 0.1]])
    for o in (0.3, 1.0):
        img, T, ok = rd.render(cam, st, mu, _iso(1, 0.02), [o], c)
        a = min(o, 0.99)
        np.testing.assert_allclose(img[:, 7, 10], c[0] * a + (1 - a) * st.background, rtol=1e-13)
        assert abs(T[7, 10] - (1 - a)) < 1e-14
        assert ok[7, 10]


def test_integral_of_one_gaussian():
    """sum over pixels of alpha = o * 2 pi sqrt(det Sigma_2D) * (1 - e^-4.5)."""
    cam = _axis_cam(w=96, h=96, f=100.0)
    st = rd.Settings(sh_degree=-1, lowpass=0.3, alpha_min=0.0, t_stop=0.0)
    rng = np.random.default_rng(5)
    cov = S.random_spd(1, np.array([[0.16, 0.1, 0.05]]), rng)
    mu = np.array([[0.03, -0.02, 2.5]])
    o = 0.5
    img, T, _ = rd.render(cam, st, mu, cov, [o], [[1, 1, 1]])
    pr = rd.project(cam, st, mu, cov, [o], [[1, 1, 1]])
    A, B, C = pr["cov2d"][0]
    want = o * 2 * math.pi * math.sqrt(A * C - B * B) * (1 - math.exp(-4.5))
    assert 3 * math.sqrt(max(A, C)) < 40             # the 3-sigma box lies inside the image
    np.testing.assert_allclose((1 - T).sum(), want, rtol=5e-3)
    np.testing.assert_allclose(img[0], 1 - T, atol=1e-14)


def _stack(alphas_o, depths, colours, st, cam=None):
    """Gaussians centred on pixel (10, 7) of the axis camera, tiny on screen."""
    cam = cam or _axis_cam()
    mus = np.array([[(10.5 - 32) * z / 80, (7.5 - 24) * z / 80, z] for z in depths])
    return rd.render(cam, st, mus, _iso(len(depths), 1e-3), alphas_o, colours)


def test_two_gaussians_closed_form_and_order():
    st = rd.Settings(sh_degree=-1, background=np.zeros(3))
    c = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 0.0]])
    img, _, _ = _stack([0.6, 0.5], [2.0, 3.0], c, st)
    np.testing.assert_allclose(img[:, 7, 10], 0.6 * c[0] + 0.5 * 0.4 * c[1], rtol=1e-13)
    # depth decides, not input order
    img2, _, _ = _stack([0.5, 0.6], [3.0, 2.0], c[::-1], st)
    np.testing.assert_allclose(img2[:, 7, 10], img[:, 7, 10], rtol=1e-13)


def test_termination_closed_form():
    st = rd.Settings(sh_degree=-1, alpha_max=0.99, t_stop=1e-4, background=np.array([1.0, 1.0, 1.0]))
    c = np.eye(3)
    img, T, _ = _stack([0.98, 0.98, 0.98], [2.0, 2.5, 3.0], c, st)
    # T after two is 4e-4 >= 1e-4; the third would give 8e-6 < 1e-4: it is not blended
    np.testing.assert_allclose(T[7, 10], 0.02 * 0.02, rtol=1e-12)
    np.testing.assert_allclose(img[:, 7, 10], np.array([0.98, 0.98 * 0.02, 0.0]) + 4e-4, rtol=1e-12)
    st0 = rd.Settings(sh_degree=-1, alpha_max=0.99, t_stop=0.0, background=np.array([1.0, 1.0, 1.0]))
    img0, T0, _ = _stack([0.98, 0.98, 0.98], [2.0, 2.5, 3.0], c, st0)
    np.testing.assert_allclose(T0[7, 10], 0.02 ** 3, rtol=1e-12)


def test_front_to_back_equals_painter():
    rng = np.random.default_rng(6)
    spec = S.orbit_camera(40, 30, focal=35.0)
    cam = _cam(spec)
    n = 80
    sc = S.render_scene(n, seed=6, positions=rng.uniform(-0.5, 0.5, size=(n, 3)).astype(np.float32),
                        sh_degree=-1, scale_factor=1.5)
    st = rd.Settings(sh_degree=-1, alpha_min=0.0, t_stop=0.0, background=np.array([0.1, 0.2, 0.3]))
    pr = rd.project(cam, st, sc["mu"], sc["cov"], sc["opacity"], sc["colours"])
    order = rd._depth_order(pr)
    checked = 0
    for (i, j) in [(5, 5), (20, 15), (33, 8), (12, 25)]:
        rgb, T, idx, a, Tb, _, _ = rd.composite_pixel(i + 0.5, j + 0.5, pr, order, st)
        assert len(idx) == len(a)
        want = rd.back_to_front(pr["rgb"][idx], a, st.background)
        np.testing.assert_allclose(rgb, want, rtol=1e-12, atol=1e-14)
        checked += len(idx) > 2
    assert checked >= 2


def test_eq1_density_from_covariance_inverse():
    """G_2D(x) = exp(-1/2 (x-mu)^T Sigma_2D^-1 (x-mu)) with Sigma_2D inverted by numpy."""
    cam = _axis_cam()
    st = rd.Settings(sh_degree=-1, alpha_min=0.0, t_stop=0.0, alpha_max=0.99)
    rng = np.random.default_rng(7)
    cov = S.random_spd(1, np.array([[0.06, 0.03, 0.02]]), rng)
    mu = np.array([[0.05, 0.02, 2.0]])
    o = 0.7
    img, T, _ = rd.render(cam, st, mu, cov, [o], [[1, 1, 1]])
    pr = rd.project(cam, st, mu, cov, [o], [[1, 1, 1]])
    A, B, C = pr["cov2d"][0]
    Si = np.linalg.inv(np.array([[A, B], [B, C]]))
    jj, ii = np.mgrid[0:cam.height, 0:cam.width]
    d = np.stack([ii + 0.5 - pr["mean2d"][0, 0], jj + 0.5 - pr["mean2d"][0, 1]], axis=-1)
    q = np.einsum("hwi,ij,hwj->hw", d, Si, d)
    want = np.where(q <= 9.0, np.minimum(o * np.exp(-0.5 * q), 0.99), 0.0)
    np.testing.assert_allclose(1 - T, want, atol=1e-13)


def test_input_permutation_invariance():
    rng = np.random.default_rng(8)
    cam = _cam(S.orbit_camera(40, 30, focal=35.0))
    n = 100
    sc = S.render_scene(n, seed=8, positions=rng.uniform(-0.5, 0.5, size=(n, 3)).astype(np.float32),
                        sh_degree=1, scale_factor=1.5)
    st = rd.Settings(sh_degree=1)
    img, T, ok = rd.render(cam, st, sc["mu"], sc["cov"], sc["opacity"], sc["colours"])
    p = rng.permutation(n)
    img2, T2, _ = rd.render(cam, st, sc["mu"][p], sc["cov"][p], sc["opacity"][p], sc["colours"][p])
    np.testing.assert_allclose(img2[:, ok], img[:, ok], atol=1e-14)


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------
def _loss(cam, st, sc, g):
    img, _, _ = rd.render(cam, st, sc["mu"], sc["cov"], sc["opacity"], sc["colours"])
    return float(np.sum(g * img))


@pytest.mark.parametrize("deg", [-1, 3])
def test_backward_matches_central_differences(deg):
    rng = np.random.default_rng(9 + deg)
    cam = _cam(S.orbit_camera(24, 18, focal=22.0))
    n = 14
    sc = S.render_scene(n, seed=9, positions=rng.uniform(-0.4, 0.4, size=(n, 3)).astype(np.float32),
                        sh_degree=deg, scale_factor=1.2, opacity_lo=0.2)
    sc = {k: v.astype(np.float64) for k, v in sc.items()}
    st = rd.Settings(sh_degree=deg, alpha_max=0.99, background=np.array([0.3, 0.1, 0.2]))
    g = S.image_grads(S.orbit_camera(24, 18), seed=9).astype(np.float64)
    grads = rd.render_backward(cam, st, sc["mu"], sc["cov"], sc["opacity"], sc["colours"], g)
    # a decision that flipped under +-h would show as a wildly wrong difference below
    assert grads["grad_ok"].mean() > 0.9
    h = 1e-6
    for key, gk in (("mu", "mu"), ("cov", "cov"), ("opacity", "opacity"), ("colours", "colours")):
        x = sc[key]
        flat = x.reshape(-1)
        got = grads[gk].reshape(-1)
        for p in rng.choice(flat.size, min(flat.size, 25), replace=False):
            old = flat[p]
            flat[p] = old + h
            lp = _loss(cam, st, sc, g)
            flat[p] = old - h
            lm = _loss(cam, st, sc, g)
            flat[p] = old
            fd = (lp - lm) / (2 * h)
            assert abs(got[p] - fd) <= 1e-6 * max(1.0, abs(fd)), (key, p, got[p], fd)


def test_view_direction_runs_from_the_camera_centre():
    """The camera centre is the point the view maps to the camera-space
    origin; a degree-1 SH colour is sqrt(3/4pi) (k_y d_y + k_z d_z + k_x d_x)
    in the direction from that centre to the Gaussian."""
    spec = S.orbit_camera(32, 24, focal=30.0, azimuth_deg=40.0, elevation_deg=25.0)
    cam = _cam(spec)
    np.testing.assert_allclose(cam.R @ cam.centre + cam.t, 0.0, atol=1e-6)
    eye = np.array([2.8 * math.cos(math.radians(25)) * math.sin(math.radians(40)), -2.8 * math.sin(math.radians(25)),
                    -2.8 * math.cos(math.radians(25)) * math.cos(math.radians(40))])
    np.testing.assert_allclose(cam.centre, eye, atol=1e-5)
    mu = np.array([[0.1, -0.2, 0.05]])
    k = np.zeros((1, 4, 3))
    k[0, 1:4, 0] = [0.3, -0.2, 0.5]            # channel 0: Y_1,-1 (y), Y_1,0 (z), Y_1,1 (x)
    k[0, 0, 1] = 1.0                           # channel 1: constant
    rgb, pre, d, _ = rd.sh_colour(mu, k.reshape(1, 12), 1, cam.centre)
    v = mu[0] - eye
    v /= np.linalg.norm(v)
    c1 = math.sqrt(3 / (4 * math.pi))
    # the view matrix is stored in fp32, so the centre agrees with the exact eye to ~1e-7
    np.testing.assert_allclose(pre[0, 0], c1 * (0.3 * v[1] - 0.2 * v[2] + 0.5 * v[0]), rtol=1e-6)
    np.testing.assert_allclose(pre[0, 1], 1 / (2 * math.sqrt(math.pi)), rtol=1e-12)


def test_backward_with_clamped_alpha_matches_central_differences():
    """Opaque Gaussians (o = 1) reach alpha_max at their centres; where the
    clamp holds, alpha does not move with o, the mean or Sigma."""
    rng = np.random.default_rng(41)
    cam = _cam(S.orbit_camera(20, 16, focal=18.0))
    n = 10
    sc = S.render_scene(n, seed=41, positions=rng.uniform(-0.35, 0.35, size=(n, 3)).astype(np.float32),
                        sh_degree=-1, scale_factor=1.5)
    sc = {k: v.astype(np.float64) for k, v in sc.items()}
    sc["opacity"][:] = 1.0
    st = rd.Settings(sh_degree=-1, alpha_max=0.99, t_stop=0.0, background=np.array([0.2, 0.5, 0.1]))
    g = S.image_grads(S.orbit_camera(20, 16), seed=42).astype(np.float64)
    pr = rd.project(cam, st, sc["mu"], sc["cov"], sc["opacity"], sc["colours"])
    order = rd._depth_order(pr)
    clamped = 0
    for j in range(16):
        for i in range(20):
            _, _, idx, a, _, _, _ = rd.composite_pixel(i + 0.5, j + 0.5, pr, order, st)
            clamped += int(np.sum(a == st.alpha_max))
    assert clamped >= 3, "the scene must clamp some alphas"
    grads = rd.render_backward(cam, st, sc["mu"], sc["cov"], sc["opacity"], sc["colours"], g)
    h = 1e-6
    for key in ("opacity", "mu", "cov"):
        flat = sc[key].reshape(-1)
        got = grads[key].reshape(-1)
        for p in range(flat.size):
            old = flat[p]
            flat[p] = old + h
            lp = _loss(cam, st, sc, g)
            flat[p] = old - h
            lm = _loss(cam, st, sc, g)
            flat[p] = old
            fd = (lp - lm) / (2 * h)
            assert abs(got[p] - fd) <= 1e-6 * max(1.0, abs(fd)), (key, p, got[p], fd)


# ---------------------------------------------------------------------------
# the bound on decisions within fp32 reach of their thresholds
# ---------------------------------------------------------------------------
def _pr(means, depths, opacities, rgbs, conic=(1.0, 0.0, 1.0)):
    """A projected scene written out by hand: 2D means, unit conic."""
    n = len(means)
    return dict(mean2d=np.asarray(means, np.float64), conic=np.tile(np.asarray(conic, np.float64), (n, 1)),
                opacity=np.asarray(opacities, np.float64), rgb=np.asarray(rgbs, np.float64),
                depth=np.asarray(depths, np.float64), visible=np.ones(n, bool))


def _bound(pr, st, px=0.5, py=0.5):
    order = rd._depth_order(pr)
    return rd.pixel_flip_bound(px, py, pr, order, st)


def test_flip_bound_is_zero_on_a_clear_pixel():
    st = rd.Settings(sh_degree=-1, background=np.zeros(3))
    pr = _pr([[0.5, 0.5], [1.5, 0.5]], [1.0, 2.0], [0.6, 0.5], [[1, 0, 0], [0, 1, 0]])
    rgb, T = _bound(pr, st)
    assert np.all(rgb == 0.0) and T == 0.0


def test_flip_bound_of_a_gaussian_on_its_three_sigma_edge():
    """d^2 = 9 exactly at the pixel: the Gaussian may be dropped, which
    removes its o e^-4.5 c from the colour and restores the transmittance."""
    st = rd.Settings(sh_degree=-1, background=np.zeros(3))
    o, c = 0.8, np.array([0.2, 0.5, 0.9])
    pr = _pr([[3.5, 0.5]], [1.0], [o], [c])
    rgb, T = _bound(pr, st)
    a = o * math.exp(-4.5)
    assert np.allclose(rgb, a * c, rtol=1e-12) and abs(T - a) < 1e-12


def test_flip_bound_of_a_depth_tie():
    """Two Gaussians at one depth on the pixel: either order may be taken;
    the orders differ by a_1 a_2 (c_1 - c_2) in colour and not at all in the
    transmittance."""
    st = rd.Settings(sh_degree=-1, background=np.zeros(3))
    c1, c2 = np.array([1.0, 0.0, 0.3]), np.array([0.0, 1.0, 0.3])
    pr = _pr([[0.5, 0.5], [0.5, 0.5]], [2.0, 2.0], [0.6, 0.3], [c1, c2])
    rgb, T = _bound(pr, st)
    assert np.allclose(rgb, 0.6 * 0.3 * np.abs(c1 - c2), rtol=1e-12, atol=1e-15) and T < 1e-15


def test_flip_bound_of_the_termination():
    """One Gaussian that leaves the transmittance exactly at t_stop: blending
    may stop before it (background, T = 1) instead."""
    st = rd.Settings(sh_degree=-1, t_stop=0.05, alpha_max=0.99, background=np.array([0.1, 0.2, 0.3]))
    c = np.array([0.9, 0.4, 0.2])
    pr = _pr([[0.5, 0.5]], [1.0], [0.95], [c])
    rgb, T = _bound(pr, st)
    bg = np.array([0.1, 0.2, 0.3])
    base = 0.95 * c + 0.05 * bg
    assert np.allclose(rgb, np.abs(bg - base), rtol=1e-12) and abs(T - 0.95) < 1e-12


def test_flip_bound_of_alpha_min():
    """alpha exactly at alpha_min: the Gaussian may not blend."""
    st = rd.Settings(sh_degree=-1, alpha_min=1 / 255, background=np.zeros(3))
    c = np.array([0.3, 0.6, 0.9])
    pr = _pr([[0.5, 0.5], [0.5, 0.5]], [1.0, 3.0], [1 / 255, 0.5], [c, [1.0, 1.0, 1.0]])
    rgb, T = _bound(pr, st)
    a = 1 / 255
    # with it: a c + (1 - a) 0.5 (1, 1, 1); without it: 0.5 (1, 1, 1)
    assert np.allclose(rgb, np.abs(a * c - a * 0.5), rtol=1e-12) and abs(T - a * 0.5) < 1e-12
