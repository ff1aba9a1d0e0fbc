"""GPU parity of spin4d_render_fwd / spin4d_render_bwd (EWA projection and
alpha compositing, SPIN-4DGS section 3.1 Eqs. 1, 3, 4) against the oracle
(B200 only).

Every pixel is compared.  Those whose decisions the oracle flags as clear of
their thresholds (almost all) are held to the plain tolerance; a flagged one
may take a decision within fp32 reach of its threshold either way, and is
held to the tolerance plus the oracle's bound on what taking each such
decision the other way changes (pixel_flip_bound).  Tile counts are ragged
(image sides not multiples of 16); the full-size case renders the
300k-Gaussian sports frame at 640 x 360 in the same launch the benchmark
times and checks sampled pixels one by one.
"""
import numpy as np
import pytest

from oracle import render as rd
from spatiotemporal_neural_field_b200 import synthetic as S
from tests import tol

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sp():
    from spatiotemporal_neural_field_b200 import spin4d
    return spin4d


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def _ocam(spec):
    return rd.Camera(view=np.array(spec.view, np.float64), fx=spec.fx, fy=spec.fy, cx=spec.cx, cy=spec.cy,
                     width=spec.width, height=spec.height, z_near=spec.z_near)


def _settings(desc_kw):
    return rd.Settings(sh_degree=desc_kw.get("sh_degree", 3), lowpass=desc_kw.get("lowpass", 0.3),
                       alpha_max=desc_kw.get("alpha_max", 0.99), alpha_min=desc_kw.get("alpha_min", 1 / 255),
                       t_stop=desc_kw.get("t_stop", 1e-4),
                       background=np.array(desc_kw.get("background", (0.0, 0.0, 0.0)), np.float64))


def _scene(n, seed, deg, spread=0.7, scale_factor=0.5):
    g = np.random.default_rng(seed)
    pos = g.uniform(-spread, spread, size=(n, 3)).astype(np.float32)
    return S.render_scene(n, seed=seed, positions=pos, sh_degree=deg, scale_factor=scale_factor)


def _gpu_render(sp, spec, sc, desc_kw, max_pairs=None, stride4=False):
    cam = sp.camera_from_spec(spec)
    kw = dict(desc_kw)
    if stride4:
        kw["mean_stride"] = 4
    desc = sp.render_desc(**kw)
    mu = sc["mu"]
    if stride4:
        mu = np.concatenate([mu, np.full((mu.shape[0], 1), 7.0, np.float32)], axis=1)
    args = [dev(mu), dev(sc["cov"]), dev(sc["opacity"]), dev(sc["colours"])]
    N = mu.shape[0]
    state = None
    if max_pairs is not None:
        state = sp.RenderState(N, spec.width, spec.height, max_pairs, "cuda")
    T = torch.empty((spec.height, spec.width), dtype=torch.float32, device="cuda")
    img, state = sp.render(cam, desc, *args, final_T=T, state=state)
    torch.cuda.synchronize()
    return cam, desc, args, host(img), host(T), state


def _check_pixels(got, got_T, want, want_T, ok, name, flip_bounds, pix):
    """got / want: k x 3 colours of the pixels pix (k x 2 column, row), T
    their transmittances; flip_bounds(pixels) -> (k' x 3, k') bounds of the
    flagged ones."""
    tol.absolute(got[ok], want[ok], tol.RENDER_ATOL, name + " clear pixels")
    tol.absolute(got_T[ok], want_T[ok], tol.RENDER_ATOL, name + " clear transmittance")
    flagged = ~ok
    if flagged.any():
        brgb, bT = flip_bounds(pix[flagged])
        tol.absolute_with_bound(got[flagged], want[flagged], brgb, tol.RENDER_ATOL, name + " flagged pixels")
        tol.absolute_with_bound(got_T[flagged], want_T[flagged], bT, tol.RENDER_ATOL,
                                name + " flagged transmittance")


def _check_image(img, T, want_img, want_T, ok, name, spec, kw, sc, min_ok=0.9):
    assert ok.mean() >= min_ok, "%s: only %.3f of pixels clear of thresholds" % (name, ok.mean())
    H, W = T.shape
    jj, ii = np.mgrid[0:H, 0:W]
    pix = np.stack([ii.reshape(-1), jj.reshape(-1)], axis=1)

    def bounds(p):
        return rd.render_flip_bounds(_ocam(spec), _settings(kw), sc["mu"], sc["cov"], sc["opacity"], sc["colours"], p)

    _check_pixels(img.reshape(3, -1).T, T.reshape(-1), want_img.reshape(3, -1).T, want_T.reshape(-1), ok.reshape(-1),
                  name, bounds, pix)


CASES = {
    # name: (n, width, height, desc overrides)
    "rgb": (1500, 120, 88, dict(sh_degree=-1, background=(0.2, 0.4, 0.6))),
    "sh3": (2000, 136, 100, dict(sh_degree=3)),
    "sh1_no_stop": (800, 70, 45, dict(sh_degree=1, t_stop=0.0)),
    "sh2_no_lowpass": (800, 64, 64, dict(sh_degree=2, lowpass=0.0)),
    "sh0_no_alpha_min": (600, 33, 17, dict(sh_degree=0, alpha_min=0.0)),
}


@pytest.mark.parametrize("case", list(CASES))
def test_forward_matches_oracle(sp, case):
    n, w, h, kw = CASES[case]
    deg = kw.get("sh_degree", 3)
    spec = S.orbit_camera(w, h, focal=0.9 * w)
    sc = _scene(n, seed=list(CASES).index(case), deg=deg)
    _, _, _, img, T, state = _gpu_render(sp, spec, sc, kw)
    want_img, want_T, ok = rd.render(_ocam(spec), _settings(kw), sc["mu"], sc["cov"], sc["opacity"], sc["colours"])
    _check_image(img, T, want_img, want_T, ok, case, spec, kw, sc)
    assert 0 < state.pairs_needed() <= state.max_pairs


def test_mean_stride_four_reads_decoder_rows(sp):
    n, w, h, kw = CASES["sh3"]
    spec = S.orbit_camera(w, h, focal=0.9 * w)
    sc = _scene(n, seed=11, deg=3)
    _, _, _, img3, T3, _ = _gpu_render(sp, spec, sc, kw)
    _, _, _, img4, T4, _ = _gpu_render(sp, spec, sc, kw, stride4=True)
    assert np.array_equal(img3, img4) and np.array_equal(T3, T4)


def test_deterministic(sp):
    n, w, h, kw = CASES["sh3"]
    spec = S.orbit_camera(w, h, focal=0.9 * w)
    sc = _scene(n, seed=12, deg=3)
    a = _gpu_render(sp, spec, sc, kw)
    b = _gpu_render(sp, spec, sc, kw)
    assert np.array_equal(a[3], b[3]) and np.array_equal(a[4], b[4])


def test_edge_cases(sp):
    spec = S.orbit_camera(40, 24, focal=36.0)
    bg = (0.25, 0.5, 0.75)
    kw = dict(sh_degree=-1, background=bg)
    # no Gaussians: background everywhere
    empty = dict(mu=np.zeros((0, 3), np.float32), cov=np.zeros((0, 6), np.float32),
                 opacity=np.zeros(0, np.float32), colours=np.zeros((0, 3), np.float32))
    _, _, _, img, T, _ = _gpu_render(sp, spec, empty, kw)
    assert np.all(T == 1.0) and np.allclose(img, np.array(bg, np.float32)[:, None, None])
    # every Gaussian behind the camera: background everywhere
    sc = _scene(50, seed=13, deg=-1)
    view = np.array(spec.view, np.float64)
    eye = -view[:, :3].T @ view[:, 3]                  # the camera looks from eye towards the origin
    sc["mu"] = (2.0 * eye[None, :] + 0.05 * sc["mu"]).astype(np.float32)
    _, _, _, img, T, _ = _gpu_render(sp, spec, sc, kw)
    assert np.all(T == 1.0) and np.allclose(img, np.array(bg, np.float32)[:, None, None])
    # one pixel image, one Gaussian on it
    spec1 = S.orbit_camera(1, 1, focal=2.0)
    one = _scene(1, seed=14, deg=-1)
    one["mu"][:] = 0.0
    one["opacity"][:] = 0.5
    _, _, _, img, T, _ = _gpu_render(sp, spec1, one, kw)
    want_img, want_T, ok = rd.render(_ocam(spec1), _settings(kw), one["mu"], one["cov"], one["opacity"],
                                     one["colours"])
    assert ok.all()
    tol.absolute(img, want_img, 1e-5, "one pixel")
    # largest image side this test affords: a 1 x 2049 strip (many tiles, one row)
    spec_strip = S.orbit_camera(2049, 1, focal=900.0)
    sc = _scene(300, seed=15, deg=-1)
    _, _, _, img, T, _ = _gpu_render(sp, spec_strip, sc, kw)
    want_img, want_T, ok = rd.render(_ocam(spec_strip), _settings(kw), sc["mu"], sc["cov"], sc["opacity"],
                                     sc["colours"])
    _check_image(img, T, want_img, want_T, ok, "strip", spec_strip, kw, sc)


def test_pair_capacity_overflow_is_reported_and_recovered(sp):
    n, w, h, kw = CASES["sh3"]
    spec = S.orbit_camera(w, h, focal=0.9 * w)
    sc = _scene(n, seed=16, deg=3)
    cam = sp.camera_from_spec(spec)
    desc = sp.render_desc(**kw)
    args = [dev(sc["mu"]), dev(sc["cov"]), dev(sc["opacity"]), dev(sc["colours"])]
    small = sp.RenderState(n, w, h, 100, "cuda")
    sp.render_fwd(cam, desc, *args, state=small)
    need = small.pairs_needed()
    assert need > 100 and small.pairs_kept() == 100
    img, state = sp.render(cam, desc, *args, state=small)
    assert state.max_pairs >= need
    _, _, _, ref, _, _ = _gpu_render(sp, spec, sc, kw)
    assert np.array_equal(host(img), ref)


def test_sports_frame_full_size_sampled(sp):
    """The benchmark's frame: 300k Gaussians at 640 x 360, 256 sampled pixels."""
    spec = S.orbit_camera(640, 360)
    sc = S.render_scene(300_000, seed=0)
    kw = dict(sh_degree=3)
    _, _, _, img, T, state = _gpu_render(sp, spec, sc, kw)
    g = np.random.default_rng(17)
    pix = np.stack([g.integers(0, 640, 256), g.integers(0, 360, 256)], axis=1)
    want, want_T, ok = rd.render_pixels(_ocam(spec), _settings(kw), sc["mu"], sc["cov"], sc["opacity"],
                                        sc["colours"], pix)
    got = img[:, pix[:, 1], pix[:, 0]].T
    got_T = T[pix[:, 1], pix[:, 0]]
    # hundreds of Gaussians are evaluated per pixel here, so more pixels hold
    # some decision within fp32 reach of its threshold: every one is checked,
    # the flagged ones against their flip bounds
    assert ok.mean() >= 0.8

    def bounds(p):
        return rd.render_flip_bounds(_ocam(spec), _settings(kw), sc["mu"], sc["cov"], sc["opacity"], sc["colours"], p)

    _check_pixels(got, got_T, want, want_T, ok, "sports frame", bounds, pix)
    assert np.all(np.isfinite(img)) and T.min() >= 0.0 and T.max() <= 1.0
    assert state.pairs_needed() <= state.max_pairs


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------
BWD_CASES = {
    # name: (n, width, height, desc overrides, means as (x, y, z, t) rows)
    "rgb": (400, 64, 48, dict(sh_degree=-1, background=(0.3, 0.1, 0.2)), False),
    "sh3": (500, 72, 40, dict(sh_degree=3), False),
    "sh2_stride4_no_stop_no_lowpass": (300, 50, 37, dict(sh_degree=2, t_stop=0.0, lowpass=0.0), True),
    "one_gaussian": (1, 24, 20, dict(sh_degree=1), False),
}


@pytest.mark.parametrize("case", list(BWD_CASES))
def test_backward_matches_oracle(sp, case):
    n, w, h, kw, stride4 = BWD_CASES[case]
    deg = kw.get("sh_degree", 3)
    spec = S.orbit_camera(w, h, focal=0.9 * w)
    sc = _scene(n, seed=20 + len(case), deg=deg, scale_factor=0.8)
    if n == 1:
        sc["mu"][:] = 0.0                      # in front of the camera, centred
        sc["cov"][:] = np.array([0.02, 0.003, 0.001, 0.015, 0.002, 0.01], np.float32)
        sc["opacity"][:] = 0.7
    cam, desc, args, img, T, state = _gpu_render(sp, spec, sc, kw, stride4=stride4)
    G = S.image_grads(spec, seed=21)
    got = sp.render_bwd(cam, desc, *args, dev(G), state)
    torch.cuda.synchronize()
    want = rd.render_backward(_ocam(spec), _settings(kw), sc["mu"], sc["cov"], sc["opacity"], sc["colours"], G)
    assert want["grad_ok"].mean() > 0.9
    for k in ("mu", "cov", "opacity", "colours"):
        tol.normwise(host(got[k]).reshape(want[k].shape), want[k], tol.RENDER_GRAD_RTOL, case + " grad " + k)


def test_backward_accumulates_and_accepts_null_outputs(sp):
    n, w, h, kw, _ = BWD_CASES["sh3"]
    spec = S.orbit_camera(w, h, focal=0.9 * w)
    sc = _scene(n, seed=30, deg=3, scale_factor=0.8)
    cam, desc, args, _, _, state = _gpu_render(sp, spec, sc, kw)
    G = dev(S.image_grads(spec, seed=31))
    a = sp.render_bwd(cam, desc, *args, G, state)
    o = a["opacity"].clone()
    sp.render_bwd(cam, desc, *args, G, state, grad_means=a["mu"], grad_cov=a["cov"], grad_opacity=a["opacity"],
                  grad_colours=a["colours"])
    torch.cuda.synchronize()
    tol.normwise(host(a["opacity"]), 2 * host(o), 1e-5, "accumulated opacity grad")
    # NULL outputs: only the opacity gradient requested
    sp._check("spin4d_render_bwd", sp.lib.spin4d_render_bwd(
        sp.ctypes.byref(cam), sp.ctypes.byref(desc), n, args[0].data_ptr(), args[1].data_ptr(), args[2].data_ptr(),
        args[3].data_ptr(), G.data_ptr(), state.buf.data_ptr(), state.buf.numel(), state.max_pairs, None, None,
        a["opacity"].data_ptr(), None, sp._stream(None)))
    torch.cuda.synchronize()
    tol.normwise(host(a["opacity"]), 3 * host(o), 1e-5, "opacity grad with NULL outputs")


def test_backward_full_size_sampled_pixels(sp):
    """Sports frame at 640 x 360: upstream gradient on 48 sampled pixels only,
    so the oracle's backward visits just those."""
    spec = S.orbit_camera(640, 360)
    sc = S.render_scene(300_000, seed=0)
    kw = dict(sh_degree=3)
    cam, desc, args, _, _, state = _gpu_render(sp, spec, sc, kw)
    g = np.random.default_rng(32)
    G = np.zeros((3, 360, 640), np.float32)
    ii, jj = g.integers(0, 640, 48), g.integers(0, 360, 48)
    G[:, jj, ii] = g.normal(size=(3, 48))
    got = sp.render_bwd(cam, desc, *args, dev(G), state)
    torch.cuda.synchronize()
    want = rd.render_backward(_ocam(spec), _settings(kw), sc["mu"], sc["cov"], sc["opacity"], sc["colours"], G)
    for k in ("mu", "cov", "opacity", "colours"):
        tol.normwise(host(got[k]).reshape(want[k].shape), want[k], tol.RENDER_GRAD_RTOL, "sports grad " + k)
