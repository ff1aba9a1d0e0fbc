"""Pins for the oracle's HexPlane encoder and deformation network (CPU only).

Pinned against: lookups at exact plane vertices (planes storing their own
flat index), partition of unity, exact reproduction of a bilinear function of
the plane coordinates, and central finite differences of every gradient on a
tiny spec.
"""
import dataclasses

import numpy as np

from oracle import decoder as dec
from oracle import hexplane as hp
from spatiotemporal_neural_field_b200 import synthetic as S

F32 = np.float32
TINY = S.HexSpec(hidden=3, n_hidden=2, channels=2, scales=(3, 5), time_res=4, n_frames=7)


def test_plane_layout_size_matches_spec():
    hx = S.HEX
    assert hx.in_dim == 576
    assert hx.n_plane_floats() == 11_483_136            # 45.9 MB of fp32 planes


def test_partition_of_unity():
    rng = np.random.default_rng(0)
    mu = rng.uniform(-1, 1, size=(300, 3))
    fr = rng.integers(0, 7, size=300)
    z = hp.encode(hp.normalise(mu, fr, 7), np.ones(TINY.n_plane_floats()), TINY)
    np.testing.assert_allclose(z, 1.0, atol=1e-14)


def test_vertex_lookup_and_bilinear_reproduction():
    hx = TINY
    offs = hp.plane_offsets(hx)
    C = hx.channels
    # planes hold f(col, row) = a*col + b*row + c*col*row + d (+ channel)
    a, b, c, d = 0.7, -1.3, 0.25, 2.0
    planes = np.zeros(hx.n_plane_floats())
    for k, (rows, cols) in enumerate(hx.plane_shapes()):
        rr, cc = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
        for ch in range(C):
            planes[offs[k] + (rr * cols + cc) * C + ch] = a * cc + b * rr + c * cc * rr + d + ch
    rng = np.random.default_rng(1)
    mu = rng.uniform(-1, 1, size=(200, 3)).astype(F32)
    fr = rng.integers(0, 7, size=200)
    xt = hp.normalise(mu, fr, 7)
    z = hp.encode(xt, planes, hx)
    k = 0
    for m in hx.scales:
        for (ax_a, ax_b) in hp.PLANE_AXES:
            ra = hx.time_res if ax_a == 3 else m
            rb = hx.time_res if ax_b == 3 else m
            pa = (xt[:, ax_a] * F32(ra - 1)).astype(np.float64)
            pb = (xt[:, ax_b] * F32(rb - 1)).astype(np.float64)
            for ch in range(C):
                want = a * pa + b * pb + c * pa * pb + d + ch
                np.testing.assert_allclose(z[:, k * C + ch], want, rtol=1e-12, atol=1e-12)
            k += 1
    # exact vertices: frame k of 7 with time_res 4 -> p = k/6*3 integer for even k
    mu_v = np.array([[-1.0, 0.0, 1.0], [0.5, -0.5, 0.0]], F32)
    fr_v = np.array([0, 6])
    zv = hp.encode(hp.normalise(mu_v, fr_v, 7), planes, hx)
    # scale 3 (res 3, p = x~*2): mu=-1 -> 0, 0 -> 1, 1 -> 2 ; XY plane value
    assert zv[0, 0] == a * 0 + b * 1 + c * 0 + d


def _tiny_inputs(n=5, seed=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    return dict(mu=rng.uniform(-1, 1, (n, 3)).astype(F32), frame=rng.integers(0, 7, n),
                q_can=q, logs_can=rng.uniform(-3, -1, (n, 3)), sh_can=rng.standard_normal((n, 48)))


def _loss(inp, planes, weights, grads):
    out = hp.forward(inp, planes, weights, TINY)
    return sum(np.sum(grads[k] * out[k]) for k in grads)


def test_backward_matches_central_finite_differences():
    rng = np.random.default_rng(3)
    inp = _tiny_inputs()
    planes = rng.uniform(0.1, 0.5, TINY.n_plane_floats())
    # trunk biases > 0 keep the ReLUs alive so gradients reach the planes
    layers = [(rng.uniform(-0.8, 0.8, sh), rng.uniform(0.5, 1.0, sh[0])) for sh in TINY.layer_shapes()]
    weights = dec.pack_layers(layers)
    grads = {k: rng.standard_normal((5, w)) for k, w in S.HEX_OUT_WIDTHS.items()}
    gp, gw = hp.backward(inp, planes, weights, TINY, grads)
    y, _, pres = dec.mlp_forward(hp.encode(hp.normalise(inp["mu"], inp["frame"], 7), planes, TINY),
                                 dec.unpack_layers(weights, TINY.layer_shapes()))
    assert all(np.any(p > 0) and np.any(p < 0) for p in pres[:-1]) or all(np.any(p > 0) for p in pres[:-1])
    h = 1e-6
    touched = np.flatnonzero(gp)
    assert touched.size > 50
    for e in rng.choice(touched, size=60, replace=False):
        pp, pm = planes.copy(), planes.copy()
        pp[e] += h
        pm[e] -= h
        fd = (_loss(inp, pp, weights, grads) - _loss(inp, pm, weights, grads)) / (2 * h)
        assert abs(fd - gp[e]) <= 1e-6 * max(1.0, abs(fd)), (e, fd, gp[e])
    for k in range(weights.size):
        wp, wm = weights.copy(), weights.copy()
        wp[k] += h
        wm[k] -= h
        fd = (_loss(inp, planes, wp, grads) - _loss(inp, planes, wm, grads)) / (2 * h)
        assert abs(fd - gw[k]) <= 1e-6 * max(1.0, abs(fd)), (k, fd, gw[k])


def test_outputs_are_valid():
    rng = np.random.default_rng(4)
    inp = _tiny_inputs(20, 5)
    out = hp.forward(inp, rng.uniform(0.1, 0.5, TINY.n_plane_floats()),
                     rng.uniform(-0.5, 0.5, TINY.n_params()), TINY)
    np.testing.assert_allclose(np.linalg.norm(out["rot"], axis=1), 1.0, atol=1e-12)
    assert np.all(out["scale"] > 0)
    Sig = out["cov"][:, [[0, 1, 2], [1, 3, 4], [2, 4, 5]]]
    assert np.all(np.linalg.eigvalsh(Sig) > -1e-15)


# ---------------------------------------------------------------------------
# Energy-flow window and the binary displacement gate (KineticGS notes)
# ---------------------------------------------------------------------------
TAU = 0.02


def _gate_setup(n=6, seed=7):
    rng = np.random.default_rng(seed)
    inp = _tiny_inputs(n, seed)
    planes = rng.uniform(0.1, 0.5, TINY.n_plane_floats())
    layers = [(rng.uniform(-0.8, 0.8, sh), rng.uniform(0.5, 1.0, sh[0])) for sh in TINY.layer_shapes()]
    return inp, planes, dec.pack_layers(layers)


def _t_norm(inp):
    return hp.normalise(inp["mu"], inp["frame"], TINY.n_frames)[:, 3].astype(np.float64)


def test_displacement_gate_threshold():
    w = np.array([0.0, 0.25, 0.5 - 1e-12, 0.5, 0.5 + 1e-12, 0.75, 1.0])
    assert list(hp.displacement_gate(w)) == [0, 0, 0, 1, 1, 1, 1]


def test_window_inside_reduces_to_ungated_and_outside_freezes_the_gaussian():
    """A wide window centred on the frame gives w = sigmoid(r/tau)^2, which is
    1 to fp64 for r/tau = 50 (sigmoid(50) = 1 - 2e-22): the gated outputs are
    the ungated ones.  A window far from the frame gives w ~ 0 and H = 0: the
    mean is the canonical mean exactly, and scale and SH are the canonical
    ones up to w * offset (w < e^-40)."""
    inp, planes, weights = _gate_setup()
    t = _t_norm(inp)
    plain = hp.forward(inp, planes, weights, TINY)
    inside = hp.forward(inp, planes, weights, TINY, gate=dict(cr=np.stack([t, np.full_like(t, 1.0)], 1), tau=TAU))
    np.testing.assert_allclose(inside["w"], 1.0, rtol=0, atol=1e-15)
    for k in ("mu", "rot", "scale", "sh", "cov"):
        np.testing.assert_allclose(inside[k], plain[k], rtol=1e-14, atol=1e-15)
    far = hp.forward(inp, planes, weights, TINY, gate=dict(cr=np.stack([t + 3.0, np.full_like(t, 0.1)], 1), tau=TAU))
    assert np.all(far["w"] < np.exp(-40))
    assert np.array_equal(far["mu"], np.asarray(inp["mu"], np.float64))
    np.testing.assert_allclose(far["scale"], np.exp(inp["logs_can"]), rtol=1e-15)
    np.testing.assert_allclose(far["sh"], inp["sh_can"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(far["rot"], plain["rot"], rtol=0, atol=0)   # rotation offset is not gated


def test_window_edge_halves_the_offsets_and_moves_the_mean():
    """At the window's upper edge t~ = c + r, w = 1/2 * sigmoid(2r/tau), just
    below 1/2 (r/tau = 10: 1/2 - 1e-9): H = 0, and log s' = log s + w d_logs."""
    inp, planes, weights = _gate_setup()
    t = _t_norm(inp)
    r = np.full_like(t, 0.2)
    cr = np.stack([t - r, r], 1)
    out = hp.forward(inp, planes, weights, TINY, gate=dict(cr=cr, tau=TAU))
    want_w = 0.5 * dec.sigmoid(2 * r / float(np.float32(TAU)))
    np.testing.assert_allclose(out["w"], want_w, rtol=1e-12)
    assert np.all(out["w"] < 0.5)
    assert np.array_equal(out["mu"], np.asarray(inp["mu"], np.float64))
    plain = hp.forward(inp, planes, weights, TINY)
    d_logs = np.log(plain["scale"]) - inp["logs_can"]
    np.testing.assert_allclose(np.log(out["scale"]), inp["logs_can"] + out["w"][:, None] * d_logs, rtol=1e-12)
    # a slightly narrower offset of the window (centre 2 tau inside) crosses 1/2: H = 1 and the mean moves
    cr2 = np.stack([t - r + 2 * TAU, r], 1)
    out2 = hp.forward(inp, planes, weights, TINY, gate=dict(cr=cr2, tau=TAU))
    assert np.all(out2["w"] > 0.5)
    np.testing.assert_allclose(out2["mu"], plain["mu"], rtol=1e-14, atol=1e-15)


def _gated_loss(inp, planes, weights, grads, cr):
    out = hp.forward(inp, planes, weights, TINY, gate=dict(cr=cr, tau=TAU))
    return sum(np.sum(grads[k] * out[k]) for k in grads)


def test_gated_backward_matches_central_finite_differences():
    """Planes, weights, c and r, with windows placed so that every Gaussian
    sits on a slope of its window (w away from 1/2, so H is locally constant)
    and some Gaussians are inside (H = 1) and some outside (H = 0)."""
    rng = np.random.default_rng(8)
    n = 6
    inp, planes, weights = _gate_setup(n, 9)
    t = _t_norm(inp)
    r = rng.uniform(0.05, 0.3, n)
    # offsets from the window edge in units of tau: inside (w > 1/2) and outside (w < 1/2)
    off = np.array([1.5, -1.5, 0.7, -0.8, 2.5, -2.0])
    cr = np.stack([t - r + off * TAU, r], 1)            # upper edge c + r = t + off*tau
    w = hp.energy_window(hp.normalise(inp["mu"], inp["frame"], TINY.n_frames), cr, TAU)
    assert np.all(np.abs(w - 0.5) > 0.1) and np.any(w > 0.5) and np.any(w < 0.5)
    grads = {k: rng.standard_normal((n, wd)) for k, wd in S.HEX_OUT_WIDTHS.items()}
    gp, gw, gcr = hp.backward(inp, planes, weights, TINY, grads, gate=dict(cr=cr, tau=TAU), want_gate=True)
    h = 1e-6
    touched = np.flatnonzero(gp)
    for e in rng.choice(touched, size=40, replace=False):
        pp, pm = planes.copy(), planes.copy()
        pp[e] += h
        pm[e] -= h
        fd = (_gated_loss(inp, pp, weights, grads, cr) - _gated_loss(inp, pm, weights, grads, cr)) / (2 * h)
        assert abs(fd - gp[e]) <= 1e-6 * max(1.0, abs(fd)), (e, fd, gp[e])
    for k in range(weights.size):
        wp, wm = weights.copy(), weights.copy()
        wp[k] += h
        wm[k] -= h
        fd = (_gated_loss(inp, planes, wp, grads, cr) - _gated_loss(inp, planes, wm, grads, cr)) / (2 * h)
        assert abs(fd - gw[k]) <= 1e-6 * max(1.0, abs(fd)), (k, fd, gw[k])
    # c and r one Gaussian at a time (the loss is a sum over Gaussians)
    hh = 1e-7
    for i in range(n):
        for j in range(2):
            cp, cm = cr.copy(), cr.copy()
            cp[i, j] += hh
            cm[i, j] -= hh
            fd = (_gated_loss(inp, planes, weights, grads, cp) - _gated_loss(inp, planes, weights, grads, cm)) / (2 * hh)
            assert abs(fd - gcr[i, j]) <= 1e-5 * max(1.0, abs(fd)), (i, j, fd, gcr[i, j])
    # the mean's gradient reaches the displacement head only where H = 1
    layers = dec.unpack_layers(weights, TINY.layer_shapes())
    dW3 = gw[-(58 * TINY.hidden + 58):-58].reshape(58, TINY.hidden)
    z = hp.encode(hp.normalise(inp["mu"], inp["frame"], TINY.n_frames), planes, TINY)
    _, acts, _ = dec.mlp_forward(z, layers)
    want_rows = (grads["mu"] * hp.displacement_gate(w)[:, None]).T @ acts[-1]
    np.testing.assert_allclose(dW3[0:3], want_rows, rtol=1e-12, atol=1e-14)


def test_window_gradient_vanishes_at_the_centre_for_c():
    """At t~ = c the two sigmoids are equal, so dw/dc = a b (a - b)/tau = 0."""
    inp, planes, weights = _gate_setup()
    t = _t_norm(inp)
    cr = np.stack([t, np.full_like(t, 0.05)], 1)
    grads = {k: np.random.default_rng(1).standard_normal((len(t), wd)) for k, wd in S.HEX_OUT_WIDTHS.items()}
    _, _, gcr = hp.backward(inp, planes, weights, TINY, grads, gate=dict(cr=cr, tau=TAU), want_gate=True)
    np.testing.assert_allclose(gcr[:, 0], 0.0, atol=1e-12)
    assert np.all(np.abs(gcr[:, 1]) > 0)
