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
