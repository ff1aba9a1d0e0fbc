"""Pins of the oracle's position gradient (trainable Gaussian means).

The position gradient is not printed anywhere in the pages; it is pinned
here against things other than its own formula:

* the contraction Jacobian against the two facts Eq. 7 fixes directly: the
  contracted point stays on the ray of mu with length 2 - 1/|mu| (radial
  derivative 1/n^2, tangential stretch (2 - 1/n)/n), and mu/4 inside;
* the encoder adjoint against multilinear reproduction: a dense level whose
  table is a linear (or bilinear) function of the vertex coordinates
  interpolates that function exactly, so its derivative is known in closed
  form at every position;
* the encoder adjoint and the whole backward against central finite
  differences, on positions exactly representable in fp32 so that the
  perturbed corner decisions and weights are exact.
"""
import dataclasses

import numpy as np
import pytest

from oracle import decoder as dec
from oracle import hashgrid as hg
from spatiotemporal_neural_field_b200 import synthetic as S

TINY = S.GRID_TINY
RES = hg.grid_resolutions(TINY.L, TINY.nmin_s, TINY.nmax_s, TINY.nmin_t, TINY.nmax_t)


def test_contraction_jacobian_inside_is_quarter_identity():
    pos = np.array([[0.3, -0.2, 0.1, 0.0], [0.0, 0.0, 0.0, 5.0], [0.6, 0.0, -0.8, 1.0]], np.float32)
    J = hg.contraction_jacobian(pos)
    assert np.array_equal(J, np.broadcast_to(0.25 * np.eye(3), J.shape))


def test_contraction_jacobian_radial_and_tangential():
    rng = np.random.default_rng(5)
    mu = rng.normal(size=(200, 3)) * 3.0
    mu = mu[np.linalg.norm(mu, axis=1) > 1.05].astype(np.float32)
    pos = np.concatenate([mu, np.zeros((len(mu), 1), np.float32)], axis=1)
    J = hg.contraction_jacobian(pos)
    m = mu.astype(np.float64)
    n = np.linalg.norm(m, axis=1)
    u = m / n[:, None]
    # |c| = 2 - 1/n along the ray: d|c|/dn = 1/n^2, so J u = u / (4 n^2)
    np.testing.assert_allclose(np.einsum("nij,nj->ni", J, u), u / (4 * n[:, None] ** 2), rtol=1e-12, atol=1e-15)
    # a direction t orthogonal to mu is stretched by |c| / n = (2 - 1/n) / n
    t = np.cross(u, rng.normal(size=u.shape))
    t /= np.linalg.norm(t, axis=1)[:, None]
    np.testing.assert_allclose(np.einsum("nij,nj->ni", J, t), t * ((2 - 1 / n) / n / 4)[:, None], rtol=1e-12,
                               atol=1e-15)
    assert np.allclose(J, np.transpose(J, (0, 2, 1)))


def _dense_level_table(fn):
    """Tiny-grid tables that are zero except level 0 feature 0 = fn(vx, vy, vz, vt)."""
    tables = np.zeros((TINY.L, 1 << TINY.log2_T, TINY.F), np.float32)
    rx, ry, rz, rt = (int(r) for r in RES[0])
    assert hg.is_dense(RES[0], TINY.log2_T)
    for vt in range(rt):
        for vz in range(rz):
            for vy in range(ry):
                for vx in range(rx):
                    tables[0, vx + rx * (vy + ry * (vz + rz * vt)), 0] = fn(vx, vy, vz, vt)
    return tables


def _dz_level0_feature0(n):
    dz = np.zeros((n, TINY.L * TINY.F))
    dz[:, 0] = 1.0
    return dz


def test_encoder_adjoint_linear_reproduction():
    a = (0.5, -1.25, 2.0, 0.75)
    tables = _dense_level_table(lambda x, y, z, t: a[0] * x + a[1] * y + a[2] * z + a[3] * t)
    xt = np.random.default_rng(1).uniform(0, 1, size=(300, 4)).astype(np.float32)
    xt[:4] = [[0, 0, 0, 0], [1, 1, 1, 1], [1, 0, 0.5, 1], [0.25, 1, 0, 0.999]]   # cell edges and the top cell
    g = hg.encode_position_grad(_dz_level0_feature0(len(xt)), xt, tables, RES, TINY.log2_T)
    want = np.array(a) * (RES[0] - 1)
    np.testing.assert_allclose(g, np.broadcast_to(want, g.shape), rtol=1e-12, atol=1e-12)


def test_encoder_adjoint_bilinear_reproduction():
    tables = _dense_level_table(lambda x, y, z, t: x * y)
    xt = np.random.default_rng(2).uniform(0, 1, size=(300, 4)).astype(np.float32)
    g = hg.encode_position_grad(_dz_level0_feature0(len(xt)), xt, tables, RES, TINY.log2_T)
    # z = p_x p_y exactly, with p = x~ (res - 1) formed in fp32 as the encoder does
    p = (xt * (RES[0] - 1).astype(np.float32)).astype(np.float64)
    np.testing.assert_allclose(g[:, 0], (RES[0, 0] - 1) * p[:, 1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[:, 1], (RES[0, 1] - 1) * p[:, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[:, 2:], 0.0, atol=1e-12)


H = 2.0 ** -12


def _grid_positions(n, seed, h=H):
    """Positions on the h lattice (exact in fp32, as are p = x~ (res-1) and
    x~ +- h, while 1/h times the largest res-1 stays under 2^24) whose +-h
    neighbours stay in the same cell at every level."""
    rng = np.random.default_rng(seed)
    k = int(round(1 / h))
    xt = rng.integers(k // 64, k - k // 64, size=(4 * n, 4)) * h
    ok = np.ones(len(xt), bool)
    for l in range(TINY.L):
        for d in range(4):
            r = int(RES[l, d]) - 1
            ok &= np.floor((xt[:, d] - h) * r) == np.floor((xt[:, d] + h) * r)
    xt = xt[ok][:n]
    assert len(xt) == n
    return xt.astype(np.float32)


def test_encoder_adjoint_matches_central_differences():
    """Inside a cell the encoder is multilinear in x~, so the central difference
    is exact up to rounding."""
    xt = _grid_positions(64, 3)
    tables = S.hash_tables(TINY, seed=4, scale=1.0)
    dz = np.random.default_rng(5).normal(size=(len(xt), TINY.L * TINY.F))
    g = hg.encode_position_grad(dz, xt, tables, RES, TINY.log2_T)
    for d in range(4):
        e = np.zeros(4, np.float32)
        e[d] = H
        fd = np.sum(dz * (hg.encode(xt + e, tables, RES, TINY.log2_T) - hg.encode(xt - e, tables, RES, TINY.log2_T)),
                    axis=1) / (2 * H)
        np.testing.assert_allclose(g[:, d], fd, rtol=1e-9, atol=1e-9)


def test_decode_backward_position_gradient_matches_central_differences():
    """Whole path on normalised inputs: L = sum_k <g_k, out_k>.  The network
    and activations curve, so the step is small (2^-18: truncation error
    ~1e-9 relative; 2^-12 and 2^-16 give 2e-2 and 3e-8, shrinking as h^2)."""
    h = 2.0 ** -18
    xt = _grid_positions(32, 6, h)
    tables = S.hash_tables(TINY, seed=7, scale=1.0)
    weights = S.mlp_weights(S.MLP_TINY, seed=8, bias_scale=0.5)
    grads = S.upstream_grads(len(xt), S.DECODE_OUT_WIDTHS, 1.0, seed=9)
    _, _, gpos = dec.decode_backward(xt, tables, weights, TINY, S.MLP_TINY, grads, normalised_input=True,
                                     want_pos=True)

    def loss(x):
        out = dec.decode_forward(x, tables, weights, TINY, S.MLP_TINY, normalised_input=True)
        return sum(np.sum(np.asarray(grads[k], np.float64) * out[k], axis=1) for k in grads)

    assert gpos.shape == (len(xt), 3)
    for d in range(3):
        e = np.zeros(4, np.float32)
        e[d] = h
        fd = (loss(xt + e) - loss(xt - e)) / (2 * h)
        np.testing.assert_allclose(gpos[:, d], fd, rtol=1e-6, atol=1e-6)


def test_decode_backward_position_gradient_composes_the_contraction():
    """Raw positions: grad_mu = J^T grad_x~ with J the contraction Jacobian,
    so inside the unit ball it is a quarter of the normalised-input gradient."""
    rng = np.random.default_rng(10)
    pos = np.concatenate([rng.uniform(-0.5, 0.5, size=(40, 3)), rng.uniform(0, 1, size=(40, 1))], axis=1)
    pos = pos.astype(np.float32)
    tables = S.hash_tables(TINY, seed=11, scale=1.0)
    weights = S.mlp_weights(S.MLP_TINY, seed=12, bias_scale=0.5)
    grads = S.upstream_grads(len(pos), S.DECODE_OUT_WIDTHS, 1.0, seed=13)
    _, _, g_raw = dec.decode_backward(pos, tables, weights, TINY, S.MLP_TINY, grads, want_pos=True)
    xt = hg.normalise(pos, TINY.t_min, TINY.t_max)
    _, _, g_norm = dec.decode_backward(xt, tables, weights, TINY, S.MLP_TINY, grads, normalised_input=True,
                                       want_pos=True)
    np.testing.assert_allclose(g_raw, 0.25 * g_norm, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------
# Gate parameters (the KineticGS window centre c and half-width r)
# ---------------------------------------------------------------------------
def test_gate_gradient_closed_forms():
    """At the centre (t = c) the window is symmetric: dw/dc = 0 and
    dw/dr = 2 a^2 (1 - a)/tau with a = sigma(r/tau); far outside, both vanish."""
    tau = 0.02
    r = np.array([0.05, 0.1, 0.3])
    t = np.array([0.4, 0.5, 0.9])
    dc, dr = dec.temporal_gate_grad(t, t, r, tau)
    a = 1 / (1 + np.exp(-r / tau))
    np.testing.assert_allclose(dc, 0.0, atol=1e-15)
    np.testing.assert_allclose(dr, 2 * a * a * (1 - a) / tau, rtol=1e-12, atol=1e-12)
    dc, dr = dec.temporal_gate_grad(np.array([0.0]), np.array([0.9]), np.array([0.05]), tau)
    assert abs(dc[0]) < 1e-12 and abs(dr[0]) < 1e-12


def test_gate_gradient_matches_central_differences():
    grid = TINY
    mlp = dataclasses.replace(S.MLP_TINY, gate=True, tau=0.02)     # the tiny decoder with the gate
    n = 64
    xt = np.random.default_rng(20).uniform(0.05, 0.95, size=(n, 4)).astype(np.float32)
    tables = S.hash_tables(grid, seed=21, scale=1.0)
    weights = S.mlp_weights(mlp, seed=22, bias_scale=0.5)
    cr = S.gate_params(n, seed=23).astype(np.float64)
    cr[:, 0] = xt[:, 3] + np.random.default_rng(24).uniform(-0.2, 0.2, n)   # windows near each t
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, 1.0, seed=25)
    _, _, gcr = dec.decode_backward(xt, tables, weights, grid, mlp, grads, gate_cr=cr, normalised_input=True,
                                    want_gate=True)

    def loss(c):
        out = dec.decode_forward(xt, tables, weights, grid, mlp, gate_cr=c, normalised_input=True)
        return sum(np.sum(np.asarray(grads[k], np.float64) * out[k], axis=1) for k in grads)

    h = 1e-6
    for j in range(2):
        e = np.zeros(2)
        e[j] = h
        fd = (loss(cr + e) - loss(cr - e)) / (2 * h)
        np.testing.assert_allclose(gcr[:, j], fd, rtol=1e-6, atol=1e-7)


def test_position_gradient_is_zero_where_the_clamp_holds():
    """Normalised input outside [0, 1] is clamped, so the output does not move
    with that coordinate: its central difference, and the gradient, are 0;
    the in-range coordinates keep their central differences."""
    h = 2.0 ** -18
    base = _grid_positions(16, 14, h)
    xt = base.copy()
    xt[:8, 0] = -0.25                       # clamped below on x
    xt[8:, 1] = 1.375                       # clamped above on y
    tables = S.hash_tables(TINY, seed=15, scale=1.0)
    weights = S.mlp_weights(S.MLP_TINY, seed=16, bias_scale=0.5)
    grads = S.upstream_grads(len(xt), S.DECODE_OUT_WIDTHS, 1.0, seed=17)
    _, _, gpos = dec.decode_backward(xt, tables, weights, TINY, S.MLP_TINY, grads, normalised_input=True,
                                     want_pos=True)

    def loss(x):
        out = dec.decode_forward(x, tables, weights, TINY, S.MLP_TINY, normalised_input=True)
        return sum(np.sum(np.asarray(grads[k], np.float64) * out[k], axis=1) for k in grads)

    for d in range(3):
        e = np.zeros(4, np.float32)
        e[d] = h
        fd = (loss(xt + e) - loss(xt - e)) / (2 * h)
        np.testing.assert_allclose(gpos[:, d], fd, rtol=1e-6, atol=1e-6)
    assert np.all(gpos[:8, 0] == 0.0) and np.all(gpos[8:, 1] == 0.0)
    assert np.abs(gpos[:8, 1:]).max() > 1e-3 and np.abs(gpos[8:, [0, 2]]).max() > 1e-3
