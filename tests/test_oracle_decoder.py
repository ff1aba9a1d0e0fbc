"""Pins for the oracle's decoder, covariance, backward pass, Adam and gate.

Pinned against: the initial-state values SPIN-4DGS section 3.3 prints
(exp(-5) ~ 0.0067, opacity ~ 0.1 from logit(0.1) ~ -2.197, rotation bias
(1,0,0,0)), closed forms of Sigma = R S S^T R^T (eigenvalues s^2, trace,
determinant, axis permutations), the quaternion sandwich product, brute-force
loops for the network, central finite differences for every gradient, the
closed form of Adam's first two steps, and the double-sigmoid window's
value at its centre and its symmetry.
"""
import dataclasses
import math

import numpy as np
import pytest

from oracle import decoder as dec
from oracle import hashgrid as hg
from spatiotemporal_neural_field_b200 import synthetic as S

F32 = np.float32


def _hamilton(a, b):
    w1, x1, y1, z1 = a
    w2, x2, y2, z2 = b
    return np.array([w1 * w2 - x1 * x2 - y1 * y2 - z1 * z2,
                     w1 * x2 + x1 * w2 + y1 * z2 - z1 * y2,
                     w1 * y2 - x1 * z2 + y1 * w2 + z1 * x2,
                     w1 * z2 + x1 * y2 - y1 * x2 + z1 * w2])


def _unit_quats(n, seed):
    q = np.random.default_rng(seed).standard_normal((n, 4))
    return q / np.linalg.norm(q, axis=1, keepdims=True)


def test_initial_state_decode_matches_printed_values():
    """Tables ~ U(+-1e-4) and the page's bias init give s ~ exp(-5) ~ 0.0067,
    r ~ (1,0,0,0), o ~ 0.1 (and sigmoid(0) = 0.5 for colour)."""
    w = S.WORKLOADS["tiny_fp32"]
    pos = S.uniform_positions(512)
    out = dec.decode_forward(pos, S.hash_tables(w["grid"]), S.mlp_weights(w["mlp"]),
                             w["grid"], w["mlp"])
    assert np.all(np.abs(out["scale"] - 0.0067) < 1e-4)
    assert np.all(np.abs(out["opacity"] - 0.1) < 1e-4)
    assert np.all(np.abs(out["rot"] - np.array([1, 0, 0, 0])) < 1e-3)
    assert np.all(np.abs(out["rgb"] - 0.5) < 1e-3)
    np.testing.assert_allclose(np.linalg.norm(out["rot"], axis=1), 1.0, atol=1e-12)


def test_rotation_matrix_matches_quaternion_sandwich():
    q = _unit_quats(50, 7)
    R = dec.quat_to_rotmat(q)
    v = np.random.default_rng(8).standard_normal((50, 3))
    for n in range(50):
        qc = q[n] * np.array([1, -1, -1, -1])
        rv = _hamilton(_hamilton(q[n], np.concatenate([[0], v[n]])), qc)[1:]
        np.testing.assert_allclose(R[n] @ v[n], rv, atol=1e-12)
        np.testing.assert_allclose(R[n].T @ R[n], np.eye(3), atol=1e-12)
        assert abs(np.linalg.det(R[n]) - 1) < 1e-12


def _unpack(c):
    i = [[0, 1, 2], [1, 3, 4], [2, 4, 5]]
    return c[:, i]


def test_covariance_closed_forms():
    q = _unit_quats(100, 9)
    s = np.exp(np.random.default_rng(10).uniform(-5, 1, size=(100, 3)))
    Sig = _unpack(dec.covariance(s, q))
    ev = np.linalg.eigvalsh(Sig)
    np.testing.assert_allclose(np.sort(ev, 1), np.sort(s ** 2, 1), rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(np.trace(Sig, axis1=1, axis2=2), np.sum(s ** 2, 1), rtol=1e-12)
    np.testing.assert_allclose(np.linalg.det(Sig), np.prod(s ** 2, 1), rtol=1e-8)
    ident = np.tile([1.0, 0, 0, 0], (100, 1))
    c0 = dec.covariance(s, ident)
    np.testing.assert_allclose(c0[:, [0, 3, 5]], s ** 2, rtol=1e-15)
    assert np.all(c0[:, [1, 2, 4]] == 0)
    # 90 degrees about z: x -> y, so Sigma_xx = s_y^2 and Sigma_yy = s_x^2
    qz = np.tile([math.cos(math.pi / 4), 0, 0, math.sin(math.pi / 4)], (100, 1))
    cz = dec.covariance(s, qz)
    np.testing.assert_allclose(cz[:, 0], s[:, 1] ** 2, rtol=1e-12)
    np.testing.assert_allclose(cz[:, 3], s[:, 0] ** 2, rtol=1e-12)
    np.testing.assert_allclose(cz[:, 5], s[:, 2] ** 2, rtol=1e-12)


def test_mlp_matches_brute_force_loops():
    rng = np.random.default_rng(11)
    shapes = [(5, 4), (5, 5), (11, 5)]
    layers = [(rng.standard_normal(sh), rng.standard_normal(sh[0])) for sh in shapes]
    z = rng.standard_normal((3, 4))
    y, _, _ = dec.mlp_forward(z, layers)
    for n in range(3):
        a = list(z[n])
        for j, (W, b) in enumerate(layers):
            nxt = []
            for o in range(W.shape[0]):
                acc = b[o]
                for i in range(W.shape[1]):
                    acc += W[o][i] * a[i]
                nxt.append(max(acc, 0.0) if j < len(layers) - 1 else acc)
            a = nxt
        np.testing.assert_allclose(y[n], a, rtol=1e-13, atol=1e-13)


def test_gate_closed_forms():
    tau = 0.02
    c = np.array([0.3, 0.7])
    r = np.array([0.1, 0.4])
    at_c = dec.temporal_gate(c, c, r, tau)
    np.testing.assert_allclose(at_c, (1 / (1 + np.exp(-r / tau))) ** 2, rtol=1e-14)
    d = np.array([0.05, 0.2])
    np.testing.assert_allclose(dec.temporal_gate(c + d, c, r, tau), dec.temporal_gate(c - d, c, r, tau),
                               rtol=1e-12)
    assert np.all(dec.temporal_gate(c + r + 0.3, c, r, tau) < 1e-6)
    assert np.all(dec.temporal_gate(c, c, r, tau) > 0.98)       # sigmoid(5)^2 = 0.9867


def test_adam_first_two_steps_closed_form():
    g1 = np.array([0.5, -2.0, 1e-3, 0.0])
    p0 = np.array([1.0, 1.0, 1.0, 1.0])
    lr, b1, b2, eps = 1e-3, 0.9, 0.99, 1e-15
    p1, m, v = dec.adam_step(p0, g1, np.zeros(4), np.zeros(4), 1, lr, b1, b2, eps)
    # first step: m^ = g, v^ = g^2, update = lr * g / (|g| + eps)
    np.testing.assert_allclose(p1, p0 - lr * g1 / (np.abs(g1) + eps), rtol=1e-15)
    g2 = np.array([-0.5, 1.0, 1e-3, 2.0])
    p2, _, _ = dec.adam_step(p1, g2, m, v, 2, lr, b1, b2, eps)
    mh = (0.9 * 0.1 * g1 + 0.1 * g2) / (1 - 0.81)
    vh = (0.99 * 0.01 * g1 ** 2 + 0.01 * g2 ** 2) / (1 - 0.9801)
    np.testing.assert_allclose(p2, p1 - lr * mh / (np.sqrt(vh) + eps), rtol=1e-12)


# ---------------------------------------------------------------------------
# Finite differences on a tiny problem, for every gradient term
# ---------------------------------------------------------------------------
TINY_GRID = S.GridSpec(L=2, F=2, log2_T=6, nmin_s=2, nmax_s=5, nmin_t=2, nmax_t=3,
                       dtype="f32", t_min=0.0, t_max=1.0)


def _tiny_problem(gate: bool, seed: int = 12):
    mlp = S.MlpSpec(in_dim=4, hidden=5, n_hidden=2, dtype="f32", gate=gate, tau=0.2)
    rng = np.random.default_rng(seed)
    pos = rng.uniform(-1.3, 1.3, size=(7, 4))
    pos[:, 3] = rng.uniform(0, 1, size=7)
    tables = rng.uniform(-1, 1, size=(2, 64, 2))
    layers = [(rng.uniform(-1, 1, size=sh), rng.uniform(-0.5, 0.5, size=sh[0])) for sh in mlp.layer_shapes()]
    W, b = layers[-1]
    b = b + np.array([-1.0, -1.0, -1.0, 1, 0, 0, 0, 0, 0, 0, -1.0])
    layers[-1] = (W, b)
    weights = dec.pack_layers(layers)
    cr = np.stack([rng.uniform(0.2, 0.8, 7), rng.uniform(0.1, 0.3, 7)], 1)
    grads = {k: rng.standard_normal((7, w)) for k, w in S.DECODE_OUT_WIDTHS.items()}
    return mlp, pos.astype(F32), tables, weights, cr, grads


def _loss(pos, tables, weights, mlp, cr, grads):
    out = dec.decode_forward(pos, tables, weights, TINY_GRID, mlp, gate_cr=cr)
    return sum(np.sum(grads[k] * out[k]) for k in grads)


@pytest.mark.parametrize("gate", [False, True])
def test_backward_matches_central_finite_differences(gate):
    mlp, pos, tables, weights, cr, grads = _tiny_problem(gate)
    gt, gw = dec.decode_backward(pos, tables, weights, TINY_GRID, mlp, grads, gate_cr=cr)
    h = 1e-6
    # tables: every entry that receives any gradient, plus a few that do not
    touched = np.argwhere(np.abs(gt) > 0)
    assert len(touched) > 20
    rng = np.random.default_rng(0)
    pick = touched[rng.choice(len(touched), size=min(60, len(touched)), replace=False)]
    for (l, e, f) in pick:
        tp, tm = tables.copy(), tables.copy()
        tp[l, e, f] += h
        tm[l, e, f] -= h
        fd = (_loss(pos, tp, weights, mlp, cr, grads) - _loss(pos, tm, weights, mlp, cr, grads)) / (2 * h)
        assert abs(fd - gt[l, e, f]) <= 1e-6 * max(1.0, abs(fd)), (l, e, f, fd, gt[l, e, f])
    for k in range(weights.size):
        wp, wm = weights.copy(), weights.copy()
        wp[k] += h
        wm[k] -= h
        fd = (_loss(pos, tables, wp, mlp, cr, grads) - _loss(pos, tables, wm, mlp, cr, grads)) / (2 * h)
        assert abs(fd - gw[k]) <= 1e-6 * max(1.0, abs(fd)), (k, fd, gw[k])


def test_scale_clip_blocks_gradient_above_20():
    """s = exp(min(s^, 20)): the gradient w.r.t. s^ is exp(s^) * g below the
    clip and exactly 0 above it (finite differences agree on both sides)."""
    y = np.zeros((4, 11))
    y[:, 3] = 1.0
    y[:, 0] = [19.5, 20.5, -5.0, 25.0]
    y[:, 1] = [0.3, 21.0, 19.99, -1.0]
    y[:, 2] = 1.0
    g = {k: np.zeros((4, w)) for k, w in S.DECODE_OUT_WIDTHS.items()}
    g["scale"] = np.random.default_rng(1).standard_normal((4, 3))
    dy = dec.heads_backward(y, g)
    for n in range(4):
        for d in range(3):
            h = 1e-3
            yp, ym = y.copy(), y.copy()
            yp[n, d] += h
            ym[n, d] -= h
            # loss restricted to this element, so other large terms add no roundoff
            lp = g["scale"][n, d] * dec.heads_forward(yp)["scale"][n, d]
            lm = g["scale"][n, d] * dec.heads_forward(ym)["scale"][n, d]
            fd = (lp - lm) / (2 * h)
            if y[n, d] > 20:
                assert dy[n, d] == 0 and fd == 0
            else:
                assert abs(fd - dy[n, d]) <= 1e-6 * abs(fd), (n, d, fd, dy[n, d])


def test_backward_terms_individually():
    """Each upstream output alone (scale, rot, rgb, opacity, cov) checked by FD
    on the head bias, so a dropped or mis-signed term is caught in isolation."""
    mlp, pos, tables, weights, cr, grads = _tiny_problem(True)
    shapes = mlp.layer_shapes()
    off = sum(o * i + o for o, i in shapes[:-1]) + shapes[-1][0] * shapes[-1][1]
    for key in S.DECODE_OUT_WIDTHS:
        g1 = {k: (v if k == key else np.zeros_like(v)) for k, v in grads.items()}
        _, gw = dec.decode_backward(pos, tables, weights, TINY_GRID, mlp, g1, gate_cr=cr)
        for k in range(off, off + 11):
            wp, wm = weights.copy(), weights.copy()
            wp[k] += 1e-6
            wm[k] -= 1e-6
            fd = (_loss(pos, tables, wp, mlp, cr, g1) - _loss(pos, tables, wm, mlp, cr, g1)) / 2e-6
            assert abs(fd - gw[k]) <= 1e-6 * max(1.0, abs(fd)), (key, k, fd, gw[k])
