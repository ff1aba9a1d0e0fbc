"""Pins of the four-head GELU decoder oracle (SPIN-4DGS section 3.3).

Against values and properties the pages and mathematics fix: the standard
normal CDF at +-1 (GELU = x Phi(x)), GELU's limits and slope at 0, brute-force
loops for one head, the initial state the page prints (zero weights leave
the final biases: exp(-5), (1,0,0,0), logit(0.1) -> 0.1, SH 0), the heads'
independence, central differences for every gradient, and the learning-rate
schedule's end points.
"""
import math

import numpy as np

from oracle import heads as hd
from spatiotemporal_neural_field_b200 import synthetic as S

SPEC = S.HEADS_TINY
GRID = S.GRID_TINY4


def test_gelu_closed_forms():
    phi1 = 0.8413447460685429                       # standard normal CDF at 1
    x = np.array([0.0, 1.0, -1.0, 8.0, -8.0])
    g = hd.gelu(x)
    np.testing.assert_allclose(g[:3], [0.0, phi1, -(1.0 - phi1)], rtol=1e-15, atol=1e-16)
    assert abs(g[3] - 8.0) < 1e-13 and abs(g[4]) < 1e-13
    assert hd.gelu_grad(np.array([0.0]))[0] == 0.5
    xs = np.linspace(-5, 5, 101)
    h = 1e-6
    np.testing.assert_allclose(hd.gelu_grad(xs), (hd.gelu(xs + h) - hd.gelu(xs - h)) / (2 * h), rtol=1e-8, atol=1e-9)


def test_head_matches_brute_force_loops():
    rng = np.random.default_rng(0)
    z = rng.normal(size=(3, SPEC.in_dim))
    heads = hd.unpack(S.heads_weights(SPEC, seed=1, bias_scale=0.3), SPEC)
    for h in range(4):
        y, _, _ = hd.head_forward(z, heads[h])
        for n in range(3):
            a = list(z[n])
            for j, (W, b) in enumerate(heads[h]):
                nxt = []
                for o in range(W.shape[0]):
                    acc = b[o]
                    for k in range(W.shape[1]):
                        acc += W[o, k] * a[k]
                    nxt.append(0.5 * acc * (1 + math.erf(acc / math.sqrt(2))) if j < 2 else acc)
                a = nxt
            np.testing.assert_allclose(y[n], a, rtol=1e-12)


def test_initial_state_is_the_papers():
    """With every weight matrix zero the heads output their final biases."""
    w = S.heads_weights(S.HEADS_PAPER).astype(np.float64)
    heads = hd.unpack(w, S.HEADS_PAPER)
    zeroed = [[(np.zeros_like(W), b) for W, b in head] for head in heads]
    w0 = np.concatenate([np.concatenate([W.reshape(-1), b]) for head in zeroed for W, b in head])
    pos = S.uniform_positions(5)
    tables = np.zeros((S.GRID_PAPER.L, 4, S.GRID_PAPER.F), np.float32)   # never read: z is multiplied by zero
    grid = S.GridSpec(L=S.GRID_PAPER.L, F=4, log2_T=2, nmin_s=2, nmax_s=2, nmin_t=2, nmax_t=2, dtype="f32",
                      t_min=0.0, t_max=1.0)
    out = hd.decode_forward(pos, tables, w0, grid, S.HEADS_PAPER)
    np.testing.assert_allclose(out["scale"], math.exp(-5.0), rtol=1e-15)
    np.testing.assert_allclose(out["rot"], np.tile([1.0, 0.0, 0.0, 0.0], (5, 1)), atol=1e-15)
    # logit(0.1) ~ -2.197 is stored as fp16 (the paper configuration's weights): 0.1 to 4e-5
    np.testing.assert_allclose(out["opacity"], 0.1, rtol=1e-4)
    assert out["sh"].shape == (5, 48) and np.all(out["sh"] == 0.0)


def test_heads_are_independent():
    pos = S.uniform_positions(40, seed=2)
    tables = S.hash_tables(GRID, seed=3, scale=1.0)
    w = S.heads_weights(SPEC, seed=4, bias_scale=0.3).astype(np.float64)
    base = hd.decode_forward(pos, tables, w, GRID, SPEC)
    # perturb the SH head's first layer only (head 2 starts after heads 0 and 1)
    o = sum(oo * ii + oo for h in range(2) for oo, ii in SPEC.layer_shapes(h))
    w2 = w.copy()
    w2[o:o + 10] += 0.5
    out = hd.decode_forward(pos, tables, w2, GRID, SPEC)
    for k in ("scale", "rot", "opacity", "cov"):
        np.testing.assert_array_equal(out[k], base[k])
    assert np.max(np.abs(out["sh"] - base["sh"])) > 1e-3


def _loss(pos, tables, w, grads):
    out = hd.decode_forward(pos, tables, w, GRID, SPEC)
    return sum(np.sum(np.asarray(grads[k], np.float64) * out[k]) for k in grads)


def test_backward_matches_central_differences():
    n = 24
    pos = S.uniform_positions(n, seed=5)
    tables = S.hash_tables(GRID, seed=6, scale=1.0).astype(np.float64)
    w = S.heads_weights(SPEC, seed=7, bias_scale=0.3).astype(np.float64)
    widths = dict(S.HEADS_OUT_WIDTHS, sh=SPEC.sh_dim)
    grads = S.upstream_grads(n, widths, 1.0, seed=8)
    gt, gw = hd.decode_backward(pos, tables, w, GRID, SPEC, grads)
    h = 1e-6
    rng = np.random.default_rng(9)
    for p in rng.choice(w.size, 60, replace=False):
        e = np.zeros_like(w)
        e[p] = h
        fd = (_loss(pos, tables, w + e, grads) - _loss(pos, tables, w - e, grads)) / (2 * h)
        np.testing.assert_allclose(gw[p], fd, rtol=1e-6, atol=1e-8)
    # table entries the positions touch
    touched = np.argwhere(np.abs(gt) > 1e-6)
    for l, i, f in touched[rng.choice(len(touched), 40, replace=False)]:
        e = np.zeros_like(tables)
        e[l, i, f] = h
        fd = (_loss(pos, tables + e, w, grads) - _loss(pos, tables - e, w, grads)) / (2 * h)
        np.testing.assert_allclose(gt[l, i, f], fd, rtol=1e-6, atol=1e-8)


def test_learning_rate_schedule():
    lr = lambda s: hd.lr_warmup_cosine(s, 8e-3, 1e-7, 100, 1100)   # noqa: E731
    assert lr(0) == 0.0 and lr(50) == 4e-3 and lr(100) == 8e-3
    assert abs(lr(600) - (8e-3 + 1e-7) / 2) < 1e-15          # half-way down the cosine
    assert lr(1100) == 1e-7 and lr(5000) == 1e-7
    vals = [lr(s) for s in range(100, 1101)]
    assert all(a >= b for a, b in zip(vals, vals[1:]))


def test_scale_clip_at_twenty():
    """Eq. 11 with the page's clip: s = exp(min(s^, 20)), and no gradient to s^
    where the clip holds."""
    raw = dict(scale=np.array([[25.0, 19.0, 0.0]]), rot=np.array([[1.0, 0.0, 0.0, 0.0]]),
               sh=np.zeros((1, 12)), opacity=np.zeros((1, 1)))
    out = hd.activations(raw)
    np.testing.assert_allclose(out["scale"][0], [math.exp(20.0), math.exp(19.0), 1.0], rtol=1e-15)
    grads = dict(scale=np.ones((1, 3)), rot=np.zeros((1, 4)), sh=np.zeros((1, 12)), opacity=np.zeros((1, 1)),
                 cov=np.zeros((1, 6)))
    d = hd.activations_backward(raw, grads)["scale"][0]
    np.testing.assert_allclose(d, [0.0, math.exp(19.0), 1.0], rtol=1e-15)
