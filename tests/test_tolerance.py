"""The parity checker itself (CPU only): the element-wise bound with the
magnitude term admits a result that differs from the oracle only by fp32
rounding, and rejects plausible mistakes, including ones confined to a
single fine hash level, one position, or one weight block.

The mistakes are planted in the oracle's own arithmetic on the CPU (its
adjoint dz is scattered with a wrong corner weight, a position is dropped, an
entry moved to its neighbour, a block transposed or off by 3 %)."""
import numpy as np
import pytest

from oracle import decoder as dec
from oracle import hashgrid as hg
from spatiotemporal_neural_field_b200 import synthetic as S
from tests import magnitude as mag
from tests import tol


def _case(n=3000):
    w = S.WORKLOADS["sports_frame_fp16"]
    grid, mlp = w["grid"], w["mlp"]
    pos = S.sports_scene(300_000).frame(75)[:n]
    tables = S.hash_tables(grid, scale=1.0)
    weights = S.mlp_weights(mlp, bias_scale=0.5)
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, 1e-2)
    wt, ww = dec.decode_backward(pos, tables, weights, grid, mlp, grads)
    rho = mag.decoder_rss(pos, tables, weights, grid, mlp, grads)
    return grid, mlp, pos, tables, weights, grads, wt, ww, rho


@pytest.fixture(scope="module")
def case():
    return _case()


def _check(got_t, got_w, grid, mlp, wt, ww, rho, rtol=tol.FP16_GRAD_RTOL):
    tol.elementwise(got_t, wt, rtol, "grad_tables", tol.table_levels(grid.L, 1 << grid.log2_T, grid.F), rho=rho[0])
    tol.elementwise(got_w, ww, rtol, "grad_weights", tol.weight_blocks(mlp.layer_shapes()), rho=rho[1])


def _dz(pos, tables, weights, grid, mlp, grads):
    """The oracle's latent adjoint, from its own pieces."""
    res, xt = dec._prepare(pos, grid, False)
    z = hg.encode(xt, tables, res, grid.log2_T)
    layers = dec.unpack_layers(weights, mlp.layer_shapes())
    y, acts, pres = dec.mlp_forward(z, layers)
    dy = dec.heads_backward(y, {k: np.asarray(v, np.float64) for k, v in grads.items()})
    dz, _ = dec.mlp_backward(dy, layers, acts, pres)
    return res, xt, dz


def test_fp32_rounding_of_the_oracle_passes(case):
    grid, mlp, _, _, _, _, wt, ww, rho = case
    _check(wt.astype(np.float32), ww.astype(np.float32), grid, mlp, wt, ww, rho)
    _check(wt.astype(np.float32), ww.astype(np.float32), grid, mlp, wt, ww, rho, tol.FP32_GRAD_RTOL)


def test_wrong_index_on_one_fine_level_fails(case):
    grid, mlp, _, _, _, _, wt, ww, rho = case
    got = wt.copy()
    l = grid.L - 2
    e = np.flatnonzero(np.any(got[l] != 0, axis=1))[17]
    got[l, e + 1], got[l, e] = got[l, e].copy(), got[l, e + 1].copy()
    with pytest.raises(AssertionError, match="level %d" % l):
        _check(got, ww, grid, mlp, wt, ww, rho)


def test_dropped_position_fails(case):
    grid, mlp, pos, tables, weights, grads, wt, ww, rho = case
    keep = np.ones(len(pos), bool)
    keep[1234] = False
    gt, gw = dec.decode_backward(pos[keep], tables, weights, grid, mlp, {k: v[keep] for k, v in grads.items()})
    with pytest.raises(AssertionError, match="grad_tables"):
        _check(gt, gw, grid, mlp, wt, ww, rho)


def test_flipped_time_weight_on_the_finest_level_fails(case):
    """The scatter of the last level uses 1 - w for w on the time axis."""
    grid, mlp, pos, tables, weights, grads, wt, ww, rho = case
    res, xt, dz = _dz(pos, tables, weights, grid, mlp, grads)
    bad = xt.copy()
    l = grid.L - 1
    rt = int(res[l, 3])
    # mirror t inside its cell: p -> base + (1 - frac), i.e. the time weights swap
    p = xt[:, 3] * np.float32(rt - 1)
    base = np.clip(np.floor(p), 0, rt - 2)
    bad[:, 3] = ((base + (1.0 - (p - base))) / (rt - 1)).astype(np.float32)
    got = wt.copy()
    got[l] = hg.scatter_table_grad(dz, bad, res, grid.log2_T, grid.L, grid.F)[l]
    with pytest.raises(AssertionError, match="level %d" % l):
        _check(got, ww, grid, mlp, wt, ww, rho)


def test_transposed_block_fails(case):
    grid, mlp, _, _, _, _, wt, ww, rho = case
    got = ww.copy()
    (m, k) = mlp.layer_shapes()[1]          # the square 64 x 64 layer
    o = m * mlp.layer_shapes()[0][1] + m     # after W0 and b0
    got[o:o + m * k] = got[o:o + m * k].reshape(m, k).T.reshape(-1)
    with pytest.raises(AssertionError, match="W1"):
        _check(wt, got, grid, mlp, wt, ww, rho)


def test_three_percent_error_on_one_block_fails(case):
    grid, mlp, _, _, _, _, wt, ww, rho = case
    got = ww.copy()
    m, k = mlp.layer_shapes()[0]
    got[:m * k] *= 1.03
    with pytest.raises(AssertionError, match="W0"):
        _check(wt, got, grid, mlp, wt, ww, rho)


def test_fp32_bound_rejects_a_relative_error_of_1e_4():
    """The fp32 path's bound: the tiny decoder's gradients off by 1e-4."""
    w = S.WORKLOADS["tiny_fp32"]
    grid, mlp = w["grid"], w["mlp"]
    n = 4099
    pos = S.uniform_positions(n)
    tables = S.hash_tables(grid, scale=1.0)
    weights = S.mlp_weights(mlp, bias_scale=0.5)
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, 1.0)
    wt, ww = dec.decode_backward(pos, tables, weights, grid, mlp, grads)
    rho = mag.decoder_rss(pos, tables, weights, grid, mlp, grads)
    _check(wt.astype(np.float32), ww.astype(np.float32), grid, mlp, wt, ww, rho, tol.FP32_GRAD_RTOL)
    with pytest.raises(AssertionError):
        _check(wt * (1 + 1e-4), ww, grid, mlp, wt, ww, rho, tol.FP32_GRAD_RTOL)
    with pytest.raises(AssertionError):
        _check(wt, ww * (1 + 1e-4), grid, mlp, wt, ww, rho, tol.FP32_GRAD_RTOL)
