"""Pins for the oracle's normalisation and 4D hash encoder (CPU only).

Each test ties the oracle to something other than itself: values worked by
hand from the hash definition, the endpoints and growth the workload spec
fixes, the closed form of the Mip-NeRF contraction (SPIN-4DGS section 3.3,
Eq. 7), bijectivity of dense indexing, partition of unity and exact
reproduction of multilinear functions by quadrilinear interpolation, and
interpolation computed a second way (successive 1D lerps).
"""
import math
import os

import numpy as np
import pytest

from oracle import hashgrid as hg

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _hashed_index(v, log2_T, res=65):
    """Oracle index of vertex v on a hashed level (res-1 = 64 makes v/64 exact)."""
    resm = np.array([[res, res, res, res]])
    assert not hg.is_dense(resm[0], log2_T)
    xt = (np.array([v], np.float64) / (res - 1)).astype(F32)
    _, frac, idx = hg.corner_select(xt, resm, log2_T)
    assert np.all(frac == 0)
    return int(idx[0, 0, 0])


def test_hash_golden_values():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "hash_pins.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) >= 9
    for r in rows:
        log2_T, vx, vy, vz, vt, want = map(int, r)
        assert _hashed_index((vx, vy, vz, vt), log2_T) == want, r


def test_level_resolutions_endpoints_and_growth():
    # "spatial resolution 4 -> 32 (growth 2.0)" over 4 levels
    assert hg.level_resolutions(4, 4, 32) == [4, 8, 16, 32]
    # 16 levels 16 -> 2048 spatial and 8 -> 150 temporal: endpoints exact,
    # strictly increasing, each step within the floor of the geometric growth.
    for nmin, nmax in ((16, 2048), (8, 150)):
        r = hg.level_resolutions(16, nmin, nmax)
        assert r[0] == nmin and r[-1] == nmax
        b = (nmax / nmin) ** (1 / 15)
        for l in range(16):
            assert r[l] <= nmin * b ** l + 1e-6 < r[l] + 1
        assert all(a < c for a, c in zip(r, r[1:]))


@pytest.mark.parametrize("L,nmin_s,nmax_s,nmin_t,nmax_t,log2_T,dense_levels", [
    (4, 4, 32, 4, 32, 12, [0, 1]),            # 8^4 = 4096 = T is still dense
    (16, 16, 2048, 8, 150, 19, [0, 1, 2]),
    (16, 16, 2048, 8, 150, 22, [0, 1, 2, 3, 4]),
])
def test_dense_levels(L, nmin_s, nmax_s, nmin_t, nmax_t, log2_T, dense_levels):
    res = hg.grid_resolutions(L, nmin_s, nmax_s, nmin_t, nmax_t)
    got = [l for l in range(L) if hg.is_dense(res[l], log2_T)]
    assert got == dense_levels


def _all_vertices(res_l):
    axes = [np.arange(int(r)) for r in res_l]
    g = np.stack(np.meshgrid(*axes, indexing="ij"), -1).reshape(-1, 4)
    return g


def test_dense_index_is_bijection_with_x_fastest():
    res = np.array([[4, 4, 4, 4], [8, 8, 8, 8]])
    for l in range(2):
        r = res[l:l + 1]
        v = _all_vertices(r[0])
        # put every vertex in corner 0 via exact coordinates v/(res-1) ... for
        # the last vertex per axis use corner bit 1 of the previous cell.
        xt = (v / (r[0] - 1)).astype(F32)
        base, frac, idx = hg.corner_select(xt, r, 12)
        # vertex actually addressed: base + (frac == 1)
        got = np.empty(len(v), np.int64)
        for n in range(len(v)):
            c = sum(1 << d for d in range(4) if frac[n, 0, d] == 1)
            assert np.all((frac[n, 0] == 0) | (frac[n, 0] == 1))
            got[n] = idx[n, 0, c]
        assert sorted(got.tolist()) == list(range(int(np.prod(r[0]))))
        # x-neighbours are adjacent entries
        assert np.all(idx[:, 0, 1].astype(np.int64) - idx[:, 0, 0] == 1)


def _inverse_dense(e, res_l):
    rx, ry, rz, rt = (int(x) for x in res_l)
    return np.stack([e % rx, (e // rx) % ry, (e // (rx * ry)) % rz, e // (rx * ry * rz)], -1)


def test_partition_of_unity_all_levels():
    res = hg.grid_resolutions(4, 4, 32, 4, 32)
    rng = np.random.default_rng(1)
    xt = rng.random((500, 4)).astype(F32)
    tables = np.ones((4, 1 << 12, 2), np.float32)
    z = hg.encode(xt, tables, res, 12)
    np.testing.assert_allclose(z, 1.0, rtol=0, atol=1e-14)


def test_multilinear_function_reproduced_at_dense_levels():
    """Table value = a . v + b + c * v_x * v_t at every vertex (v recovered by
    div/mod, the inverse of dense indexing): quadrilinear interpolation must
    return the same multilinear function at p = x~ * (res - 1)."""
    res = hg.grid_resolutions(4, 4, 32, 4, 32)
    T = 1 << 12
    a = np.array([0.3, -1.7, 2.5, 0.9])
    tables = np.zeros((4, T, 1), np.float64)
    for l in range(2):                               # dense levels only
        n = int(np.prod(res[l]))
        v = _inverse_dense(np.arange(n), res[l]).astype(np.float64)
        tables[l, :n, 0] = v @ a + 0.25 + 0.125 * v[:, 0] * v[:, 3]
    rng = np.random.default_rng(2)
    xt = rng.random((400, 4)).astype(F32)
    z = hg.encode(xt, tables, res, 12)
    for l in range(2):
        p = xt.astype(F32) * (res[l] - 1).astype(F32)        # fp32 like the cell decision
        p = p.astype(np.float64)
        want = p @ a + 0.25 + 0.125 * p[:, 0] * p[:, 3]
        np.testing.assert_allclose(z[:, l], want, rtol=1e-12, atol=1e-12)


def test_interpolation_equals_successive_lerps_on_hashed_levels():
    """Quadrilinear weights vs four nested 1D linear interpolations."""
    res = hg.grid_resolutions(4, 4, 32, 4, 32)
    rng = np.random.default_rng(3)
    tables = rng.standard_normal((4, 1 << 12, 2))
    xt = rng.random((64, 4)).astype(F32)
    z = hg.encode(xt, tables, res, 12)
    base, frac, idx = hg.corner_select(xt, res, 12)
    for l in (2, 3):
        for n in range(64):
            vals = tables[l, idx[n, l].astype(np.int64), :]          # 16 x F, bit0 = x
            w = frac[n, l].astype(np.float64)
            cube = vals.reshape(2, 2, 2, 2, -1)                        # [t][z][y][x]
            for d, ax in ((0, 3), (1, 2), (2, 1), (3, 0)):            # lerp x, y, z, t
                lo = np.take(cube, 0, axis=ax)
                hi = np.take(cube, 1, axis=ax)
                cube = lo + w[d] * (hi - lo)
            np.testing.assert_allclose(z[n, l * 2:(l + 1) * 2], cube.reshape(-1), rtol=1e-12, atol=1e-13)


def test_vertex_lookup_returns_table_entry():
    """At an exact vertex, encode returns that vertex's entry (one weight is 1)."""
    res = np.array([[65, 65, 65, 65], [5, 5, 5, 5]])     # hashed level, then dense level
    T = 1 << 12
    tables = np.zeros((2, T, 2), np.float32)
    tables[:, :, 0] = np.arange(T)
    tables[:, :, 1] = -np.arange(T) * 0.5
    v = np.array([[17, 0, 9, 3], [3, 5, 7, 2], [63, 63, 63, 63], [1, 1, 1, 1]])
    xt = (v / 64.0).astype(F32)
    z = hg.encode(xt, tables, res, 12)
    for n in range(len(v)):
        e = _hashed_index(tuple(v[n]), 12)
        assert z[n, 0] == e and z[n, 1] == -0.5 * e
    # level 1 (dense, res 5 -> scale 4): x~ = v/64 is a vertex only when v % 16 == 0
    xt2 = (np.array([[0, 16, 32, 48], [64, 64, 0, 16]]) / 64.0).astype(F32)
    z2 = hg.encode(xt2, tables, res, 12)
    for n, vv in enumerate([[0, 1, 2, 3], [4, 4, 0, 1]]):
        e = vv[0] + 5 * (vv[1] + 5 * (vv[2] + 5 * vv[3]))
        assert z2[n, 2] == e


def test_hash_pairs_even_x_neighbours():
    """With prime 1 on x, vertices x and x+1 (x even) land in entries e, e^1."""
    rng = np.random.default_rng(4)
    v = rng.integers(0, 32, size=(200, 4)) * np.array([2, 1, 1, 1])
    v = np.minimum(v, 62)
    xt = (v / 64.0).astype(F32)
    _, _, idx = hg.corner_select(xt, np.array([[65, 65, 65, 65]]), 19)
    assert np.all(idx[:, 0, 1] == (idx[:, 0, 0] ^ 1))


# ---------------------------------------------------------------------------
# Eq. 7 / Eq. 8
# ---------------------------------------------------------------------------
def _contract_back(xt):
    return (xt[:, :3].astype(np.float64) - 0.5) * 4.0


def test_contraction_identity_inside_unit_ball():
    rng = np.random.default_rng(5)
    d = rng.standard_normal((1000, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    mu = d * rng.random((1000, 1)) * 0.999
    pos = np.concatenate([mu, np.zeros((1000, 1))], 1).astype(F32)
    xt = hg.normalise(pos, 0.0, 1.0)
    np.testing.assert_allclose(_contract_back(xt), pos[:, :3], rtol=0, atol=2e-7)


def test_contraction_closed_form_outside():
    rng = np.random.default_rng(6)
    d = rng.standard_normal((1000, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    r = 1.0 + rng.random((1000, 1)) * 50.0
    mu = (d * r).astype(F32)
    pos = np.concatenate([mu, np.zeros((1000, 1), F32)], 1)
    c = _contract_back(hg.normalise(pos, 0.0, 1.0))
    n = np.linalg.norm(mu.astype(np.float64), axis=1)
    # ||contract(mu)|| = 2 - 1/||mu|| and the direction is kept
    np.testing.assert_allclose(np.linalg.norm(c, axis=1), 2 - 1 / n, rtol=0, atol=3e-6)
    cosang = np.sum(c * mu, 1) / (np.linalg.norm(c, axis=1) * n)
    assert np.all(cosang > 1 - 1e-6)
    assert np.all(np.linalg.norm(c, axis=1) < 2.0)


def test_contraction_continuous_at_unit_norm_and_bounded():
    d = np.array([[0.6, 0.0, 0.8], [0.0, 1.0, 0.0]])
    eps = 1e-4
    a = np.concatenate([d * (1 - eps), np.zeros((2, 1))], 1).astype(F32)
    b = np.concatenate([d * (1 + eps), np.zeros((2, 1))], 1).astype(F32)
    ca, cb = _contract_back(hg.normalise(a, 0, 1)), _contract_back(hg.normalise(b, 0, 1))
    assert np.max(np.abs(ca - cb)) < 4 * eps
    # (squares stay below fp32 overflow: beyond |mu| ~ 1.8e19 the fp32 norm is inf)
    far = np.array([[1e15, -1e15, 3e14, 0.0], [-7e18, 0.0, 0.0, 0.0]], F32)
    xt = hg.normalise(far, 0, 1)
    assert np.all((xt >= 0) & (xt <= 1))
    np.testing.assert_allclose(np.linalg.norm(_contract_back(xt), axis=1), 2.0, atol=1e-6)


def test_time_normalisation():
    pos = np.zeros((6, 4), F32)
    pos[:, 3] = [0, 149, 75, -3, 200, 74.5]
    xt = hg.normalise(pos, 0.0, 149.0)
    assert xt[0, 3] == 0.0 and xt[1, 3] == 1.0 and xt[3, 3] == 0.0 and xt[4, 3] == 1.0
    assert xt[2, 3] == F32(75) / F32(149)
    assert abs(float(xt[5, 3]) - 0.5) < 1e-7
    # identity on [0,1] for t_min = 0, t_max = 1
    t = np.linspace(0, 1, 11, dtype=F32)
    p2 = np.zeros((11, 4), F32)
    p2[:, 3] = t
    assert np.array_equal(hg.normalise(p2, 0.0, 1.0)[:, 3], t)


def test_upper_boundary_last_cell_weight_one():
    res = np.array([[4, 8, 16, 32]])
    base, frac, _ = hg.corner_select(np.ones((1, 4), F32), res, 12)
    assert base[0, 0].tolist() == [2, 6, 14, 30] and np.all(frac == 1)
    base, frac, _ = hg.corner_select(np.zeros((1, 4), F32), res, 12)
    assert base[0, 0].tolist() == [0, 0, 0, 0] and np.all(frac == 0)


def test_nan_coordinate_treated_as_zero():
    pos = np.array([[np.nan, 0.0, 0.0, np.nan]], F32)
    xt = hg.normalise(pos, 0, 1)
    assert np.all(np.isfinite(xt))
    assert xt[0, 3] == 0.0
