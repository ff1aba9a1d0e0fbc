"""GPU parity of the Z-order ordering: keys bit-exact, the permutation equal
to the stable sort of the oracle's keys, row permutation exact, and the
decoder's outputs in sorted order equal to the permuted outputs (B200 only)."""
import numpy as np
import pytest

from oracle import ordering as od
from spatiotemporal_neural_field_b200 import synthetic as S

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sp():
    from spatiotemporal_neural_field_b200 import spin4d
    return spin4d


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def _check(sp, grid, pos, normalised=False):
    g = sp.grid_from_spec(grid)
    if normalised:
        g.flags |= sp.INPUT_NORMALISED
    keys, perm = sp.morton_order(g, dev(pos))
    want_keys = od.morton_keys(pos, grid.t_min, grid.t_max, normalised_input=normalised)
    want_perm = od.morton_order(want_keys)
    assert np.array_equal(u32(perm), want_perm)
    assert np.array_equal(u32(keys), want_keys[want_perm])
    return perm


@pytest.mark.parametrize("n", [1, 3, 2047, 2048, 2049, 70001])
def test_morton_order_uniform(sp, n):
    pos = S.uniform_positions(n, seed=n)
    pos[:, :3] *= 1.7                      # inside and outside the unit ball
    _check(sp, S.GRID_TINY, pos)


def test_morton_order_sports_frame_full_size(sp):
    w = S.WORKLOADS["sports_frame_fp16"]
    _check(sp, w["grid"], S.sports_scene(w["N"]).frame(w["frame"]))


def test_morton_order_stress_full_size(sp):
    w = S.WORKLOADS["stress_fp16_gate"]
    _check(sp, w["grid"], S.stress_positions(w["N"]))


def test_morton_order_ties_and_edges(sp):
    n = 5000
    pos = np.zeros((n, 4), np.float32)     # all equal: the stable order is the identity
    perm = _check(sp, S.GRID_TINY, pos)
    assert np.array_equal(u32(perm), np.arange(n, dtype=np.uint32))
    pos = S.uniform_positions(n, seed=9)
    pos[::7, 0] = np.nan
    pos[1::7, :3] = 1e30
    pos[2::7, :3] = -1e30
    _check(sp, S.GRID_TINY, pos)
    xt = np.random.default_rng(3).uniform(-0.2, 1.2, size=(n, 4)).astype(np.float32)
    _check(sp, S.GRID_TINY, xt, normalised=True)


@pytest.mark.parametrize("cols,dtype", [(1, np.float32), (3, np.float32), (4, np.float32), (16, np.float32),
                                        (2, np.int32)])
def test_permute_rows(sp, cols, dtype):
    rng = np.random.default_rng(cols)
    n = 9001
    src = rng.normal(size=(n, cols)).astype(dtype) if dtype == np.float32 else rng.integers(-9, 9, (n, cols)).astype(dtype)
    perm = rng.permutation(n).astype(np.int32)
    out = sp.permute_rows(dev(src), dev(perm))
    assert np.array_equal(out.cpu().numpy(), src[perm])


def test_decode_in_sorted_order_is_the_permuted_decode(sp):
    w = S.WORKLOADS["sports_frame_fp16"]
    grid, mlp = w["grid"], w["mlp"]
    n = 50_000
    pos = S.sports_scene(n).frame(w["frame"])
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    P, T, W = dev(pos), dev(S.hash_tables(grid)), dev(S.mlp_weights(mlp, bias_scale=0.5))
    _, perm = sp.morton_order(g, P)
    Ps = sp.permute_rows(P, perm)
    a = sp.decode_fwd(g, m, P, T, W)
    b = sp.decode_fwd(g, m, Ps, T, W)
    idx = perm.long()
    for k in a:
        assert torch.equal(b[k], a[k][idx]), k
