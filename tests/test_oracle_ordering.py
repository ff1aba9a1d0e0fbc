"""Pins of the Morton-ordering oracle: hand-worked codes, the defining
properties of the Z-order curve, and the sort against its definition."""
import numpy as np

from oracle import ordering as od


def test_interleave_hand_worked():
    q = np.array([[1, 0, 0], [0, 1, 0], [0, 0, 1], [1, 1, 1], [3, 3, 3], [2, 0, 0], [1023, 1023, 1023],
                  [5, 3, 6]])
    # [5,3,6]: x=101 y=011 z=110 -> bits (b0: x1 y1 z0)(b1: x0 y1 z1)(b2: x1 y0 z1) = 101 110 011 (b2 b1 b0)
    want = [1, 2, 4, 7, 63, 8, (1 << 30) - 1, 0b101110011]
    assert od.interleave(q).tolist() == want


def test_quantise_edges():
    x = np.array([[0.0, 0.5, 1.0], [1 / 1024, 1023 / 1024, 0.9999999]], np.float32)
    assert od.quantise(x).tolist() == [[0, 512, 1023], [1, 1023, 1023]]


def test_z_order_locality_and_monotonicity():
    rng = np.random.default_rng(0)
    q = rng.integers(0, 1024, size=(5000, 3))
    k = od.interleave(q).astype(np.int64)
    # keys are monotone in each axis separately (the other two fixed)
    for d in range(3):
        q2 = q.copy()
        q2[:, d] = np.minimum(q2[:, d] + 1, 1023)
        assert np.all(od.interleave(q2).astype(np.int64) >= k)
    # an aligned 2^j cube is one contiguous key range of length 8^j
    base = (q >> 4) << 4
    lo = od.interleave(base).astype(np.int64)
    assert np.all((k - lo >= 0) & (k - lo < 8 ** 4))


def test_order_is_a_stable_sort():
    keys = np.array([5, 3, 5, 0, 3, 3, 7], np.uint32)
    assert od.morton_order(keys).tolist() == [3, 1, 4, 5, 0, 2, 6]


def test_keys_of_raw_positions():
    """Through Eq. 7: inside the unit ball mu_bar = mu/4 + 1/2, so mu = (0.25, 0, -0.5)
    and the origin have known cells; the timestamp does not enter the key."""
    pos = np.array([[0.25, 0.0, -0.5, 0.0], [0.25, 0.0, -0.5, 0.9], [0.0, 0.0, 0.0, 0.3]], np.float32)
    keys = od.morton_keys(pos, 0.0, 1.0)
    # (0.25, 0, -0.5) -> mu_bar (0.5625, 0.5, 0.375) -> q (576, 512, 384)
    want = od.interleave(np.array([[576, 512, 384]]))[0]
    assert keys[0] == want and keys[1] == want
    assert keys[2] == od.interleave(np.array([[512, 512, 512]]))[0]
