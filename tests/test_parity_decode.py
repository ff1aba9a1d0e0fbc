"""GPU parity of the hash-grid decoder against the CPU oracle (B200 only).

Every call goes through the C ABI (ctypes binding).  Inputs are the seeded
synthetic workloads; the oracle sees exactly the same arrays.  Sizes are
chosen so the oracle finishes in seconds yet every kernel runs many tiles
and a ragged tail; the full-size workloads are checked on sampled rows.
"""
import numpy as np
import pytest

from oracle import decoder as dec
from oracle import hashgrid as hg
from spatiotemporal_neural_field_b200 import synthetic as S
from tests import magnitude as mag
from tests import tol

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
KEYS = ("scale", "rot", "rgb", "opacity", "cov")


@pytest.fixture(scope="module")
def sp():
    from spatiotemporal_neural_field_b200 import spin4d
    return spin4d


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def _positions(kind, n, seed=0):
    if kind == "uniform":
        return S.uniform_positions(n, seed)
    if kind == "sports":
        # a seeded subset of frame 75: static background and the moving blobs
        frame = S.sports_scene(300_000, seed).frame(75)
        return frame[np.random.default_rng(seed + 9).choice(len(frame), n, replace=False)]
    if kind == "stress":
        return S.stress_positions(n, seed)
    raise ValueError(kind)


def _edge_positions():
    """Outside the unit ball, far away, on the axes, at the origin, t out of range, NaN."""
    p = np.array([
        [0, 0, 0, 0.5], [1, 0, 0, 0], [0, -1, 0, 1], [0, 0, 1, 0.25], [3, 4, 12, 0.9], [-1e6, 2e6, 5e5, 0.1],
        [0.5773503, 0.5773503, 0.5773503, 0.3], [1.0000001, 0, 0, 0.3], [0.9999999, 0, 0, 0.3],
        [0.2, 0.3, 0.1, -5.0], [0.2, 0.3, 0.1, 7.0], [np.nan, 0.1, 0.2, 0.3], [0.1, 0.2, 0.3, np.nan],
        [1e15, -1e15, 3e14, 0.6],
    ], np.float32)
    return p


# ---------------------------------------------------------------------------
# corner selection: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("grid,kind,n", [(S.GRID_TINY, "uniform", 4096), (S.GRID_SPORTS, "sports", 20011),
                                         (S.GRID_STRESS, "stress", 20011)])
def test_corner_indices_bit_exact(sp, grid, kind, n):
    pos = np.concatenate([_positions(kind, n), _edge_positions()])
    if grid.t_max > 1:
        pos[-14:, 3] *= grid.t_max
    g = sp.grid_from_spec(grid)
    idx, frac = sp.debug_corners(g, dev(pos))
    res = hg.grid_resolutions(grid.L, grid.nmin_s, grid.nmax_s, grid.nmin_t, grid.nmax_t)
    xt = hg.normalise(pos, grid.t_min, grid.t_max)
    _, ofrac, oidx = hg.corner_select(xt, res, grid.log2_T)
    assert np.array_equal(host(idx).view(np.uint32), oidx)
    assert np.array_equal(host(frac), ofrac)


def test_corner_indices_normalised_input_vertices(sp):
    """x~ given directly (flag set): exact vertices of every level."""
    grid = S.GRID_TINY
    g = sp.grid_from_spec(grid, normalised_input=True)
    rng = np.random.default_rng(3)
    xt = rng.random((5000, 4)).astype(np.float32)
    xt[:100] = (rng.integers(0, 32, size=(100, 4)) / 31.0).astype(np.float32)
    xt[100:110] = 1.0
    xt[110:120] = 0.0
    idx, frac = sp.debug_corners(g, dev(xt))
    res = hg.grid_resolutions(grid.L, grid.nmin_s, grid.nmax_s, grid.nmin_t, grid.nmax_t)
    _, ofrac, oidx = hg.corner_select(hg._clamp01(xt), res, grid.log2_T)
    assert np.array_equal(host(idx).view(np.uint32), oidx)
    assert np.array_equal(host(frac), ofrac)


# ---------------------------------------------------------------------------
# encode
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("grid,kind,n,scale", [(S.GRID_TINY, "uniform", 4096, 1e-4), (S.GRID_TINY, "uniform", 4099, 1.0),
                                               (S.GRID_SPORTS, "sports", 30001, 1.0),
                                               (S.GRID_STRESS, "stress", 10007, 1.0)])
def test_encode_matches_oracle(sp, grid, kind, n, scale):
    pos = _positions(kind, n)
    tables = S.hash_tables(grid, scale=scale)
    g = sp.grid_from_spec(grid)
    z = host(sp.encode_fwd(g, dev(pos), dev(tables)))
    res = hg.grid_resolutions(grid.L, grid.nmin_s, grid.nmax_s, grid.nmin_t, grid.nmax_t)
    xt = hg.normalise(pos, grid.t_min, grid.t_max)
    want = hg.encode(xt, tables, res, grid.log2_T)
    # fp32 accumulation of exactly-read table values: per-level 16-term sums,
    # held to the terms' root-sum-square where they cancel
    tol.elementwise(z, want, tol.FP32_RTOL, "z", tol.column_groups(grid.L * grid.F),
                    rho=mag.encode_mag(xt, tables, res, grid.log2_T))


# ---------------------------------------------------------------------------
# decode forward
# ---------------------------------------------------------------------------
def check_fp32_outputs(got, want, keys=KEYS, tag="", extra_mag=None):
    """fp32 attributes, element-wise per attribute.  A rotation component is
    r^_k / ||r^||, rounded relative to the unit row norm, so its magnitude is
    1; a covariance entry is computed from R's O(1) entries, so its
    magnitude is the spectral norm max_k s_k^2 (tests/magnitude.py);
    ``extra_mag`` gives the magnitudes of further keys."""
    for k in keys:
        rho = None
        if k == "rot":
            rho = np.ones_like(want[k])
        elif k == "cov":
            rho = mag.cov_mag(want["scale"])
        elif extra_mag and k in extra_mag:
            rho = extra_mag[k]
        tol.elementwise(got[k], want[k], tol.FP32_RTOL, tag + k, rho=rho)


def _check_outputs(out, want, fp32: bool):
    if fp32:
        check_fp32_outputs({k: host(out[k]) for k in KEYS}, want)
    else:
        for k in KEYS:
            tol.absolute(host(out[k]), want[k], tol.FP16_ATOL, k)
    np.testing.assert_allclose(np.linalg.norm(host(out["rot"]), axis=1), 1.0, atol=1e-5)


CASES = {
    "tiny_spec_init": ("tiny_fp32", 4096, 1e-4, 0.0),
    "tiny_stress_init": ("tiny_fp32", 4099, 1.0, 0.5),
    "sports_spec_init": ("sports_frame_fp16", 20011, 1e-4, 0.0),
    "sports_stress_init": ("sports_frame_fp16", 20011, 1.0, 0.5),
    "stress_gate": ("stress_fp16_gate", 8009, 1.0, 0.5),
}


def _workload(name, n, tscale, bscale):
    w = S.WORKLOADS[name]
    grid, mlp = w["grid"], w["mlp"]
    kind = {"tiny_fp32": "uniform", "sports_frame_fp16": "sports", "stress_fp16_gate": "stress"}[name]
    pos = _positions(kind, n)
    tables = S.hash_tables(grid, scale=tscale)
    weights = S.mlp_weights(mlp, bias_scale=bscale)
    cr = S.gate_params(n) if mlp.gate else None
    return grid, mlp, pos, tables, weights, cr


@pytest.mark.parametrize("case", list(CASES))
def test_decode_fwd_matches_oracle(sp, case):
    grid, mlp, pos, tables, weights, cr = _workload(*CASES[case])
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    out = sp.decode_fwd(g, m, dev(pos), dev(tables), dev(weights), dev(cr) if cr is not None else None)
    want = dec.decode_forward(pos, tables, weights, grid, mlp, gate_cr=cr)
    _check_outputs(out, want, grid.dtype == "f32")


def test_decode_fwd_edge_positions(sp):
    grid, mlp, _, tables, weights, _ = _workload("tiny_fp32", 16, 1.0, 0.5)
    pos = _edge_positions()
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    for n in (1, 3, len(pos)):
        out = sp.decode_fwd(g, m, dev(pos[:n]), dev(tables), dev(weights))
        want = dec.decode_forward(pos[:n], tables, weights, grid, mlp)
        _check_outputs(out, want, True)


def test_decode_fwd_full_size_sampled(sp):
    """The full 300k sports frame in one launch; 3000 sampled rows vs the oracle."""
    w = S.WORKLOADS["sports_frame_fp16"]
    grid, mlp = w["grid"], w["mlp"]
    pos = S.sports_scene(300_000).frame(75)
    tables = S.hash_tables(grid, scale=1.0)
    weights = S.mlp_weights(mlp, bias_scale=0.5)
    out = sp.decode_fwd(sp.grid_from_spec(grid), sp.mlp_from_spec(mlp), dev(pos), dev(tables), dev(weights))
    rows = np.sort(np.random.default_rng(0).choice(len(pos), 3000, replace=False))
    rows[-1] = len(pos) - 1
    want = dec.decode_forward(pos[rows], tables, weights, grid, mlp)
    for k in KEYS:
        tol.absolute(host(out[k])[rows], want[k], tol.FP16_ATOL, k)


def test_decode_fwd_stress_full_size_sampled(sp):
    """4M positions, 512 MiB of fp16 tables, gated opacity: sampled rows."""
    w = S.WORKLOADS["stress_fp16_gate"]
    grid, mlp = w["grid"], w["mlp"]
    n = w["N"]
    pos = S.stress_positions(n)
    tables = S.hash_tables(grid, scale=1.0)
    weights = S.mlp_weights(mlp, bias_scale=0.5)
    cr = S.gate_params(n)
    out = sp.decode_fwd(sp.grid_from_spec(grid), sp.mlp_from_spec(mlp), dev(pos), dev(tables), dev(weights), dev(cr))
    rows = np.sort(np.random.default_rng(1).choice(n, 2000, replace=False))
    rows[-1] = n - 1
    want = dec.decode_forward(pos[rows], tables, weights, grid, mlp, gate_cr=cr[rows])
    for k in KEYS:
        tol.absolute(host(out[k])[rows], want[k], tol.FP16_ATOL, k)


# ---------------------------------------------------------------------------
# decode backward
# ---------------------------------------------------------------------------
BWD_CASES = {
    "tiny_spec": ("tiny_fp32", 4096, 1e-4, 0.0, 1.0),
    "tiny_stress": ("tiny_fp32", 4099, 1.0, 0.5, 1.0),
    "sports": ("sports_frame_fp16", 20011, 1.0, 0.5, 1e-2),
    # initial state: 1e-4 tables, so latent and activations are ~1e-5 (fp16-subnormal unless rescaled)
    "sports_spec_init": ("sports_frame_fp16", 20011, 1e-4, 0.0, 1e-2),
    "stress_gate": ("stress_fp16_gate", 6007, 1.0, 0.5, 1.0),
}


def check_decode_grads(gt, gw, wt, ww, grid, mlp, rtol, rho=(None, None), tag=""):
    """Element-wise per table level and per weight block (see tests/tol.py)."""
    tol.elementwise(gt, wt, rtol, tag + "grad_tables", tol.table_levels(grid.L, 1 << grid.log2_T, grid.F),
                    rho=rho[0])
    tol.elementwise(gw, ww, rtol, tag + "grad_weights", tol.weight_blocks(mlp.layer_shapes()), rho=rho[1])


def _bwd(sp, grid, mlp, pos, tables, weights, cr, grads):
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), dtype=torch.float32, device="cuda")
    gw = torch.zeros(mlp.n_params(), dtype=torch.float32, device="cuda")
    sp.decode_bwd(g, m, dev(pos), dev(tables), dev(weights), {k: dev(v) for k, v in grads.items()}, gt, gw,
                  gate_cr=dev(cr) if cr is not None else None)
    return host(gt), host(gw)


@pytest.mark.parametrize("case", list(BWD_CASES))
def test_decode_bwd_matches_oracle(sp, case):
    name, n, tscale, bscale, gstd = BWD_CASES[case]
    grid, mlp, pos, tables, weights, cr = _workload(name, n, tscale, bscale)
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, gstd)
    gt, gw = _bwd(sp, grid, mlp, pos, tables, weights, cr, grads)
    wt, ww = dec.decode_backward(pos, tables, weights, grid, mlp, grads, gate_cr=cr)
    rtol = tol.FP32_GRAD_RTOL if grid.dtype == "f32" else tol.FP16_GRAD_RTOL
    check_decode_grads(gt, gw, wt, ww, grid, mlp, rtol,
                       mag.decoder_rss(pos, tables, weights, grid, mlp, grads, gate_cr=cr))


@pytest.mark.parametrize("name,n", [("sports_frame_fp16", 20011), ("stress_fp16_gate", 3001)])
def test_decode_bwd_covariance_only_gradient(sp, name, n):
    """Upstream gradient on Sigma alone: Sigma ~ s^2 ~ 1e-5, so the gradients
    that reach the network are ~1e-7..1e-9, far below fp16's normal range."""
    grid, mlp, pos, tables, weights, cr = _workload(name, n, 1.0, 0.5)
    full = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, 1e-2)
    grads = {"cov": full["cov"]}
    gt, gw = _bwd(sp, grid, mlp, pos, tables, weights, cr, grads)
    zeros = {k: np.zeros_like(v) for k, v in full.items()}
    zeros["cov"] = full["cov"]
    wt, ww = dec.decode_backward(pos, tables, weights, grid, mlp, zeros, gate_cr=cr)
    check_decode_grads(gt, gw, wt, ww, grid, mlp, tol.FP16_GRAD_RTOL,
                       mag.decoder_rss(pos, tables, weights, grid, mlp, zeros, gate_cr=cr))


@pytest.mark.parametrize("name,n", [("tiny_fp32", 4099), ("sports_frame_fp16", 20011), ("stress_fp16_gate", 3001)])
def test_saved_latent_matches_encoder_and_feeds_backward(sp, name, n):
    """decode_fwd's saved latent equals encode_fwd's z bit for bit, and the
    backward fed with it matches the oracle (and the re-gathering backward)."""
    grid, mlp, pos, tables, weights, cr = _workload(name, n, 1.0, 0.5)
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    P, T, W = dev(pos), dev(tables), dev(weights)
    C = dev(cr) if cr is not None else None
    out = sp.decode_fwd(g, m, P, T, W, C, out=sp.alloc_outputs(n, "cuda", latent_dim=grid.L * grid.F))
    z = sp.encode_fwd(g, P, T)
    assert torch.equal(out["latent"], z)
    gstd = 1e-2 if grid.dtype == "f16" else 1.0
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, gstd)
    G = {k: dev(v) for k, v in grads.items()}
    res = []
    for lat in (out["latent"], None):
        gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), dtype=torch.float32, device="cuda")
        gw = torch.zeros(mlp.n_params(), dtype=torch.float32, device="cuda")
        sp.decode_bwd(g, m, P, T, W, G, gt, gw, gate_cr=C, latent=lat)
        res.append((host(gt), host(gw)))
    levels = tol.table_levels(grid.L, 1 << grid.log2_T, grid.F)
    blocks = tol.weight_blocks(mlp.layer_shapes())
    tol.normwise(res[0][0], res[1][0], 1e-4, "tables: saved latent vs re-gather", levels)
    tol.normwise(res[0][1], res[1][1], 1e-4, "weights: saved latent vs re-gather", blocks)
    wt, ww = dec.decode_backward(pos, tables, weights, grid, mlp, grads, gate_cr=cr)
    rtol = tol.FP32_GRAD_RTOL if grid.dtype == "f32" else tol.FP16_GRAD_RTOL
    check_decode_grads(res[0][0], res[0][1], wt, ww, grid, mlp, rtol,
                       mag.decoder_rss(pos, tables, weights, grid, mlp, grads, gate_cr=cr))


def test_decode_bwd_null_upstream_means_zero(sp):
    """A NULL upstream pointer is a zero gradient: only rgb given."""
    grid, mlp, pos, tables, weights, _ = _workload("tiny_fp32", 1000, 1.0, 0.5)
    grads = S.upstream_grads(1000, {"rgb": 3}, 1.0)
    gt, gw = _bwd(sp, grid, mlp, pos, tables, weights, None, grads)
    assert np.any(gt != 0)
    full = {k: np.zeros((1000, w), np.float32) for k, w in S.DECODE_OUT_WIDTHS.items()}
    full["rgb"] = grads["rgb"]
    wt, ww = dec.decode_backward(pos, tables, weights, grid, mlp, full)
    check_decode_grads(gt, gw, wt, ww, grid, mlp, tol.FP32_GRAD_RTOL,
                       mag.decoder_rss(pos, tables, weights, grid, mlp, full))


def test_decode_bwd_accumulates_and_is_linear_at_full_batch(sp):
    """1M positions (one training launch): gradients accumulate (+=), and the
    full batch equals the sum of its two halves launched separately."""
    w = S.WORKLOADS["sports_train_fp16"]
    grid, mlp = w["grid"], w["mlp"]
    scene = S.sports_scene(300_000)
    pos = scene.frames(range(0, 4))[:1_000_000]
    tables = S.hash_tables(grid, scale=1.0)
    weights = S.mlp_weights(mlp, bias_scale=0.5)
    grads = S.upstream_grads(len(pos), S.DECODE_OUT_WIDTHS, 1e-2)
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    P, T, W, G = dev(pos), dev(tables), dev(weights), {k: dev(v) for k, v in grads.items()}
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), dtype=torch.float32, device="cuda")
    gw = torch.zeros(mlp.n_params(), dtype=torch.float32, device="cuda")
    sp.decode_bwd(g, m, P, T, W, G, gt, gw)
    h = 499_999
    gt2 = torch.zeros_like(gt)
    gw2 = torch.zeros_like(gw)
    sp.decode_bwd(g, m, P[:h].contiguous(), T, W, {k: v[:h].contiguous() for k, v in G.items()}, gt2, gw2)
    sp.decode_bwd(g, m, P[h:].contiguous(), T, W, {k: v[h:].contiguous() for k, v in G.items()}, gt2, gw2)
    # Same arithmetic per position; only the fp32 accumulation order differs
    # (atomics, per-block weight slots).  A coarse-level entry receives up to
    # K ~ 10^3 additions here, so the rounding bound is ~K * 2^-24 ~ 6e-5.
    levels = tol.table_levels(grid.L, 1 << grid.log2_T, grid.F)
    blocks = tol.weight_blocks(mlp.layer_shapes())
    tol.normwise(host(gt2), host(gt), 1e-4, "tables: halves vs whole", levels)
    tol.normwise(host(gw2), host(gw), 1e-4, "weights: halves vs whole", blocks)
    # sampled oracle check: the head-bias gradient is a plain sum of dy over
    # positions; check it on a 4000-row subset launched alone
    rows = np.random.default_rng(2).choice(len(pos), 4000, replace=False)
    gt3 = torch.zeros_like(gt)
    gw3 = torch.zeros_like(gw)
    sub = {k: v[rows] for k, v in grads.items()}
    sp.decode_bwd(g, m, dev(pos[rows]), T, W, {k: dev(v) for k, v in sub.items()}, gt3, gw3)
    wt, ww = dec.decode_backward(pos[rows], tables, weights, grid, mlp, sub)
    check_decode_grads(host(gt3), host(gw3), wt, ww, grid, mlp, tol.FP16_GRAD_RTOL,
                       mag.decoder_rss(pos[rows], tables, weights, grid, mlp, sub), tag="subset ")


# ---------------------------------------------------------------------------
# covariance and Adam
# ---------------------------------------------------------------------------
def test_cov_assemble_matches_oracle(sp):
    rng = np.random.default_rng(5)
    n = 100_003
    q = rng.standard_normal((n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    s = np.exp(rng.uniform(-6, 1, size=(n, 3)))
    q32, s32 = q.astype(np.float32), s.astype(np.float32)
    cov = host(sp.cov_assemble(dev(s32), dev(q32)))
    want = dec.covariance(s32.astype(np.float64), q32.astype(np.float64))
    tol.elementwise(cov, want, tol.FP32_RTOL, "cov", tol.column_groups(6), rho=mag.cov_mag(s32))


def test_adam_matches_oracle(sp):
    rng = np.random.default_rng(6)
    n = 1_000_003
    p = rng.uniform(-1, 1, n).astype(np.float32)
    P, M, V = dev(p), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    work = torch.empty(n, dtype=torch.float16, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    wp, wm, wv = p.astype(np.float64), np.zeros(n), np.zeros(n)
    for step in (1, 2, 3):
        g = (rng.standard_normal(n) * 10.0 ** rng.uniform(-8, 0, n)).astype(np.float32)
        g[:7] = 0.0
        G = dev(g)
        sp.adam_step(P, G, M, V, step, 1e-3, 0.9, 0.99, 1e-15, params_work=work, zero_grad=True,
                     nonfinite_flag=flag)
        wp, wm, wv = dec.adam_step(wp, g, wm, wv, step, 1e-3, float(np.float32(0.9)), float(np.float32(0.99)), 1e-15)
        assert float(G.abs().max()) == 0.0
    tol.normwise(host(P) - p, wp - p, 1e-4, "adam update")
    tol.normwise(host(P), wp, 1e-6, "adam params")
    assert np.array_equal(host(work), host(P).astype(np.float16))
    assert int(flag.item()) == 0
