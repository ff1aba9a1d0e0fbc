"""GPU parity of the paper's four-head GELU decoder and the grouped Adam
against the oracle (B200 only)."""
import numpy as np
import pytest

from oracle import decoder as dec
from oracle import heads as hd
from spatiotemporal_neural_field_b200 import synthetic as S
from tests import tol

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sp():
    from spatiotemporal_neural_field_b200 import spin4d
    return spin4d


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


CASES = {
    # name: (grid, heads, positions, n, table scale, bias scale, grad std)
    "tiny_fp32": (S.GRID_TINY4, S.HEADS_TINY, "uniform", 4099, 1.0, 0.3, 1.0),
    "paper_fp16": (S.GRID_PAPER, S.HEADS_PAPER, "sports", 3001, 1.0, 0.3, 1e-2),
    "paper_fp16_init": (S.GRID_PAPER, S.HEADS_PAPER, "sports", 2003, 1e-4, 0.0, 1e-2),
}


def _setup(case):
    grid, spec, kind, n, ts, bs, gstd = CASES[case]
    pos = S.uniform_positions(n, seed=3) if kind == "uniform" else S.sports_scene(n).frames(range(4))[:n]
    tables = S.hash_tables(grid, seed=4, scale=ts)
    weights = S.heads_weights(spec, seed=5, bias_scale=bs)
    widths = dict(S.HEADS_OUT_WIDTHS, sh=spec.sh_dim)
    grads = S.upstream_grads(n, widths, gstd, seed=6)
    return grid, spec, pos, tables, weights, grads


@pytest.mark.parametrize("case", list(CASES))
def test_heads_forward_matches_oracle(sp, case):
    grid, spec, pos, tables, weights, _ = _setup(case)
    g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec)
    out = sp.heads_fwd(g, h, dev(pos), dev(tables), dev(weights), latent=True)
    want = hd.decode_forward(pos, tables, weights, grid, spec)
    for k in ("scale", "rot", "sh", "opacity", "cov"):
        if grid.dtype == "f32":
            tol.rowwise(host(out[k]), want[k], tol.FP32_RTOL, k)
        else:
            tol.absolute(host(out[k]), want[k], tol.FP16_ATOL, k)
    tol.rowwise(host(out["latent"]), want["z"], tol.FP32_RTOL, "latent")


@pytest.mark.parametrize("case,latent", [("tiny_fp32", False), ("paper_fp16", False), ("paper_fp16", True),
                                         ("paper_fp16_init", False)])
def test_heads_backward_matches_oracle(sp, case, latent):
    grid, spec, pos, tables, weights, grads = _setup(case)
    g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec)
    P, T, W = dev(pos), dev(tables), dev(weights)
    lat = sp.heads_fwd(g, h, P, T, W, latent=True)["latent"] if latent else None
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda")
    gw = torch.zeros(spec.n_params(), device="cuda")
    sp.heads_bwd(g, h, P, T, W, {k: dev(v) for k, v in grads.items()}, gt, gw, latent=lat)
    wt, ww = hd.decode_backward(pos, tables, weights, grid, spec, grads)
    rtol = tol.FP32_GRAD_RTOL if grid.dtype == "f32" else tol.FP16_GRAD_RTOL
    tol.normwise(host(gt), wt, rtol, "grad_tables")
    gwh = host(gw)
    o = 0
    for head in range(4):
        for (out_d, in_d) in spec.layer_shapes(head):
            tol.normwise(gwh[o:o + out_d * in_d], ww[o:o + out_d * in_d], rtol, "dW head %d %dx%d" % (head, out_d, in_d))
            o += out_d * in_d
            tol.normwise(gwh[o:o + out_d], ww[o:o + out_d], rtol, "db head %d %d" % (head, out_d))
            o += out_d
    assert o == gwh.size


def test_grouped_adam_matches_oracle(sp):
    """The paper's decoder rates per head (section 4) over the packed weights."""
    spec = S.HEADS_PAPER
    n = spec.n_params()
    rng = np.random.default_rng(7)
    p = rng.normal(size=n).astype(np.float32)
    grad = rng.normal(size=n).astype(np.float32)
    m = rng.normal(size=n).astype(np.float32) * 0.1
    v = np.abs(rng.normal(size=n)).astype(np.float32) * 0.01
    rates = (3e-4, 3e-5, 1e-3, 8e-4)            # scale, rotation, colour, opacity
    ends, o = [], 0
    for head in range(4):
        o += sum(a * b + a for a, b in spec.layer_shapes(head))
        ends.append(o)
    P, G, M, V = dev(p), dev(grad), dev(m), dev(v)
    sp.adam_step_groups(P, G, M, V, 3, list(zip(ends, rates)), 0.9, 0.99, 1e-15)
    start = 0
    for end, lr in zip(ends, rates):
        wp, wm, wv = dec.adam_step(p[start:end], grad[start:end], m[start:end], v[start:end], 3, lr, 0.9, 0.99, 1e-15)
        # fp32 arithmetic: p' to fp32 rounding; the update p' - p to two ulp of the largest |p| (the
        # representation limit of p') plus 1e-5 of the largest update; each state to fp32 rounding
        tol.normwise(host(P)[start:end], wp, 1e-6, "grouped adam params")
        du, dw = host(P)[start:end] - p[start:end], wp - p[start:end]
        bound = 2 * np.spacing(np.float32(np.max(np.abs(p[start:end])))) + 1e-5 * np.max(np.abs(dw))
        assert np.max(np.abs(du - dw)) <= bound, (lr, np.max(np.abs(du - dw)), bound)
        tol.normwise(host(M)[start:end], wm, 1e-6, "grouped adam m")
        tol.normwise(host(V)[start:end], wv, 1e-6, "grouped adam v")
        start = end
