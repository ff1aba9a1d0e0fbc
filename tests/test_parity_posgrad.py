"""GPU parity of the extra gradients of spin4d_decode_bwd_ext (position and
gate parameters) against the oracle (B200 only)."""
import dataclasses

import numpy as np
import pytest

from oracle import decoder as dec
from spatiotemporal_neural_field_b200 import synthetic as S
from tests import magnitude as mag
from tests import tol
from tests.test_parity_decode import check_decode_grads

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


def _positions(kind, n):
    if kind == "uniform":
        # half inside the unit ball, half out to |mu| ~ 1.7 (both branches of Eq. 7)
        return S.uniform_positions(n)
    if kind == "sports":
        return S.sports_scene(n).frame(75)
    return S.stress_positions(n)


CASES = {
    # name: (workload, positions, n, table scale, bias scale, grad std)
    "tiny": ("tiny_fp32", "uniform", 4099, 1.0, 0.5, 1.0),
    "sports": ("sports_frame_fp16", "sports", 20011, 1.0, 0.5, 1e-2),
    "stress_gate": ("stress_fp16_gate", "stress", 6007, 1.0, 0.5, 1.0),
}


def _run(sp, case, latent=False):
    name, kind, n, ts, bs, gstd = CASES[case]
    w = S.WORKLOADS[name]
    grid, mlp = w["grid"], w["mlp"]
    pos = _positions(kind, n)
    tables = S.hash_tables(grid, scale=ts)
    weights = S.mlp_weights(mlp, bias_scale=bs)
    cr = S.gate_params(n) if mlp.gate else None
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, gstd, seed=21)
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    P, T, W = dev(pos), dev(tables), dev(weights)
    CR = dev(cr) if cr is not None else None
    lat = None
    if latent:
        out = sp.alloc_outputs(n, "cuda", latent_dim=grid.L * grid.F)
        sp.decode_fwd(g, m, P, T, W, CR, out=out)
        lat = out["latent"]
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), dtype=torch.float32, device="cuda")
    gw = torch.zeros(mlp.n_params(), dtype=torch.float32, device="cuda")
    gp = torch.zeros((n, 3), dtype=torch.float32, device="cuda")
    sp.decode_bwd(g, m, P, T, W, {k: dev(v) for k, v in grads.items()}, gt, gw, gate_cr=CR, latent=lat, grad_pos=gp)
    sp.check_device_errors()
    want = dec.decode_backward(pos, tables, weights, grid, mlp, grads, gate_cr=cr, want_pos=True)
    rho = mag.decoder_rss(pos, tables, weights, grid, mlp, grads, gate_cr=cr, want_pos=True)
    return grid, mlp, host(gt), host(gw), host(gp), want, rho


AXES = tol.column_groups(3, ["x", "y", "z"])


@pytest.mark.parametrize("case", list(CASES))
def test_position_gradient_matches_oracle(sp, case):
    grid, mlp, gt, gw, gp, (wt, ww, wp), rho = _run(sp, case)
    rtol = tol.FP32_GRAD_RTOL if grid.dtype == "f32" else tol.FP16_GRAD_RTOL
    tol.elementwise(gp, wp, rtol, "grad_pos", AXES, rho=rho[2])
    # the table and weight gradients of the same call are unchanged by it
    check_decode_grads(gt, gw, wt, ww, grid, mlp, rtol, rho[:2])


@pytest.mark.parametrize("case", ["sports", "stress_gate"])
def test_position_gradient_with_saved_latent(sp, case):
    """The corners are gathered again for the position gradient even when the
    forward's latent replaces the second gather of z."""
    grid, _, _, _, gp, (_, _, wp), rho = _run(sp, case, latent=True)
    tol.elementwise(gp, wp, tol.FP16_GRAD_RTOL, "grad_pos (saved latent)", AXES, rho=rho[2])


def test_position_gradient_accumulates_and_matches_plain_backward(sp):
    grid, mlp = S.GRID_SPORTS, S.MLP_SPORTS
    n = 5003
    pos = _positions("sports", n)
    T, W, P = dev(S.hash_tables(grid, scale=1.0)), dev(S.mlp_weights(mlp, bias_scale=0.5)), dev(pos)
    G = {k: dev(v) for k, v in S.upstream_grads(n, S.DECODE_OUT_WIDTHS, 1e-2, seed=3).items()}
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)

    def zeros():
        return (torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda"),
                torch.zeros(mlp.n_params(), device="cuda"))

    gt1, gw1 = zeros()
    sp.decode_bwd(g, m, P, T, W, G, gt1, gw1)
    gt2, gw2 = zeros()
    gp = torch.zeros((n, 3), device="cuda")
    sp.decode_bwd(g, m, P, T, W, G, gt2, gw2, grad_pos=gp)
    # weight gradients are summed in a fixed order: bit-identical to the plain call
    assert torch.equal(gw1, gw2)
    tol.normwise(host(gt2), host(gt1), 1e-5, "tables with and without grad_pos",
                 tol.table_levels(grid.L, 1 << grid.log2_T, grid.F))
    first = gp.clone()
    sp.decode_bwd(g, m, P, T, W, G, gt2, gw2, grad_pos=gp)
    # each position is written by one thread, so the second call adds the same values
    assert torch.equal(gp, 2 * first)


def test_position_gradient_normalised_input(sp):
    """With SPIN4D_INPUT_NORMALISED the gradient is w.r.t. x~ itself, zero
    where the clamp to [0, 1] bound."""
    grid, mlp = S.GRID_TINY, S.MLP_TINY
    n = 2049
    xt = np.random.default_rng(4).uniform(-0.1, 1.1, size=(n, 4)).astype(np.float32)
    tables = S.hash_tables(grid, scale=1.0)
    weights = S.mlp_weights(mlp, bias_scale=0.5)
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, 1.0, seed=5)
    g = sp.grid_from_spec(grid)
    g.flags |= sp.INPUT_NORMALISED
    m = sp.mlp_from_spec(mlp)
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda")
    gw = torch.zeros(mlp.n_params(), device="cuda")
    gp = torch.zeros((n, 3), device="cuda")
    sp.decode_bwd(g, m, dev(xt), dev(tables), dev(weights), {k: dev(v) for k, v in grads.items()}, gt, gw,
                  grad_pos=gp)
    _, _, wp = dec.decode_backward(xt, tables, weights, grid, mlp, grads, normalised_input=True, want_pos=True)
    rho = mag.decoder_rss(xt, tables, weights, grid, mlp, grads, normalised_input=True, want_pos=True)[2]
    tol.elementwise(host(gp), wp, tol.FP32_GRAD_RTOL, "grad_pos (normalised input)", AXES, rho=rho)
    out_of_range = (xt[:, :3] < 0) | (xt[:, :3] > 1)
    assert out_of_range.any() and np.all(host(gp)[out_of_range] == 0)



# ---------------------------------------------------------------------------
# gradient w.r.t. the gate's window centre and half-width
# ---------------------------------------------------------------------------
def _gate_case(sp, grid, mlp, pos, n, tscale, gstd, latent=False):
    tables = S.hash_tables(grid, scale=tscale)
    weights = S.mlp_weights(mlp, bias_scale=0.5)
    cr = S.gate_params(n, seed=31)
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, gstd, seed=32)
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    P, T, W, CR = dev(pos), dev(tables), dev(weights), dev(cr)
    lat = None
    if latent:
        out = sp.alloc_outputs(n, "cuda", latent_dim=grid.L * grid.F)
        sp.decode_fwd(g, m, P, T, W, CR, out=out)
        lat = out["latent"]
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda")
    gw = torch.zeros(mlp.n_params(), device="cuda")
    gp = torch.zeros((n, 3), device="cuda")
    gg = torch.zeros((n, 2), device="cuda")
    sp.decode_bwd(g, m, P, T, W, {k: dev(v) for k, v in grads.items()}, gt, gw, gate_cr=CR, latent=lat, grad_pos=gp,
                  grad_gate=gg)
    sp.check_device_errors()
    _, _, wp, wg = dec.decode_backward(pos, tables, weights, grid, mlp, grads, gate_cr=cr, want_pos=True,
                                       want_gate=True)
    rho_pos = mag.decoder_rss(pos, tables, weights, grid, mlp, grads, gate_cr=cr, want_pos=True)[2]
    rho_gate = mag.gate_rss(pos, tables, weights, grid, mlp, grads, cr)
    return host(gp), host(gg), wp, wg, rho_pos, rho_gate


GATE = tol.column_groups(2, ["c", "r"])


def test_gate_gradient_stress_tensor_core_path(sp):
    w = S.WORKLOADS["stress_fp16_gate"]
    n = 6007
    gp, gg, wp, wg, rp, rg = _gate_case(sp, w["grid"], w["mlp"], S.stress_positions(n), n, 1.0, 1.0)
    tol.elementwise(gg, wg, tol.FP16_GRAD_RTOL, "grad_gate", GATE, rho=rg)
    tol.elementwise(gp, wp, tol.FP16_GRAD_RTOL, "grad_pos alongside grad_gate", AXES, rho=rp)


def test_gate_gradient_stress_saved_latent(sp):
    w = S.WORKLOADS["stress_fp16_gate"]
    n = 3001
    _, gg, _, wg, _, rg = _gate_case(sp, w["grid"], w["mlp"], S.stress_positions(n), n, 1.0, 1.0, latent=True)
    tol.elementwise(gg, wg, tol.FP16_GRAD_RTOL, "grad_gate (saved latent)", GATE, rho=rg)


def test_gate_gradient_fp32_simt_path(sp):
    mlp = dataclasses.replace(S.MLP_TINY, gate=True, tau=0.05)
    n = 4099
    pos = S.uniform_positions(n, seed=33)
    gp, gg, wp, wg, rp, rg = _gate_case(sp, S.GRID_TINY, mlp, pos, n, 1.0, 1.0)
    tol.elementwise(gg, wg, tol.FP32_GRAD_RTOL, "grad_gate (fp32)", GATE, rho=rg)
    tol.elementwise(gp, wp, tol.FP32_GRAD_RTOL, "grad_pos (fp32, gated)", AXES, rho=rp)
