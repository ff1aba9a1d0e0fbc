"""GPU parity of the HexPlane encoder + deformation network (B200 only)."""
import numpy as np
import pytest

from oracle import hexplane as hp
from spatiotemporal_neural_field_b200 import synthetic as S
from tests import tol

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
HEX_KEYS = ("mu", "rot", "scale", "sh", "cov")


@pytest.fixture(scope="module")
def sp():
    from spatiotemporal_neural_field_b200 import spin4d
    return spin4d


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def _inputs(n, bias_scale=0.0, seed=0):
    hx = S.HEX
    inp = S.hexplane_inputs(n, seed)
    planes = S.hexplane_planes(hx, seed)
    weights = S.hexplane_weights(hx, seed, bias_scale=bias_scale)
    return hx, inp, planes, weights


@pytest.mark.parametrize("n,bias_scale", [(2053, 0.0), (1, 0.5), (777, 0.5)])
def test_hexplane_fwd_matches_oracle(sp, n, bias_scale):
    hx, inp, planes, weights = _inputs(n, bias_scale)
    h = sp.hex_from_spec(hx)
    out = sp.hexplane_fwd(h, {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights))
    want = hp.forward(inp, planes, weights, hx)
    for k in HEX_KEYS:
        tol.rowwise(host(out[k]), want[k], tol.FP32_RTOL, k)


def test_hexplane_fwd_full_size_sampled(sp):
    n = S.WORKLOADS["hexplane_fp32"]["N"]
    hx, inp, planes, weights = _inputs(n, 0.5)
    out = sp.hexplane_fwd(sp.hex_from_spec(hx), {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights))
    rows = np.sort(np.random.default_rng(4).choice(n, 1500, replace=False))
    rows[-1] = n - 1
    want = hp.forward({k: v[rows] for k, v in inp.items()}, planes, weights, hx)
    for k in HEX_KEYS:
        tol.rowwise(host(out[k])[rows], want[k], tol.FP32_RTOL, k)


@pytest.mark.parametrize("n", [1500, 65])
def test_hexplane_bwd_matches_oracle(sp, n):
    hx, inp, planes, weights = _inputs(n, 0.5)
    grads = S.upstream_grads(n, S.HEX_OUT_WIDTHS, 1.0, seed=3)
    h = sp.hex_from_spec(hx)
    gp = torch.zeros(hx.n_plane_floats(), dtype=torch.float32, device="cuda")
    gw = torch.zeros(hx.n_params(), dtype=torch.float32, device="cuda")
    sp.hexplane_bwd(h, {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights),
                    {k: dev(v) for k, v in grads.items()}, gp, gw)
    wp, ww = hp.backward(inp, planes, weights, hx, grads)
    tol.normwise(host(gp), wp, tol.FP32_GRAD_RTOL, "grad_planes")
    o = 0
    gwh = host(gw)
    for (out_d, in_d) in hx.layer_shapes():
        tol.normwise(gwh[o:o + out_d * in_d], ww[o:o + out_d * in_d], tol.FP32_GRAD_RTOL, "dW %dx%d" % (out_d, in_d))
        o += out_d * in_d
        tol.normwise(gwh[o:o + out_d], ww[o:o + out_d], tol.FP32_GRAD_RTOL, "db %d" % out_d)
        o += out_d


def test_hexplane_fwd_saved_latent_matches_oracle_encoder(sp):
    n = 3001
    hx, inp, planes, weights = _inputs(n, 0.5)
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["latent"] = torch.empty((n, hx.in_dim), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(sp.hex_from_spec(hx), {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights), out=out)
    z = hp.encode(hp.normalise(inp["mu"], inp["frame"], hx.n_frames), planes, hx)
    tol.rowwise(host(out["latent"]), z, tol.FP32_RTOL, "latent")
