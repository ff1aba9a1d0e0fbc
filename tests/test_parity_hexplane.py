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


def _check_grads(hx, gp, gw, wp, ww, rtol):
    tol.normwise(host(gp), wp, rtol, "grad_planes")
    o = 0
    gwh = host(gw)
    for (out_d, in_d) in hx.layer_shapes():
        tol.normwise(gwh[o:o + out_d * in_d], ww[o:o + out_d * in_d], rtol, "dW %dx%d" % (out_d, in_d))
        o += out_d * in_d
        tol.normwise(gwh[o:o + out_d], ww[o:o + out_d], rtol, "db %d" % out_d)
        o += out_d


def _zero_grads(hx):
    return (torch.zeros(hx.n_plane_floats(), dtype=torch.float32, device="cuda"),
            torch.zeros(hx.n_params(), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("n", [1500, 65, 128])
def test_hexplane_bwd_matches_oracle(sp, n):
    hx, inp, planes, weights = _inputs(n, 0.5)
    grads = S.upstream_grads(n, S.HEX_OUT_WIDTHS, 1.0, seed=3)
    h = sp.hex_from_spec(hx)
    gp, gw = _zero_grads(hx)
    sp.hexplane_bwd(h, {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights),
                    {k: dev(v) for k, v in grads.items()}, gp, gw)
    wp, ww = hp.backward(inp, planes, weights, hx, grads)
    _check_grads(hx, gp, gw, wp, ww, tol.FP32_GRAD_RTOL)


def test_hexplane_bwd_from_saved_latent_matches_oracle(sp):
    n = 2001
    hx, inp, planes, weights = _inputs(n, 0.5, seed=1)
    grads = S.upstream_grads(n, S.HEX_OUT_WIDTHS, 1.0, seed=5)
    h = sp.hex_from_spec(hx)
    I, P, W = {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights)
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["latent"] = torch.empty((n, hx.in_dim), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(h, I, P, W, out=out)
    gp, gw = _zero_grads(hx)
    sp.hexplane_bwd(h, I, P, W, {k: dev(v) for k, v in grads.items()}, gp, gw, latent=out["latent"])
    wp, ww = hp.backward(inp, planes, weights, hx, grads)
    _check_grads(hx, gp, gw, wp, ww, tol.FP32_GRAD_RTOL)


def test_hexplane_bwd_partial_upstream(sp):
    """Only the covariance and sh gradients given; the others are NULL (zero)."""
    n = 700
    hx, inp, planes, weights = _inputs(n, 0.5, seed=2)
    full = S.upstream_grads(n, S.HEX_OUT_WIDTHS, 1.0, seed=7)
    grads = {k: full[k] for k in ("cov", "sh")}
    gp, gw = _zero_grads(hx)
    sp.hexplane_bwd(sp.hex_from_spec(hx), {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights),
                    {k: dev(v) for k, v in grads.items()}, gp, gw)
    zeros = {k: np.zeros_like(v) for k, v in full.items()}
    zeros.update(grads)
    wp, ww = hp.backward(inp, planes, weights, hx, zeros)
    _check_grads(hx, gp, gw, wp, ww, tol.FP32_GRAD_RTOL)


def test_hexplane_bwd_full_batch_halves_latent_and_sample(sp):
    """500k Gaussians (one training launch): gradients accumulate (+=); the
    batch equals the sum of its two halves launched separately; reading the
    saved latent equals gathering again; a subset launched alone matches the
    oracle."""
    n = S.WORKLOADS["hexplane_fp32"]["N"]
    hx, inp, planes, weights = _inputs(n, 0.5)
    grads = S.upstream_grads(n, S.HEX_OUT_WIDTHS, 1e-2)
    h = sp.hex_from_spec(hx)
    I, P, W = {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights)
    G = {k: dev(v) for k, v in grads.items()}
    gp, gw = _zero_grads(hx)
    sp.hexplane_bwd(h, I, P, W, G, gp, gw)
    half = 249_999
    gp2, gw2 = _zero_grads(hx)
    for sl in (slice(0, half), slice(half, n)):
        sp.hexplane_bwd(h, {k: v[sl].contiguous() for k, v in I.items()}, P, W,
                        {k: v[sl].contiguous() for k, v in G.items()}, gp2, gw2)
    # Same arithmetic per Gaussian; only the fp32 accumulation order differs
    # (plane atomics, per-CTA weight slots).  A cell of the coarsest plane
    # receives ~10^3 additions here, so the rounding bound is ~K * 2^-24 ~ 6e-5.
    tol.normwise(host(gp2), host(gp), 1e-4, "planes: halves vs whole")
    tol.normwise(host(gw2), host(gw), 1e-4, "weights: halves vs whole")
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["latent"] = torch.empty((n, hx.in_dim), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(h, I, P, W, out=out)
    gp3, gw3 = _zero_grads(hx)
    sp.hexplane_bwd(h, I, P, W, G, gp3, gw3, latent=out["latent"])
    tol.normwise(host(gp3), host(gp), 1e-4, "planes: saved latent vs gather")
    tol.normwise(host(gw3), host(gw), 1e-4, "weights: saved latent vs gather")
    rows = np.sort(np.random.default_rng(6).choice(n, 2000, replace=False))
    rows[-1] = n - 1
    sub_inp = {k: v[rows] for k, v in inp.items()}
    sub = {k: v[rows] for k, v in grads.items()}
    gp4, gw4 = _zero_grads(hx)
    sp.hexplane_bwd(h, {k: dev(v) for k, v in sub_inp.items()}, P, W, {k: dev(v) for k, v in sub.items()}, gp4, gw4)
    wp, ww = hp.backward(sub_inp, planes, weights, hx, sub)
    _check_grads(hx, gp4, gw4, wp, ww, tol.FP32_GRAD_RTOL)


def test_hexplane_fwd_saved_latent_matches_oracle_encoder(sp):
    n = 3001
    hx, inp, planes, weights = _inputs(n, 0.5)
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["latent"] = torch.empty((n, hx.in_dim), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(sp.hex_from_spec(hx), {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights), out=out)
    z = hp.encode(hp.normalise(inp["mu"], inp["frame"], hx.n_frames), planes, hx)
    tol.rowwise(host(out["latent"]), z, tol.FP32_RTOL, "latent")
