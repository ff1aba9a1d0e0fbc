"""GPU parity of the HexPlane encoder + deformation network (B200 only)."""
import numpy as np
import pytest

from oracle import hexplane as hp
from spatiotemporal_neural_field_b200 import synthetic as S
from tests import magnitude as mag
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


def check_hex_outputs(got, want, m, tag=""):
    """fp32 deformed Gaussians, element-wise per attribute.  mu' = mu + dmu and
    sh' = sh + dsh are held to the magnitudes of their terms ``m``
    (tests/magnitude.py); a rotation component is rounded relative to the
    unit row norm; a Sigma entry to the spectral norm max_k s_k^2."""
    for k in HEX_KEYS:
        rho = None
        if k in ("mu", "sh"):
            rho = m[k]
        elif k == "rot":
            rho = np.ones_like(want[k])
        elif k == "cov":
            rho = mag.cov_mag(want["scale"])
        tol.elementwise(got[k], want[k], tol.FP32_RTOL, tag + k, rho=rho)


@pytest.mark.parametrize("n,bias_scale", [(2053, 0.0), (1, 0.5), (777, 0.5)])
def test_hexplane_fwd_matches_oracle(sp, n, bias_scale):
    hx, inp, planes, weights = _inputs(n, bias_scale)
    h = sp.hex_from_spec(hx)
    out = sp.hexplane_fwd(h, {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights))
    want = hp.forward(inp, planes, weights, hx)
    check_hex_outputs({k: host(out[k]) for k in HEX_KEYS}, want, mag.hexplane_output_mag(inp, planes, weights, hx))


def test_hexplane_fwd_full_size_sampled(sp):
    n = S.WORKLOADS["hexplane_fp32"]["N"]
    hx, inp, planes, weights = _inputs(n, 0.5)
    out = sp.hexplane_fwd(sp.hex_from_spec(hx), {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights))
    rows = np.sort(np.random.default_rng(4).choice(n, 1500, replace=False))
    rows[-1] = n - 1
    sub = {k: v[rows] for k, v in inp.items()}
    want = hp.forward(sub, planes, weights, hx)
    check_hex_outputs({k: host(out[k])[rows] for k in HEX_KEYS}, want, mag.hexplane_output_mag(sub, planes, weights, hx))


def _check_grads(hx, gp, gw, wp, ww, rtol, rho=(None, None)):
    """Element-wise per plane and per weight block."""
    tol.elementwise(host(gp), wp, rtol, "grad_planes", tol.plane_groups(hx), rho=rho[0])
    tol.elementwise(host(gw), ww, rtol, "grad_weights", tol.weight_blocks(hx.layer_shapes()), rho=rho[1])


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
    _check_grads(hx, gp, gw, wp, ww, tol.FP32_GRAD_RTOL, mag.hexplane_rss(inp, planes, weights, hx, grads))


@pytest.mark.parametrize("saved_h1", [False, True])
@pytest.mark.parametrize("n", [1, 129, 2001, 40_000])
def test_hexplane_bwd_from_saved_latent_matches_oracle(sp, n, saved_h1):
    """From the forward's saved latent (and its saved h1): one Gaussian, a
    ragged second tile, several tiles, and more tiles than SMs (the
    persistent CTAs run two, so the sample ring carries across tiles)."""
    hx, inp, planes, weights = _inputs(n, 0.5, seed=1)
    grads = S.upstream_grads(n, S.HEX_OUT_WIDTHS, 1.0, seed=5)
    h = sp.hex_from_spec(hx)
    I, P, W = {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights)
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["latent"] = torch.empty((n, hx.in_dim), dtype=torch.float32, device="cuda")
    if saved_h1:
        out["hidden"] = torch.empty((n, hx.hidden), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(h, I, P, W, out=out)
    gp, gw = _zero_grads(hx)
    sp.hexplane_bwd(h, I, P, W, {k: dev(v) for k, v in grads.items()}, gp, gw, latent=out["latent"],
                    hidden=out.get("hidden"))
    wp, ww = hp.backward(inp, planes, weights, hx, grads)
    _check_grads(hx, gp, gw, wp, ww, tol.FP32_GRAD_RTOL, mag.hexplane_rss(inp, planes, weights, hx, grads))


@pytest.mark.parametrize("n", [129, 3001])
def test_hexplane_fwd_saved_h1_matches_oracle(sp, n):
    """The forward's saved first hidden layer, relu(W1 z + b1), element-wise
    against the oracle's (the magnitude of its pre-activation's terms where
    it is positive); the other outputs are unchanged by saving it."""
    hx, inp, planes, weights = _inputs(n, 0.5, seed=4)
    h = sp.hex_from_spec(hx)
    I, P, W = {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights)
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["hidden"] = torch.empty((n, hx.hidden), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(h, I, P, W, out=out)
    want = hp.forward(inp, planes, weights, hx)
    tol.elementwise(host(out["hidden"]), want["h1"], tol.FP32_RTOL, "h1", tol.column_groups(hx.hidden),
                    rho=mag.hexplane_hidden_mag(inp, planes, weights, hx))
    plain = sp.hexplane_fwd(h, I, P, W)
    for k, _ in sp.HEX_KEYS:
        assert torch.equal(plain[k], out[k]), k


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
    _check_grads(hx, gp, gw, wp, ww, tol.FP32_GRAD_RTOL, mag.hexplane_rss(inp, planes, weights, hx, zeros))


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
    tol.normwise(host(gp2), host(gp), 1e-4, "planes: halves vs whole", tol.plane_groups(hx))
    tol.normwise(host(gw2), host(gw), 1e-4, "weights: halves vs whole", tol.weight_blocks(hx.layer_shapes()))
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["latent"] = torch.empty((n, hx.in_dim), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(h, I, P, W, out=out)
    gp3, gw3 = _zero_grads(hx)
    sp.hexplane_bwd(h, I, P, W, G, gp3, gw3, latent=out["latent"])
    tol.normwise(host(gp3), host(gp), 1e-4, "planes: saved latent vs gather", tol.plane_groups(hx))
    tol.normwise(host(gw3), host(gw), 1e-4, "weights: saved latent vs gather", tol.weight_blocks(hx.layer_shapes()))
    out["hidden"] = torch.empty((n, hx.hidden), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(h, I, P, W, out=out)
    gp5, gw5 = _zero_grads(hx)
    sp.hexplane_bwd(h, I, P, W, G, gp5, gw5, latent=out["latent"], hidden=out["hidden"])
    tol.normwise(host(gp5), host(gp), 1e-4, "planes: saved h1 vs gather", tol.plane_groups(hx))
    tol.normwise(host(gw5), host(gw), 1e-4, "weights: saved h1 vs gather", tol.weight_blocks(hx.layer_shapes()))
    rows = np.sort(np.random.default_rng(6).choice(n, 2000, replace=False))
    rows[-1] = n - 1
    sub_inp = {k: v[rows] for k, v in inp.items()}
    sub = {k: v[rows] for k, v in grads.items()}
    gp4, gw4 = _zero_grads(hx)
    sp.hexplane_bwd(h, {k: dev(v) for k, v in sub_inp.items()}, P, W, {k: dev(v) for k, v in sub.items()}, gp4, gw4)
    wp, ww = hp.backward(sub_inp, planes, weights, hx, sub)
    _check_grads(hx, gp4, gw4, wp, ww, tol.FP32_GRAD_RTOL, mag.hexplane_rss(sub_inp, planes, weights, hx, sub))


def test_hexplane_fwd_saved_latent_matches_oracle_encoder(sp):
    n = 3001
    hx, inp, planes, weights = _inputs(n, 0.5)
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["latent"] = torch.empty((n, hx.in_dim), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(sp.hex_from_spec(hx), {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights), out=out)
    z = hp.encode(hp.normalise(inp["mu"], inp["frame"], hx.n_frames), planes, hx)
    # four-term bilinear sums of positive plane values (U(0.1, 0.5)): no cancellation
    tol.elementwise(host(out["latent"]), z, tol.FP32_RTOL, "latent", tol.column_groups(hx.in_dim))


# ---------------------------------------------------------------------------
# The energy-flow window: H(w) gates the displacement, w the scale and SH
# offsets (KineticGS notes, "learnable energy-flow activation")
# ---------------------------------------------------------------------------
TAU = 0.02


def _window(inp, n, seed):
    """Window centres and half-widths for the inputs, moved away from the
    threshold of H(w): the GPU decides w >= 1/2 in fp32, the oracle in fp64,
    and the two agree wherever |w - 1/2| exceeds fp32's reach (~1e-6 here)."""
    cr = S.gate_params(n, seed)
    xt = hp.normalise(inp["mu"], inp["frame"], S.HEX.n_frames)
    for _ in range(20):
        amb = np.abs(hp.energy_window(xt, cr, TAU) - 0.5) < 1e-4
        if not amb.any():
            break
        cr[amb, 0] += np.float32(0.01)
    assert not amb.any()
    return cr


@pytest.mark.parametrize("n,bias_scale", [(2053, 0.5), (1, 0.5), (128, 0.0)])
def test_hexplane_gated_fwd_matches_oracle(sp, n, bias_scale):
    hx, inp, planes, weights = _inputs(n, bias_scale, seed=3)
    cr = _window(inp, n, 4)
    gate = dict(cr=cr, tau=TAU)
    out = sp.hexplane_fwd(sp.hex_from_spec(hx), {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights),
                          gate_cr=dev(cr), tau=TAU)
    want = hp.forward(inp, planes, weights, hx, gate=gate)
    got = {k: host(out[k]) for k in HEX_KEYS}
    check_hex_outputs(got, want, mag.hexplane_output_mag(inp, planes, weights, hx, gate))
    frozen = hp.displacement_gate(want["w"]) == 0
    # outside the window the mean is the canonical mean, bit for bit
    assert np.array_equal(got["mu"][frozen], inp["mu"][frozen])
    if n > 1000:
        assert 0.1 < frozen.mean() < 0.9


def _gated_bwd_check(hx, inp, planes, weights, grads, cr, gp, gw, gcr):
    gate = dict(cr=cr, tau=TAU)
    wp, ww, wg = hp.backward(inp, planes, weights, hx, grads, gate=gate, want_gate=True)
    mp, mw, mg = mag.hexplane_rss(inp, planes, weights, hx, grads, gate)
    _check_grads(hx, gp, gw, wp, ww, tol.FP32_GRAD_RTOL, (mp, mw))
    tol.elementwise(host(gcr), wg, tol.FP32_GRAD_RTOL, "grad_cr", tol.column_groups(2, ["c", "r"]), rho=mg)


@pytest.mark.parametrize("n", [1500, 65])
def test_hexplane_gated_bwd_matches_oracle(sp, n):
    hx, inp, planes, weights = _inputs(n, 0.5, seed=5)
    cr = _window(inp, n, 6)
    grads = S.upstream_grads(n, S.HEX_OUT_WIDTHS, 1.0, seed=7)
    h = sp.hex_from_spec(hx)
    gp, gw = _zero_grads(hx)
    gcr = torch.zeros((n, 2), dtype=torch.float32, device="cuda")
    I, P, W, G = {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights), {k: dev(v) for k, v in grads.items()}
    sp.hexplane_bwd(h, I, P, W, G, gp, gw, gate_cr=dev(cr), tau=TAU, grad_cr=gcr)
    _gated_bwd_check(hx, inp, planes, weights, grads, cr, gp, gw, gcr)
    # the window's gradient accumulates, and the saved latent gives the same gradients
    out = {k: torch.empty((n, w), dtype=torch.float32, device="cuda") for k, w in sp.HEX_KEYS}
    out["latent"] = torch.empty((n, hx.in_dim), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(h, I, P, W, out=out, gate_cr=dev(cr), tau=TAU)
    gp2, gw2 = _zero_grads(hx)
    first = gcr.clone()
    sp.hexplane_bwd(h, I, P, W, G, gp2, gw2, latent=out["latent"], gate_cr=dev(cr), tau=TAU, grad_cr=gcr)
    _gated_bwd_check(hx, inp, planes, weights, grads, cr, gp2, gw2, gcr - first)
    # and the saved latent with the saved h1
    out["hidden"] = torch.empty((n, hx.hidden), dtype=torch.float32, device="cuda")
    sp.hexplane_fwd(h, I, P, W, out=out, gate_cr=dev(cr), tau=TAU)
    gp3, gw3 = _zero_grads(hx)
    second = gcr.clone()
    sp.hexplane_bwd(h, I, P, W, G, gp3, gw3, latent=out["latent"], hidden=out["hidden"], gate_cr=dev(cr), tau=TAU,
                    grad_cr=gcr)
    _gated_bwd_check(hx, inp, planes, weights, grads, cr, gp3, gw3, gcr - second)


def test_hexplane_gated_full_size_sampled(sp):
    """The 500k-Gaussian launch with the window: forward on sampled rows, and
    the backward of a subset launched alone."""
    n = S.WORKLOADS["hexplane_fp32"]["N"]
    hx, inp, planes, weights = _inputs(n, 0.5, seed=8)
    cr = _window(inp, n, 9)
    h = sp.hex_from_spec(hx)
    I, P, W = {k: dev(v) for k, v in inp.items()}, dev(planes), dev(weights)
    out = sp.hexplane_fwd(h, I, P, W, gate_cr=dev(cr), tau=TAU)
    rows = np.sort(np.random.default_rng(10).choice(n, 1500, replace=False))
    rows[-1] = n - 1
    sub = {k: v[rows] for k, v in inp.items()}
    gate = dict(cr=cr[rows], tau=TAU)
    want = hp.forward(sub, planes, weights, hx, gate=gate)
    check_hex_outputs({k: host(out[k])[rows] for k in HEX_KEYS}, want,
                      mag.hexplane_output_mag(sub, planes, weights, hx, gate))
    grads = S.upstream_grads(len(rows), S.HEX_OUT_WIDTHS, 1.0, seed=11)
    gp, gw = _zero_grads(hx)
    gcr = torch.zeros((len(rows), 2), dtype=torch.float32, device="cuda")
    sp.hexplane_bwd(h, {k: dev(v) for k, v in sub.items()}, P, W, {k: dev(v) for k, v in grads.items()}, gp, gw,
                    gate_cr=dev(cr[rows]), tau=TAU, grad_cr=gcr)
    _gated_bwd_check(hx, sub, planes, weights, grads, cr[rows], gp, gw, gcr)
