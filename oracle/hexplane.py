"""Oracle: HexPlane encoder and the two-branch deformation network.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  fp64 except the
fp32 cell decision.

Source: the 4D Gaussian Splatting reading notes (Wu et al.'s 4DGaussians),
section 3.1 (six feature planes XY, XZ, YZ, XT, YT, ZT; project the point
onto each, sample bilinearly, join the samples into one spatio-temporal
feature) and section 3.2 / 2.2 (a small MLP on that feature with a geometry
branch giving position, rotation and scale offsets and an appearance branch
giving spherical-harmonic offsets; the rotation is renormalised, the scale
lives in log space).  Sigma is SPIN-4DGS section 3.1 Eq. 2.

Readings: planes at spatial resolutions 64/128/256 and 75 time samples, 32
channels, channel-last [rows = second axis][cols = first axis][C]; samples
joined by concatenation (scale-major, then plane, then channel) into 576
features; align-corners bilinear (p = x~ * (res - 1), cell clamped to
[0, res-2]); x~ = (mu + 1)/2 clamped to [0,1]; t~ = frame / 149; trunk
576 -> 64 -> 64 with ReLU, then one 58-row linear layer
[d_mu 3 | d_q 4 | d_logs 3 | d_sh 48]; outputs mu' = mu + d_mu,
q' = (q + d_q)/||q + d_q||, s' = exp(log s + d_logs), sh' = sh + d_sh and
Sigma(s', q').

Optional energy-flow window (KineticGS notes, "learnable energy-flow
activation"): each Gaussian carries a window centre c and half-width r, and
w = sigma((t~ - (c - r))/tau) sigma(((c + r) - t~)/tau) on the normalised
time t~.  The notes gate the spatial displacement with a binary H(w) in
{0, 1}, so that a Gaussian moves only inside its window, and modulate the
features and the scale continuously by w.  Readings: H(w) = [w >= 1/2] (the
notes give no threshold; 1/2 is where the window's two edges sit);
mu' = mu + H(w) d_mu, s' = exp(log s + w d_logs), sh' = sh + w d_sh; the
rotation offset, which the notes do not name among the modulated
quantities, is left as it is.  H has zero derivative, so c and r receive
gradient only through w (d_logs and d_sh).
"""
from __future__ import annotations

from typing import Dict, List, Tuple

import numpy as np

from . import decoder

F32 = np.float32
PLANE_AXES = ((0, 1), (0, 2), (1, 2), (0, 3), (1, 3), (2, 3))   # XY XZ YZ XT YT ZT


def plane_offsets(hx) -> List[int]:
    offs, o = [], 0
    for rows, cols in hx.plane_shapes():
        offs.append(o)
        o += rows * cols * hx.channels
    return offs


def normalise(mu: np.ndarray, frame: np.ndarray, n_frames: int) -> np.ndarray:
    mu = np.asarray(mu, F32)
    xt = np.empty((mu.shape[0], 4), F32)
    xt[:, :3] = (mu + F32(1)) * F32(0.5)
    xt[:, 3] = np.asarray(frame).astype(F32) / F32(n_frames - 1)
    xt = np.where(np.isnan(xt), F32(0), xt)
    return np.minimum(np.maximum(xt, F32(0)), F32(1)).astype(F32)


def _cell(x: np.ndarray, r: int):
    p = x * F32(r - 1)
    i = np.clip(np.floor(p).astype(np.int64), 0, r - 2)
    return i, (p - i.astype(F32)).astype(np.float64)


def _resolution(hx, scale: int, axis: int) -> int:
    return hx.time_res if axis == 3 else scale


def _corners(xt, hx):
    """Yields (feature offset, plane flat offset, rows, cols, [(flat idx, weight)] x 4)."""
    offs = plane_offsets(hx)
    C = hx.channels
    k = 0
    for si, m in enumerate(hx.scales):
        for pi, (a, b) in enumerate(PLANE_AXES):
            ra, rb = _resolution(hx, m, a), _resolution(hx, m, b)
            ia, wa = _cell(xt[:, a], ra)
            ib, wb = _cell(xt[:, b], rb)
            corners = []
            for db in (0, 1):
                for da in (0, 1):
                    w = (wa if da else 1 - wa) * (wb if db else 1 - wb)
                    cell = (ib + db) * ra + (ia + da)            # row-major [rows][cols]
                    corners.append((offs[k] + cell * C, w))
            yield (si * 6 + pi) * C, corners
            k += 1


def encode(xt: np.ndarray, planes: np.ndarray, hx) -> np.ndarray:
    """N x 576 fp64 concatenated bilinear samples."""
    planes = np.asarray(planes).astype(np.float64)
    N, C = xt.shape[0], hx.channels
    z = np.zeros((N, hx.in_dim))
    for fo, corners in _corners(xt, hx):
        for c in range(C):
            acc = np.zeros(N)
            for flat, w in corners:
                acc += w * np.take(planes, flat + c)
            z[:, fo + c] = acc
    return z


def scatter_plane_grad(dz: np.ndarray, xt: np.ndarray, hx) -> np.ndarray:
    grad = np.zeros(hx.n_plane_floats())
    n = grad.size
    ch = np.arange(hx.channels)
    for fo, corners in _corners(xt, hx):
        g = dz[:, fo:fo + hx.channels]                       # N x C
        idx = np.concatenate([(flat[:, None] + ch).reshape(-1) for flat, _ in corners])
        val = np.concatenate([(w[:, None] * g).reshape(-1) for _, w in corners])
        grad += np.bincount(idx, weights=val, minlength=n)
    return grad


def energy_window(xt: np.ndarray, gate_cr, tau: float) -> np.ndarray:
    """The double-sigmoid window w on the normalised time t~ (fp64)."""
    cr = np.asarray(gate_cr, np.float64)
    return decoder.temporal_gate(xt[:, 3].astype(np.float64), cr[:, 0], cr[:, 1], float(np.float32(tau)))


def displacement_gate(w: np.ndarray) -> np.ndarray:
    """H(w) in {0, 1}: 1 inside the window, read as w >= 1/2."""
    return (np.asarray(w) >= 0.5).astype(np.float64)


def _outputs(y, inp, w=None):
    """Deformed Gaussians from the head output y; with the window weight w
    the displacement is gated by H(w) and the scale and SH offsets scaled by w."""
    mu = np.asarray(inp["mu"], np.float64)
    ones = np.ones(y.shape[0])
    wm = ones if w is None else w
    hm = ones if w is None else displacement_gate(w)
    qh = np.asarray(inp["q_can"], np.float64) + y[:, 3:7]
    q, _ = decoder.normalise_quat(qh)
    s = np.exp(np.asarray(inp["logs_can"], np.float64) + wm[:, None] * y[:, 7:10])
    return dict(mu=mu + hm[:, None] * y[:, 0:3], rot=q, scale=s,
                sh=np.asarray(inp["sh_can"], np.float64) + wm[:, None] * y[:, 10:58],
                cov=decoder.covariance(s, q)), qh


def _window(xt, hx, gate):
    if gate is None:
        return None
    return energy_window(xt, gate["cr"], gate["tau"])


def forward(inp: Dict[str, np.ndarray], planes, weights, hx, gate=None) -> Dict[str, np.ndarray]:
    """``gate``: None, or dict(cr=N x 2 (c, r), tau=...) for the energy-flow window."""
    xt = normalise(inp["mu"], inp["frame"], hx.n_frames)
    z = encode(xt, planes, hx)
    layers = decoder.unpack_layers(weights, hx.layer_shapes())
    y, acts, _ = decoder.mlp_forward(z, layers)
    w = _window(xt, hx, gate)
    out, _ = _outputs(y, inp, w)
    out["z"] = z
    out["h1"] = acts[1]   # the first hidden layer, relu(W1 z + b1)
    if w is not None:
        out["w"] = w
    return out


def backward(inp, planes, weights, hx, grads, gate=None, want_gate=False):
    """Gradients of sum_k <grads[k], output_k> w.r.t. planes and weights, and
    with ``want_gate`` (gated only) w.r.t. the window's (c, r), N x 2."""
    xt = normalise(inp["mu"], inp["frame"], hx.n_frames)
    z = encode(xt, planes, hx)
    layers = decoder.unpack_layers(weights, hx.layer_shapes())
    y, acts, pres = decoder.mlp_forward(z, layers)
    w = _window(xt, hx, gate)
    out, qh = _outputs(y, inp, w)
    g = {k: np.asarray(v, np.float64) for k, v in grads.items()}
    ds_cov, dq_cov = decoder.covariance_backward(out["scale"], out["rot"], g["cov"])
    dlogs = (g["scale"] + ds_cov) * out["scale"]          # d loss / d (log s + w d_logs)
    wm = np.ones(y.shape[0]) if w is None else w
    hm = np.ones(y.shape[0]) if w is None else displacement_gate(w)
    dy = np.zeros_like(y)
    dy[:, 0:3] = hm[:, None] * g["mu"]
    dy[:, 3:7] = decoder.normalise_quat_backward(qh, g["rot"] + dq_cov)
    dy[:, 7:10] = wm[:, None] * dlogs
    dy[:, 10:58] = wm[:, None] * g["sh"]
    dz, wgrads = decoder.mlp_backward(dy, layers, acts, pres)
    result = (scatter_plane_grad(dz, xt, hx), decoder.pack_layers(wgrads))
    if want_gate:
        assert w is not None, "the window gradient needs a gated call"
        # H(w) is piecewise constant: only the w-scaled offsets carry d loss / d w
        dw = np.sum(dlogs * y[:, 7:10], axis=1) + np.sum(g["sh"] * y[:, 10:58], axis=1)
        cr = np.asarray(gate["cr"], np.float64)
        dwdc, dwdr = decoder.temporal_gate_grad(xt[:, 3].astype(np.float64), cr[:, 0], cr[:, 1],
                                                float(np.float32(gate["tau"])))
        result = result + (np.stack([dw * dwdc, dw * dwdr], axis=1),)
    return result
