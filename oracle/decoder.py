"""Oracle: attribute decoder, activations, covariance, backward pass, Adam.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  All arithmetic fp64.

Sources, on *Implicit 4D Gaussian Splatting for Fast Motion with Large
Inter-Frame Displacements* (SPIN-4DGS):

* section 3.1, Eq. 2: Sigma = R S S^T R^T with S = diag(s) and R the rotation
  matrix of the quaternion r, which keeps Sigma positive semi-definite;
* section 3.3 "attribute-aware decoder", Eq. 10: one head per attribute on
  the shared latent z;
* section 3.3, Eq. 11: s = exp(s^), r = r^/||r^||, o = sigmoid(o^); the
  scale pre-activation is clipped at 20 ("clip(s^, max=20)"), the scale bias
  starts at -5, the rotation bias at (1,0,0,0) (real part first) and the
  opacity bias at logit(0.1);
* section 4 "implementation details": Adam (Kingma & Ba).

The decoder form follows the workload definition: a shared ReLU trunk
(n_hidden layers of width ``hidden``) followed by one linear layer of 11 rows
[scale 3 | rotation 4 | rgb 3 | opacity 1]; colour is sigmoid(rgb^).  The
page's own per-head three-layer GELU form is not what is computed here.

Optional temporal gate (KineticGS notes, "learnable energy-flow activation"):
w = sigmoid((t - (c - r))/tau) * sigmoid(((c + r) - t)/tau), multiplying the
opacity, with t the normalised time.

Readings: ||r^|| is floored at 1e-12; the clip passes the gradient where
s^ <= 20 and blocks it above (the clamp convention); ReLU passes the
gradient where its input is > 0; Sigma is returned packed as
(xx, xy, xz, yy, yz, zz) and an upstream gradient on a packed off-diagonal
entry counts once.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from . import hashgrid

SCALE_CLIP = 20.0
NORM_FLOOR = 1e-12
PACK = ((0, 0), (0, 1), (0, 2), (1, 1), (1, 2), (2, 2))


# ---------------------------------------------------------------------------
# Parameters
# ---------------------------------------------------------------------------
def unpack_layers(flat: np.ndarray, shapes: Sequence[Tuple[int, int]]) -> List[Tuple[np.ndarray, np.ndarray]]:
    """Flat vector -> [(W [out][in], b [out])] in fp64 (values read exactly)."""
    flat = np.asarray(flat).astype(np.float64)
    out, o = [], 0
    for (m, k) in shapes:
        W = flat[o:o + m * k].reshape(m, k)
        o += m * k
        b = flat[o:o + m]
        o += m
        out.append((W, b))
    assert o == flat.size, (o, flat.size)
    return out


def pack_layers(layers: Sequence[Tuple[np.ndarray, np.ndarray]]) -> np.ndarray:
    return np.concatenate([np.concatenate([W.reshape(-1), b]) for W, b in layers])


# ---------------------------------------------------------------------------
# Elementary pieces
# ---------------------------------------------------------------------------
def sigmoid(x):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def quat_to_rotmat(q: np.ndarray) -> np.ndarray:
    """N x 4 unit quaternions (w, x, y, z) -> N x 3 x 3 rotation matrices."""
    w, x, y, z = q[:, 0], q[:, 1], q[:, 2], q[:, 3]
    R = np.empty((q.shape[0], 3, 3))
    R[:, 0, 0] = 1 - 2 * (y * y + z * z)
    R[:, 0, 1] = 2 * (x * y - w * z)
    R[:, 0, 2] = 2 * (x * z + w * y)
    R[:, 1, 0] = 2 * (x * y + w * z)
    R[:, 1, 1] = 1 - 2 * (x * x + z * z)
    R[:, 1, 2] = 2 * (y * z - w * x)
    R[:, 2, 0] = 2 * (x * z - w * y)
    R[:, 2, 1] = 2 * (y * z + w * x)
    R[:, 2, 2] = 1 - 2 * (x * x + y * y)
    return R


def rotmat_jacobian(q: np.ndarray) -> np.ndarray:
    """N x 3 x 3 x 4: d R_ij / d q_k of ``quat_to_rotmat`` (same polynomials)."""
    w, x, y, z = q[:, 0], q[:, 1], q[:, 2], q[:, 3]
    J = np.zeros((q.shape[0], 3, 3, 4))
    J[:, 0, 0] = np.stack([0 * w, 0 * x, -4 * y, -4 * z], 1)
    J[:, 0, 1] = np.stack([-2 * z, 2 * y, 2 * x, -2 * w], 1)
    J[:, 0, 2] = np.stack([2 * y, 2 * z, 2 * w, 2 * x], 1)
    J[:, 1, 0] = np.stack([2 * z, 2 * y, 2 * x, 2 * w], 1)
    J[:, 1, 1] = np.stack([0 * w, -4 * x, 0 * y, -4 * z], 1)
    J[:, 1, 2] = np.stack([-2 * x, -2 * w, 2 * z, 2 * y], 1)
    J[:, 2, 0] = np.stack([-2 * y, 2 * z, -2 * w, 2 * x], 1)
    J[:, 2, 1] = np.stack([2 * x, 2 * w, 2 * z, 2 * y], 1)
    J[:, 2, 2] = np.stack([0 * w, -4 * x, -4 * y, 0 * z], 1)
    return J


def covariance(s: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Eq. 2: Sigma = R diag(s) diag(s)^T R^T, packed (xx, xy, xz, yy, yz, zz)."""
    R = quat_to_rotmat(q)
    M = R * s[:, None, :]                      # M = R S
    Sig = M @ np.transpose(M, (0, 2, 1))
    return np.stack([Sig[:, i, j] for i, j in PACK], axis=1)


def covariance_backward(s: np.ndarray, q: np.ndarray, g_cov: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Gradients of sum(g_cov * covariance(s, q)) w.r.t. s and q."""
    R = quat_to_rotmat(q)
    G = np.zeros((s.shape[0], 3, 3))
    for k, (i, j) in enumerate(PACK):
        if i == j:
            G[:, i, i] = g_cov[:, k]
        else:
            G[:, i, j] = 0.5 * g_cov[:, k]
            G[:, j, i] = 0.5 * g_cov[:, k]
    M = R * s[:, None, :]
    dM = 2.0 * G @ M                            # d tr(G M M^T) / dM
    ds = np.sum(dM * R, axis=1)                 # M_ik = R_ik s_k
    dR = dM * s[:, None, :]
    dq = np.einsum("nij,nijk->nk", dR, rotmat_jacobian(q))
    return ds, dq


def normalise_quat(rh: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    nrm = np.sqrt(np.sum(rh * rh, axis=1))
    den = np.maximum(nrm, NORM_FLOOR)
    return rh / den[:, None], nrm


def normalise_quat_backward(rh: np.ndarray, g_r: np.ndarray) -> np.ndarray:
    r, nrm = normalise_quat(rh)
    proj = g_r - r * np.sum(r * g_r, axis=1, keepdims=True)
    return np.where((nrm > NORM_FLOOR)[:, None], proj / np.maximum(nrm, NORM_FLOOR)[:, None],
                    g_r / NORM_FLOOR)


def temporal_gate(t: np.ndarray, c: np.ndarray, r: np.ndarray, tau: float) -> np.ndarray:
    """KineticGS double-sigmoid window on the normalised time t."""
    return sigmoid((t - (c - r)) / tau) * sigmoid(((c + r) - t) / tau)


def temporal_gate_grad(t: np.ndarray, c: np.ndarray, r: np.ndarray, tau: float) -> Tuple[np.ndarray, np.ndarray]:
    """(dw/dc, dw/dr) of w = a b, a = sigma((t - (c - r))/tau), b = sigma(((c + r) - t)/tau).

    sigma' = sigma (1 - sigma): da/dc = -a(1-a)/tau, db/dc = b(1-b)/tau, so
    dw/dc = a b (a - b)/tau; da/dr = a(1-a)/tau, db/dr = b(1-b)/tau, so
    dw/dr = a b (2 - a - b)/tau."""
    a = sigmoid((t - (c - r)) / tau)
    b = sigmoid(((c + r) - t) / tau)
    return a * b * (a - b) / tau, a * b * (2.0 - a - b) / tau


# ---------------------------------------------------------------------------
# Network
# ---------------------------------------------------------------------------
def mlp_forward(z: np.ndarray, layers) -> Tuple[np.ndarray, List[np.ndarray], List[np.ndarray]]:
    """Trunk (ReLU) then linear head.  Returns (y, inputs per layer, pre-acts)."""
    a = z
    acts, pres = [], []
    for j, (W, b) in enumerate(layers):
        acts.append(a)
        pre = a @ W.T + b
        pres.append(pre)
        a = np.maximum(pre, 0.0) if j < len(layers) - 1 else pre
    return a, acts, pres


def mlp_backward(dy: np.ndarray, layers, acts, pres):
    """Returns (dz, [(dW, db)])."""
    grads = [None] * len(layers)
    d = dy
    for j in range(len(layers) - 1, -1, -1):
        W, _ = layers[j]
        if j < len(layers) - 1:
            d = d * (pres[j] > 0)
        grads[j] = (d.T @ acts[j], d.sum(axis=0))
        d = d @ W
    return d, grads


def heads_forward(y: np.ndarray, gate: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Eq. 11 activations on the 11 head outputs, then Eq. 2."""
    sh, rh, ch, oh = y[:, 0:3], y[:, 3:7], y[:, 7:10], y[:, 10]
    s = np.exp(np.minimum(sh, SCALE_CLIP))
    r, _ = normalise_quat(rh)
    rgb = sigmoid(ch)
    o = sigmoid(oh)
    if gate is not None:
        o = o * gate
    return dict(scale=s, rot=r, rgb=rgb, opacity=o[:, None], cov=covariance(s, r))


def heads_backward(y: np.ndarray, grads: Dict[str, np.ndarray], gate: Optional[np.ndarray] = None) -> np.ndarray:
    """d loss / d y for loss = sum over outputs of grads[k] * output[k]."""
    sh, rh, ch, oh = y[:, 0:3], y[:, 3:7], y[:, 7:10], y[:, 10]
    s = np.exp(np.minimum(sh, SCALE_CLIP))
    r, _ = normalise_quat(rh)
    ds_cov, dr_cov = covariance_backward(s, r, grads["cov"].astype(np.float64))
    ds = grads["scale"] + ds_cov
    dr = grads["rot"] + dr_cov
    dy = np.zeros_like(y)
    dy[:, 0:3] = np.where(sh <= SCALE_CLIP, ds * s, 0.0)
    dy[:, 3:7] = normalise_quat_backward(rh, dr)
    rgb = sigmoid(ch)
    dy[:, 7:10] = grads["rgb"] * rgb * (1.0 - rgb)
    so = sigmoid(oh)
    go = grads["opacity"][:, 0] * (gate if gate is not None else 1.0)
    dy[:, 10] = go * so * (1.0 - so)
    return dy


# ---------------------------------------------------------------------------
# End to end
# ---------------------------------------------------------------------------
def _prepare(pos, grid, normalised_input: bool):
    res = hashgrid.grid_resolutions(grid.L, grid.nmin_s, grid.nmax_s, grid.nmin_t, grid.nmax_t)
    if normalised_input:
        xt = hashgrid._clamp01(np.asarray(pos, np.float32))
    else:
        xt = hashgrid.normalise(pos, grid.t_min, grid.t_max)
    return res, xt


def _gate_for(xt, mlp, gate_cr):
    if not mlp.gate:
        return None
    t = xt[:, 3].astype(np.float64)
    cr = np.asarray(gate_cr, np.float64)
    return temporal_gate(t, cr[:, 0], cr[:, 1], float(np.float32(mlp.tau)))


def decode_forward(pos, tables, weights, grid, mlp, gate_cr=None, normalised_input=False):
    """Normalise -> encode -> trunk + heads -> activations -> Sigma (fp64)."""
    res, xt = _prepare(pos, grid, normalised_input)
    z = hashgrid.encode(xt, tables, res, grid.log2_T)
    layers = unpack_layers(weights, mlp.layer_shapes())
    y, _, _ = mlp_forward(z, layers)
    out = heads_forward(y, _gate_for(xt, mlp, gate_cr))
    out["z"] = z
    return out


def decode_backward(pos, tables, weights, grid, mlp, grads, gate_cr=None, normalised_input=False,
                    want_pos=False, want_gate=False):
    """Gradients of sum_k <grads[k], output_k> w.r.t. the tables and weights.

    Returns (grad_tables L x T x F, grad_weights packed like ``weights``), and
    with ``want_pos`` also grad_pos N x 3: the gradient w.r.t. the spatial
    position (x, y, z) through the interpolation weights and Eq. 7 (w.r.t. the
    normalised coordinates themselves when ``normalised_input``).  The
    timestamp is data, not a parameter, and gets none.  With ``want_gate``
    (gated decoders) also grad_cr N x 2, the gradient w.r.t. the window
    centre c and half-width r of the KineticGS gate: o = sigma(o^) w, so
    dloss/dw = g_o sigma(o^), times (dw/dc, dw/dr)."""
    res, xt = _prepare(pos, grid, normalised_input)
    z = hashgrid.encode(xt, tables, res, grid.log2_T)
    layers = unpack_layers(weights, mlp.layer_shapes())
    y, acts, pres = mlp_forward(z, layers)
    g64 = {k: np.asarray(v, np.float64) for k, v in grads.items()}
    dy = heads_backward(y, g64, _gate_for(xt, mlp, gate_cr))
    dz, wgrads = mlp_backward(dy, layers, acts, pres)
    gt = hashgrid.scatter_table_grad(dz, xt, res, grid.log2_T, grid.L, grid.F)
    result = [gt, pack_layers(wgrads)]
    if want_pos:
        gx = hashgrid.encode_position_grad(dz, xt, tables, res, grid.log2_T)[:, :3]
        p32 = np.asarray(pos, np.float32)
        if normalised_input:
            gpos = gx * hashgrid.clamp_passes(p32[:, :3])
        else:
            gpos = np.einsum("ni,nij->nj", gx, hashgrid.contraction_jacobian(p32))
        result.append(gpos)
    if want_gate:
        assert mlp.gate, "the gate gradient needs a gated decoder"
        t = xt[:, 3].astype(np.float64)
        cr = np.asarray(gate_cr, np.float64)
        dc, dr = temporal_gate_grad(t, cr[:, 0], cr[:, 1], float(np.float32(mlp.tau)))
        gw = g64["opacity"][:, 0] * sigmoid(y[:, 10])
        result.append(np.stack([gw * dc, gw * dr], axis=1))
    return tuple(result)


def adam_step(p, g, m, v, step: int, lr: float, b1: float, b2: float, eps: float):
    """Kingma & Ba with bias correction; ``step`` counts from 1.  fp64."""
    p = np.asarray(p, np.float64)
    g = np.asarray(g, np.float64)
    m = b1 * np.asarray(m, np.float64) + (1 - b1) * g
    v = b2 * np.asarray(v, np.float64) + (1 - b2) * g * g
    mh = m / (1 - b1 ** step)
    vh = v / (1 - b2 ** step)
    return p - lr * mh / (np.sqrt(vh) + eps), m, v
