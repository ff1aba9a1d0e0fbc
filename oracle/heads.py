"""Oracle: the paper's attribute-aware decoder (four GELU heads).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: *Implicit 4D Gaussian Splatting for Fast Motion with Large
Inter-Frame Displacements* (SPIN-4DGS), section 3.3 "attribute-aware
decoder": every attribute (scale, rotation, spherical-harmonic colour,
opacity) is predicted by its own head, a three-layer MLP on the shared
latent z (Eq. 10), all heads with GELU activations instead of ReLU; Eq. 11
maps the raw outputs to exp(s^), r^/|r^|, sh^ (identity) and sigma(o^);
the scale is clipped at 20 before the exponential in backprop; Sigma is
Eq. 2.  Section 4: hidden width 64, Adam with linear warm-up and cosine
decay of every parameter group's learning rate to 1e-7.

Readings: "three-layer MLP" = three linear layers in -> hidden -> hidden ->
out with GELU after the first two; GELU is the exact form
x * Phi(x) = x (1 + erf(x / sqrt 2)) / 2 (Hendrycks & Gimpel); the SH output
has 48 values (degree 3, three colour channels); the heads are packed in
the order (scale, rotation, SH, opacity), each as [W1 b1 W2 b2 W3 b3].
"""
from __future__ import annotations

import math
from typing import Dict, List, Tuple

import numpy as np
from scipy.special import erf

from . import decoder, hashgrid

HEADS = ("scale", "rot", "sh", "opacity")
SQRT2 = math.sqrt(2.0)


def gelu(x: np.ndarray) -> np.ndarray:
    return 0.5 * x * (1.0 + erf(x / SQRT2))


def gelu_grad(x: np.ndarray) -> np.ndarray:
    """d gelu/dx = Phi(x) + x phi(x)."""
    return 0.5 * (1.0 + erf(x / SQRT2)) + x * np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def unpack(weights: np.ndarray, spec) -> List[List[Tuple[np.ndarray, np.ndarray]]]:
    w = np.asarray(weights).astype(np.float64)
    heads, o = [], 0
    for h in range(4):
        layers = []
        for out_d, in_d in spec.layer_shapes(h):
            W = w[o:o + out_d * in_d].reshape(out_d, in_d)
            o += out_d * in_d
            b = w[o:o + out_d]
            o += out_d
            layers.append((W, b))
        heads.append(layers)
    assert o == w.size
    return heads


def pack(grads: List[List[Tuple[np.ndarray, np.ndarray]]]) -> np.ndarray:
    return np.concatenate([np.concatenate([dW.reshape(-1), db]) for head in grads for dW, db in head])


def head_forward(z: np.ndarray, layers):
    """y = W3 gelu(W2 gelu(W1 z + b1) + b2) + b3; returns (y, [inputs], [pre-activations])."""
    a = z
    ins, pres = [], []
    for j, (W, b) in enumerate(layers):
        ins.append(a)
        pre = a @ W.T + b
        pres.append(pre)
        a = gelu(pre) if j < 2 else pre
    return a, ins, pres


def head_backward(dy: np.ndarray, layers, ins, pres):
    """Returns (dz, [(dW, db)]) of one head."""
    grads = [None] * 3
    d = dy
    for j in (2, 1, 0):
        W, _ = layers[j]
        if j < 2:
            d = d * gelu_grad(pres[j])
        grads[j] = (d.T @ ins[j], d.sum(axis=0))
        d = d @ W
    return d, grads


def activations(raw: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """Eq. 11 and Eq. 2 on the raw head outputs."""
    s = np.exp(np.minimum(raw["scale"], decoder.SCALE_CLIP))
    r, _ = decoder.normalise_quat(raw["rot"])
    return dict(scale=s, rot=r, sh=raw["sh"].copy(), opacity=decoder.sigmoid(raw["opacity"]),
                cov=decoder.covariance(s, r))


def activations_backward(raw: Dict[str, np.ndarray], grads: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """d loss / d raw output of each head for loss = sum_k <grads[k], output_k>."""
    g = {k: np.asarray(v, np.float64) for k, v in grads.items()}
    sh_ = raw["scale"]
    s = np.exp(np.minimum(sh_, decoder.SCALE_CLIP))
    r, _ = decoder.normalise_quat(raw["rot"])
    ds_cov, dr_cov = decoder.covariance_backward(s, r, g["cov"])
    o = decoder.sigmoid(raw["opacity"])
    return dict(scale=np.where(sh_ <= decoder.SCALE_CLIP, (g["scale"] + ds_cov) * s, 0.0),
                rot=decoder.normalise_quat_backward(raw["rot"], g["rot"] + dr_cov),
                sh=g["sh"].copy(),
                opacity=g["opacity"] * o * (1.0 - o))


def _latent(pos, tables, grid, normalised_input):
    res, xt = decoder._prepare(pos, grid, normalised_input)
    return res, xt, hashgrid.encode(xt, tables, res, grid.log2_T)


def decode_forward(pos, tables, weights, grid, spec, normalised_input=False) -> Dict[str, np.ndarray]:
    """Normalise -> encode -> four heads -> Eq. 11 -> Sigma (fp64)."""
    _, _, z = _latent(pos, tables, grid, normalised_input)
    heads = unpack(weights, spec)
    raw = {name: head_forward(z, heads[h])[0] for h, name in enumerate(HEADS)}
    out = activations(raw)
    out["z"] = z
    return out


def latent_backward(pos, tables, weights, grid, spec, grads, normalised_input=False):
    """(res, xt, dz N x LF, grad_weights packed): the backward up to the
    latent's adjoint dz, which ``hashgrid.scatter_table_grad`` (or, a level
    at a time, ``scatter_table_grad_level``) spreads over the tables."""
    res, xt, z = _latent(pos, tables, grid, normalised_input)
    heads = unpack(weights, spec)
    fw = [head_forward(z, heads[h]) for h in range(4)]
    raw = {name: fw[h][0] for h, name in enumerate(HEADS)}
    dy = activations_backward(raw, grads)
    dz = np.zeros_like(z)
    wgrads = []
    for h, name in enumerate(HEADS):
        d, g = head_backward(dy[name], heads[h], fw[h][1], fw[h][2])
        dz += d
        wgrads.append(g)
    return res, xt, dz, pack(wgrads)


def decode_backward(pos, tables, weights, grid, spec, grads, normalised_input=False):
    """(grad_tables L x T x F, grad_weights packed like ``weights``)."""
    res, xt, dz, gw = latent_backward(pos, tables, weights, grid, spec, grads, normalised_input)
    return hashgrid.scatter_table_grad(dz, xt, res, grid.log2_T, grid.L, grid.F), gw


def lr_warmup_cosine(step: int, lr_max: float, lr_min: float, warmup: int, total: int) -> float:
    """Learning rate at optimiser step ``step`` (counted from 1): linear
    warm-up from 0 to lr_max over the first ``warmup`` steps, then a cosine
    from lr_max down to lr_min at step ``total`` (and lr_min after)."""
    if warmup > 0 and step <= warmup:
        return lr_max * step / warmup
    if step >= total:
        return lr_min
    u = (step - warmup) / max(total - warmup, 1)
    return lr_min + 0.5 * (lr_max - lr_min) * (1.0 + math.cos(math.pi * u))
