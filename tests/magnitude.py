"""Magnitudes of the terms behind every value the parity tests compare.

Test infrastructure for the parity bound (``tests/tol.py``).  Every value the
decoders compute is built from sums: a table-gradient entry sums w_c * dz
over the positions that reach it, dz sums dh1_j * W1_jf over the hidden
units, dh1 sums over the next layer, a covariance entry sums over three
axes, and so on.  When the terms of such a sum cancel, the result is small
next to them, and no fp32 (or fp16-operand) arithmetic can hold it to a
bound relative to its own size: each term carries a rounding error of about
eps times its own magnitude, and those errors do not cancel.

The magnitude m(v) of a value is therefore defined through the computation
that produces it: for v = sum_k t_k, m(v) = sqrt(sum_k m(t_k)^2) (independent
errors add in quadrature), for a product m(a b) = m(a) m(b), for an input
m(x) = |x|, and for a smooth activation f, m(f(v)) = max(|f(v)|, |f'(v)| m(v))
(a ReLU mask passes m where it passes the value).  Without cancellation
anywhere m(v) = |v|; with it, m(v) is what the rounding errors scale with.
The element-wise bound then reads

    |g - o| <= rtol * max(|o|, floor * max|o|_group, m(o))

with rtol 1e-5 for fp32 arithmetic (about 170 fp32 ulps) and 1e-2 for the
fp16 path (fp16 operands round at 2^-12).  A mistake -- a wrong index, a
transposed weight, a dropped term -- moves a value by the order of its terms,
i.e. of m itself, and still fails.

Everything here calls the oracle's own pieces (normalisation, corner
selection and weights, the network's forward pass, R(q)) and only propagates
magnitudes; it computes no result the tests compare against.
"""
from __future__ import annotations

import numpy as np

from oracle import decoder as dec
from oracle import hashgrid as hg
from oracle import heads as hd
from oracle import hexplane as hp


def _relu_grad(p):
    return (p > 0).astype(np.float64)


# ---------------------------------------------------------------------------
# Networks
# ---------------------------------------------------------------------------
def mlp_forward_mag(mz, layers, pres, act_grad, act):
    """Magnitudes of every layer's input (mz first) and of the output y.

    pre_j = a_j W_j^T + b_j: m(pre_j) = sqrt(m(a_j)^2 (W_j^2)^T + b_j^2);
    a_{j+1} = act(pre_j): m = max(|act(pre_j)|, |act'(pre_j)| m(pre_j))."""
    ms = [mz]
    m = mz
    for j, (W, b) in enumerate(layers):
        mp = np.sqrt(m * m @ (W * W).T + b * b)
        if j < len(layers) - 1:
            m = np.maximum(np.abs(act(pres[j])), np.abs(act_grad(pres[j])) * mp)
            ms.append(m)
        else:
            m = mp
    return ms, m


def mlp_backward_mag(mdy, layers, pres, act_grad):
    """Magnitudes of each layer's output delta and of dz:
    d_in = delta_j W_j: m = sqrt(m(delta_j)^2 W_j^2); delta_{j-1} = d_in act'(pre)."""
    mdeltas = [None] * len(layers)
    m = mdy
    for j in range(len(layers) - 1, -1, -1):
        if j < len(layers) - 1:
            m = m * np.abs(act_grad(pres[j]))
        mdeltas[j] = m
        m = np.sqrt(m * m @ (layers[j][0] ** 2))
    return m, mdeltas


def weight_mag(macts, mdeltas):
    """Packed [W0 b0 W1 b1 ...]: dW_jk = sum_n d_nj a_nk, db_j = sum_n d_nj."""
    out = []
    for a, d in zip(macts, mdeltas):
        out.append(np.sqrt((d * d).T @ (a * a)).reshape(-1))
        out.append(np.sqrt(np.sum(d * d, axis=0)))
    return np.concatenate(out)


# ---------------------------------------------------------------------------
# Encoders
# ---------------------------------------------------------------------------
def encode_mag(xt, tables, res, log2_T):
    """N x LF: sqrt(sum_c (w_c table[idx_c, f])^2), the terms of Eq. 9."""
    L, T, F = tables.shape
    _, frac, idx = hg.corner_select(xt, res, log2_T)
    w2 = hg.corner_weights(frac) ** 2
    out = np.zeros((xt.shape[0], L * F))
    for l in range(L):
        for f in range(F):
            col = np.ascontiguousarray(tables[l, :, f]).astype(np.float64)
            out[:, l * F + f] = np.sqrt(np.sum(w2[:, l, :] * np.take(col, idx[:, l, :].astype(np.int64)) ** 2, axis=1))
    return out


def table_mag(mdz, xt, res, log2_T, L, F):
    """L x T x F: sqrt(sum over (position, corner) reaching the entry of (w_c m(dz))^2)."""
    T = 1 << log2_T
    _, frac, idx = hg.corner_select(xt, res, log2_T)
    w2 = hg.corner_weights(frac) ** 2
    out = np.zeros((L, T, F), np.float32)       # a magnitude: fp32 storage is ample
    for l in range(L):
        for f in range(F):
            g2 = mdz[:, l * F + f] ** 2
            out[l, :, f] = np.sqrt(np.bincount(idx[:, l, :].astype(np.int64).reshape(-1),
                                               weights=(w2[:, l, :] * g2[:, None]).reshape(-1), minlength=T))
    return out


def position_mag(mdz, xt, tables, res, log2_T, jac=None):
    """N x 3: the terms (res_d - 1) (dz_l . e_c) dW_c/dw_d over levels,
    corners and features, with m(dz) for dz, carried through the Jacobian
    ``jac`` (N x 3 x 3, rows = normalised axis) in squares."""
    L, T, F = tables.shape
    _, frac, idx = hg.corner_select(xt, res, log2_T)
    w = frac.astype(np.float64)
    N = xt.shape[0]
    s2 = np.zeros((N, 4))
    for l in range(L):
        e2 = np.zeros((N, 16))
        for f in range(F):
            col = np.ascontiguousarray(tables[l, :, f]).astype(np.float64)
            e2 += (mdz[:, l * F + f][:, None] * np.take(col, idx[:, l, :].astype(np.int64))) ** 2
        for d in range(4):
            for c in range(16):
                dw = np.ones(N)
                for e in range(4):
                    if e != d:
                        dw = dw * (w[:, l, e] if (c >> e) & 1 else 1.0 - w[:, l, e])
                s2[:, d] += (int(res[l, d]) - 1) ** 2 * e2[:, c] * dw * dw
    if jac is None:
        return np.sqrt(s2[:, :3])
    return np.sqrt(np.einsum("ni,nij->nj", s2[:, :3], jac ** 2))


# ---------------------------------------------------------------------------
# Eq. 11 and Eq. 2 adjoints
# ---------------------------------------------------------------------------
def cov_mag(scale):
    """N x 6: every entry of Sigma = R diag(s^2) R^T is computed from R's
    entries, which are O(1) and carry absolute rounding errors; the error of
    any entry therefore scales with the spectral norm max_k s_k^2."""
    return np.repeat(np.max(np.asarray(scale, np.float64) ** 2, axis=1, keepdims=True), 6, axis=1)


def _cov_backward_mag(s, q, g_cov):
    """Magnitudes of (ds, dq) of Eq. 2's adjoint: ds_k = sum_i dM_ik R_ik with
    dM = 2 G M, and dq = sum_ij dR_ij dR_ij/dq with dR = dM s."""
    R = dec.quat_to_rotmat(q)
    G = np.zeros((s.shape[0], 3, 3))
    for k, (i, j) in enumerate(dec.PACK):
        if i == j:
            G[:, i, i] = g_cov[:, k]
        else:
            G[:, i, j] = G[:, j, i] = 0.5 * g_cov[:, k]
    M = R * s[:, None, :]
    mdM = 2.0 * np.sqrt(np.einsum("nij,njk->nik", G * G, M * M))
    mds = np.sqrt(np.sum((mdM * R) ** 2, axis=1))
    mdR = mdM * s[:, None, :]
    mdq = np.sqrt(np.einsum("nij,nijk->nk", mdR ** 2, dec.rotmat_jacobian(q) ** 2))
    return mds, mdq


def _sigmoid_adjoint_mag(g, x):
    """g sigma(x) (1 - sigma(x)): 1 - sigma has the terms 1 and sigma."""
    sg = dec.sigmoid(x)
    return np.abs(g) * sg * np.sqrt(1.0 + sg * sg)


def _rotation_adjoint_mag(rh, g_r, mdq):
    """(g - r (r . g))/||r^||: every component's terms are bounded by the row
    norm of g (with the covariance part at its magnitude)."""
    nrm = np.maximum(np.sqrt(np.sum(rh * rh, axis=1)), dec.NORM_FLOOR)
    row = np.sqrt(np.sum(g_r * g_r + mdq * mdq, axis=1)) / nrm
    return np.repeat(row[:, None], 4, axis=1)


def _scale_adjoint_mag(sh, s, g_s, mds):
    return np.where(sh <= dec.SCALE_CLIP, s * np.sqrt(g_s * g_s + mds * mds), 0.0)


def decoder_head_adjoint_mag(y, g, gate=None):
    """N x 11 magnitudes of ``oracle.decoder.heads_backward``'s dy."""
    sh, rh, ch, oh = y[:, 0:3], y[:, 3:7], y[:, 7:10], y[:, 10]
    s = np.exp(np.minimum(sh, dec.SCALE_CLIP))
    r, _ = dec.normalise_quat(rh)
    mds, mdq = _cov_backward_mag(s, r, g["cov"])
    m = np.zeros_like(y)
    m[:, 0:3] = _scale_adjoint_mag(sh, s, g["scale"], mds)
    m[:, 3:7] = _rotation_adjoint_mag(rh, g["rot"], mdq)
    m[:, 7:10] = _sigmoid_adjoint_mag(g["rgb"], ch)
    go = g["opacity"][:, 0] * (gate if gate is not None else 1.0)
    m[:, 10] = _sigmoid_adjoint_mag(go, oh)
    return m


# ---------------------------------------------------------------------------
# Per decoder: (tables, packed weights[, positions]) magnitudes
# ---------------------------------------------------------------------------
def decoder_rss(pos, tables, weights, grid, mlp, grads, gate_cr=None, normalised_input=False, want_pos=False):
    """The hash-grid decoder with the shared ReLU trunk."""
    res, xt = dec._prepare(pos, grid, normalised_input)
    z = hg.encode(xt, tables, res, grid.log2_T)
    layers = dec.unpack_layers(weights, mlp.layer_shapes())
    y, acts, pres = dec.mlp_forward(z, layers)
    g64 = {k: np.asarray(v, np.float64) for k, v in grads.items()}
    macts, _ = mlp_forward_mag(encode_mag(xt, tables, res, grid.log2_T), layers, pres, _relu_grad,
                               lambda p: np.maximum(p, 0.0))
    mdy = decoder_head_adjoint_mag(y, g64, dec._gate_for(xt, mlp, gate_cr))
    mdz, mdeltas = mlp_backward_mag(mdy, layers, pres, _relu_grad)
    out = [table_mag(mdz, xt, res, grid.log2_T, grid.L, grid.F), weight_mag(macts, mdeltas)]
    if want_pos:
        jac = None if normalised_input else hg.contraction_jacobian(pos)
        out.append(position_mag(mdz, xt, tables, res, grid.log2_T, jac))
    return tuple(out)


def table_mag_level(mdz, xt, res, log2_T, l, F):
    """Level l of ``table_mag``, T x F."""
    T = 1 << log2_T
    _, frac, idx = hg.corner_select(xt, res, log2_T)
    w2 = hg.corner_weights(frac) ** 2
    out = np.zeros((T, F))
    for f in range(F):
        g2 = mdz[:, l * F + f] ** 2
        out[:, f] = np.sqrt(np.bincount(idx[:, l, :].astype(np.int64).reshape(-1),
                                        weights=(w2[:, l, :] * g2[:, None]).reshape(-1), minlength=T))
    return out


def heads_rss(pos, tables, weights, grid, spec, grads):
    """The paper's four GELU heads."""
    xt, res, mdz, mw = heads_latent_mag(pos, tables, weights, grid, spec, grads)
    return table_mag(mdz, xt, res, grid.log2_T, grid.L, grid.F), mw


def heads_latent_mag(pos, tables, weights, grid, spec, grads):
    """(xt, res, m(dz) N x LF, packed weight magnitudes) of the paper's four
    GELU heads: the four heads' dz add up before the scatter."""
    res, xt = dec._prepare(pos, grid, False)
    z = hg.encode(xt, tables, res, grid.log2_T)
    mz = encode_mag(xt, tables, res, grid.log2_T)
    heads = hd.unpack(weights, spec)
    fw = [hd.head_forward(z, heads[h]) for h in range(4)]
    raw = {name: fw[h][0] for h, name in enumerate(hd.HEADS)}
    g = {k: np.asarray(v, np.float64) for k, v in grads.items()}
    s = np.exp(np.minimum(raw["scale"], dec.SCALE_CLIP))
    r, _ = dec.normalise_quat(raw["rot"])
    mds, mdq = _cov_backward_mag(s, r, g["cov"])
    mdy = dict(scale=_scale_adjoint_mag(raw["scale"], s, g["scale"], mds),
               rot=_rotation_adjoint_mag(raw["rot"], g["rot"], mdq),
               sh=np.abs(g["sh"]),
               opacity=_sigmoid_adjoint_mag(g["opacity"], raw["opacity"]))
    mdz2 = np.zeros_like(z)
    wr = []
    for h, name in enumerate(hd.HEADS):
        macts, _ = mlp_forward_mag(mz, heads[h], fw[h][2], hd.gelu_grad, hd.gelu)
        mdz, mdeltas = mlp_backward_mag(mdy[name], heads[h], fw[h][2], hd.gelu_grad)
        mdz2 += mdz * mdz
        wr.append(weight_mag(macts, mdeltas))
    return xt, res, np.sqrt(mdz2), np.concatenate(wr)


def heads_output_mag(pos, tables, weights, grid, spec):
    """Magnitudes of the SH head's outputs (identity activation)."""
    res, xt = dec._prepare(pos, grid, False)
    z = hg.encode(xt, tables, res, grid.log2_T)
    mz = encode_mag(xt, tables, res, grid.log2_T)
    layers = hd.unpack(weights, spec)[2]
    _, _, pres = hd.head_forward(z, layers)
    return mlp_forward_mag(mz, layers, pres, hd.gelu_grad, hd.gelu)[1]


def _hex_forward(inp, planes, weights, hx):
    xt = hp.normalise(inp["mu"], inp["frame"], hx.n_frames)
    z = hp.encode(xt, planes, hx)
    layers = dec.unpack_layers(weights, hx.layer_shapes())
    y, acts, pres = dec.mlp_forward(z, layers)
    # the bilinear terms of the plane samples: magnitude |z| for positive planes
    macts, my = mlp_forward_mag(np.abs(z), layers, pres, _relu_grad, lambda p: np.maximum(p, 0.0))
    return xt, layers, y, pres, macts, my


def hexplane_hidden_mag(inp, planes, weights, hx):
    """Magnitude for h1 = relu(W1 z + b1): that of its pre-activation's terms,
    sqrt(|z|^2 (W1^2)^T + b1^2), on both sides of zero, since
    |relu(a) - relu(b)| <= |a - b| holds where the rounding of W1 z + b1
    carries it across."""
    xt = hp.normalise(inp["mu"], inp["frame"], hx.n_frames)
    z = hp.encode(xt, planes, hx)
    W, b = dec.unpack_layers(weights, hx.layer_shapes())[0]
    return np.sqrt((z * z) @ (W * W).T + b * b)


def _hex_window(xt, hx, gate, n):
    """(w, H(w)) of the energy-flow window, ones without one."""
    if gate is None:
        return np.ones(n), np.ones(n)
    w = hp.energy_window(xt, gate["cr"], gate["tau"])
    return w, hp.displacement_gate(w)


def hexplane_output_mag(inp, planes, weights, hx, gate=None):
    """Magnitudes of mu' = mu + H d_mu and sh' = sh + w d_sh (their terms: the
    canonical value and the gated head output's magnitude)."""
    xt, _, y, _, _, my = _hex_forward(inp, planes, weights, hx)
    w, hg_ = _hex_window(xt, hx, gate, y.shape[0])
    mu = np.asarray(inp["mu"], np.float64)
    sh = np.asarray(inp["sh_can"], np.float64)
    return dict(mu=np.sqrt(mu * mu + (hg_[:, None] * my[:, 0:3]) ** 2),
                sh=np.sqrt(sh * sh + (w[:, None] * my[:, 10:58]) ** 2))


def hexplane_rss(inp, planes, weights, hx, grads, gate=None):
    """The HexPlane deformation network (with the energy-flow window when
    ``gate`` is given); with a window also the N x 2 magnitudes of
    d loss / d(c, r) = (d loss / d w) (dw/dc, dw/dr), where d loss / d w sums
    the products of the w-scaled offsets with their adjoints."""
    xt, layers, y, pres, macts, my = _hex_forward(inp, planes, weights, hx)
    w, hg_ = _hex_window(xt, hx, gate, y.shape[0])
    out, qh = hp._outputs(y, inp, None if gate is None else w)
    g = {k: np.asarray(v, np.float64) for k, v in grads.items()}
    mds, mdq = _cov_backward_mag(out["scale"], out["rot"], g["cov"])
    mdl = out["scale"] * np.sqrt(g["scale"] ** 2 + mds ** 2)       # d loss / d(log s + w d_logs)
    mdy = np.zeros_like(y)
    mdy[:, 0:3] = hg_[:, None] * np.abs(g["mu"])
    mdy[:, 3:7] = _rotation_adjoint_mag(qh, g["rot"], mdq)
    mdy[:, 7:10] = w[:, None] * mdl
    mdy[:, 10:58] = w[:, None] * np.abs(g["sh"])
    mdz, mdeltas = mlp_backward_mag(mdy, layers, pres, _relu_grad)
    n = hx.n_plane_floats()
    acc = np.zeros(n)
    ch = np.arange(hx.channels)
    for fo, corners in hp._corners(xt, hx):
        g2 = mdz[:, fo:fo + hx.channels] ** 2
        idx = np.concatenate([(flat[:, None] + ch).reshape(-1) for flat, _ in corners])
        val = np.concatenate([((w * w)[:, None] * g2).reshape(-1) for _, w in corners])
        acc += np.bincount(idx, weights=val, minlength=n)
    if gate is None:
        return np.sqrt(acc), weight_mag(macts, mdeltas)
    mdw = np.sqrt(np.sum((mdl * my[:, 7:10]) ** 2, axis=1) + np.sum((g["sh"] * my[:, 10:58]) ** 2, axis=1))
    cr = np.asarray(gate["cr"], np.float64)
    t = xt[:, 3].astype(np.float64)
    tau = float(np.float32(gate["tau"]))
    a = dec.sigmoid((t - (cr[:, 0] - cr[:, 1])) / tau)
    b = dec.sigmoid(((cr[:, 0] + cr[:, 1]) - t) / tau)
    mgc = np.stack([mdw * a * b * np.sqrt(a * a + b * b) / tau, mdw * a * b * np.sqrt(4 + a * a + b * b) / tau], 1)
    return np.sqrt(acc), weight_mag(macts, mdeltas), mgc


def gate_rss(pos, tables, weights, grid, mlp, grads, gate_cr):
    """N x 2 magnitudes of the gate-parameter gradient g_o sigma(o^) (dw/dc, dw/dr):
    dw/dc = a b (a - b)/tau and dw/dr = a b (2 - a - b)/tau cancel near the
    window centre and deep inside it; their terms give a b sqrt(a^2 + b^2)/tau
    and a b sqrt(4 + a^2 + b^2)/tau."""
    res, xt = dec._prepare(pos, grid, False)
    z = hg.encode(xt, tables, res, grid.log2_T)
    y, _, _ = dec.mlp_forward(z, dec.unpack_layers(weights, mlp.layer_shapes()))
    t = xt[:, 3].astype(np.float64)
    cr = np.asarray(gate_cr, np.float64)
    tau = float(np.float32(mlp.tau))
    a = dec.sigmoid((t - (cr[:, 0] - cr[:, 1])) / tau)
    b = dec.sigmoid(((cr[:, 0] + cr[:, 1]) - t) / tau)
    gw = np.abs(np.asarray(grads["opacity"], np.float64)[:, 0] * dec.sigmoid(y[:, 10]))
    return np.stack([gw * a * b * np.sqrt(a * a + b * b) / tau, gw * a * b * np.sqrt(4 + a * a + b * b) / tau], axis=1)
