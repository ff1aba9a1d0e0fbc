"""GPU parity of the paper's four-head GELU decoder and the grouped Adam
against the oracle (B200 only)."""
import dataclasses

import numpy as np
import pytest

from oracle import decoder as dec
from oracle import hashgrid
from oracle import heads as hd
from spatiotemporal_neural_field_b200 import synthetic as S
from tests import magnitude as mag
from tests import tol
from tests.test_parity_decode import check_fp32_outputs

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
    keys = ("scale", "rot", "sh", "opacity", "cov")
    if grid.dtype == "f32":
        check_fp32_outputs({k: host(out[k]) for k in keys}, want, keys,
                           extra_mag=dict(sh=mag.heads_output_mag(pos, tables, weights, grid, spec)))
    else:
        for k in keys:
            tol.absolute(host(out[k]), want[k], tol.FP16_ATOL, k)
    res, xt = dec._prepare(pos, grid, False)
    z_rho = mag.encode_mag(xt, tables, res, grid.log2_T)
    tol.elementwise(host(out["latent"]), want["z"], tol.FP32_RTOL, "latent", tol.column_groups(grid.L * grid.F),
                    rho=z_rho)
    # the raw head outputs the forward saves for the backward: Eq. 11 inverts them
    raw = host(sp.heads_fwd(g, h, dev(pos), dev(tables), dev(weights), raw=True)["raw"]).astype(np.float64)
    tol.absolute(np.exp(np.minimum(raw[:, :3], 20.0)), want["scale"], tol.FP16_ATOL, "raw scale")
    tol.absolute(raw[:, 3:7] / np.linalg.norm(raw[:, 3:7], axis=1, keepdims=True), want["rot"], tol.FP16_ATOL,
                 "raw rotation")
    tol.absolute(1.0 / (1.0 + np.exp(-raw[:, 7])), want["opacity"][:, 0], tol.FP16_ATOL, "raw opacity")
    if grid.dtype != "f32":
        # without a workspace the tensor-core configuration runs as one fused kernel
        fused = sp.heads_fwd(g, h, dev(pos), dev(tables), dev(weights), latent=True, workspace=None)
        for k in ("scale", "rot", "sh", "opacity", "cov"):
            tol.absolute(host(fused[k]), want[k], tol.FP16_ATOL, "fused " + k)
        tol.elementwise(host(fused["latent"]), want["z"], tol.FP32_RTOL, "fused latent",
                        tol.column_groups(grid.L * grid.F), rho=z_rho)


@pytest.mark.parametrize("case,saved", [("tiny_fp32", ""), ("tiny_fp32", "latent+raw"), ("paper_fp16", ""),
                                        ("paper_fp16", "latent"), ("paper_fp16", "raw"), ("paper_fp16", "latent+raw"),
                                        ("paper_fp16_init", ""), ("paper_fp16_init", "latent+raw")])
def test_heads_backward_matches_oracle(sp, case, saved):
    """With the forward's z and / or raw head outputs the backward skips the
    gather and / or the first recompute of the scale, rotation and opacity
    heads; the gradients are the same.  With both, the paper's configuration
    runs the tensor-core backward."""
    grid, spec, pos, tables, weights, grads = _setup(case)
    g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec)
    P, T, W = dev(pos), dev(tables), dev(weights)
    fw = sp.heads_fwd(g, h, P, T, W, latent=True, raw=True)
    lat = fw["latent"] if "latent" in saved else None
    raw = fw["raw"] if "raw" in saved else None
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda")
    gw = torch.zeros(spec.n_params(), device="cuda")
    sp.heads_bwd(g, h, P, T, W, {k: dev(v) for k, v in grads.items()}, gt, gw, latent=lat, raw=raw)
    wt, ww = hd.decode_backward(pos, tables, weights, grid, spec, grads)
    rtol = tol.FP32_GRAD_RTOL if grid.dtype == "f32" else tol.FP16_GRAD_RTOL
    check_heads_grads(host(gt), host(gw), wt, ww, grid, spec, rtol,
                      mag.heads_rss(pos, tables, weights, grid, spec, grads))


def check_heads_grads(gt, gw, wt, ww, grid, spec, rtol, rho=(None, None), tag=""):
    """Element-wise per table level and per weight block of each head."""
    tol.elementwise(gt, wt, rtol, tag + "grad_tables", tol.table_levels(grid.L, 1 << grid.log2_T, grid.F),
                    rho=rho[0])
    blocks, o = [], 0
    for head in range(4):
        hb = tol.weight_blocks(spec.layer_shapes(head), "head %d " % head, o)
        blocks += hb
        o = hb[-1][1].stop
    assert o == spec.n_params()
    tol.elementwise(gw, ww, rtol, tag + "grad_weights", blocks, rho=rho[1])


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


def test_heads_edge_sizes(sp):
    """N = 0 launches nothing; N = 1, 33 and 129 (one block and one more
    position; one tensor-core tile and one more) match the oracle, with the
    SIMT backward and with the tensor-core one (saved z and raw outputs);
    the backward accumulates."""
    grid, spec = S.GRID_PAPER, S.HEADS_PAPER
    g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec)
    tables = S.hash_tables(grid, seed=8, scale=1.0)
    weights = S.heads_weights(spec, seed=9, bias_scale=0.3)
    T, W = dev(tables), dev(weights)
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda")
    gw = torch.zeros(spec.n_params(), device="cuda")
    empty = torch.zeros((0, 4), device="cuda")
    out = sp.heads_fwd(g, h, empty, T, W)
    assert all(v.numel() == 0 for v in out.values())
    widths = dict(S.HEADS_OUT_WIDTHS, sh=spec.sh_dim)
    sp.heads_bwd(g, h, empty, T, W, {k: torch.zeros((0, w), device="cuda") for k, w in widths.items()}, gt, gw)
    torch.cuda.synchronize()
    assert not gt.any() and not gw.any()
    for n in (1, 33, 129):
        pos = S.sports_scene(300_000).frame(75)[:n]
        grads = S.upstream_grads(n, widths, 1e-2, seed=10 + n)
        P = dev(pos)
        out = sp.heads_fwd(g, h, P, T, W)
        want = hd.decode_forward(pos, tables, weights, grid, spec)
        for k in ("scale", "rot", "sh", "opacity", "cov"):
            tol.absolute(host(out[k]), want[k], tol.FP16_ATOL, "%s (N=%d)" % (k, n))
        gt.zero_()
        gw.zero_()
        G = {k: dev(v) for k, v in grads.items()}
        sp.heads_bwd(g, h, P, T, W, G, gt, gw)
        first = (gt.clone(), gw.clone())
        sp.heads_bwd(g, h, P, T, W, G, gt, gw)
        wt, ww = hd.decode_backward(pos, tables, weights, grid, spec, grads)
        rho = mag.heads_rss(pos, tables, weights, grid, spec, grads)
        check_heads_grads(host(first[0]), host(first[1]), wt, ww, grid, spec, tol.FP16_GRAD_RTOL, rho,
                          "(N=%d) " % n)
        # a second call adds the same gradient again
        tol.normwise(host(gt), 2 * host(first[0]), 1e-5, "accumulated grad_tables (N=%d)" % n)
        tol.normwise(host(gw), 2 * host(first[1]), 1e-5, "accumulated grad_weights (N=%d)" % n)
        saved = sp.heads_fwd(g, h, P, T, W, latent=True, raw=True)
        gt.zero_()
        gw.zero_()
        sp.heads_bwd(g, h, P, T, W, G, gt, gw, latent=saved["latent"], raw=saved["raw"])
        tc_first = (gt.clone(), gw.clone())
        sp.heads_bwd(g, h, P, T, W, G, gt, gw, latent=saved["latent"], raw=saved["raw"])
        check_heads_grads(host(tc_first[0]), host(tc_first[1]), wt, ww, grid, spec, tol.FP16_GRAD_RTOL, rho,
                          "tc (N=%d) " % n)
        tol.normwise(host(gt), 2 * host(tc_first[0]), 1e-5, "tc accumulated grad_tables (N=%d)" % n)
        tol.normwise(host(gw), 2 * host(tc_first[1]), 1e-5, "tc accumulated grad_weights (N=%d)" % n)


def test_heads_full_launch_sampled_and_by_halves(sp):
    """The timed 1M-position launch: forward on 400 sampled positions against
    the oracle; the backward of the whole launch equals that of its two
    halves (linearity; atomics only reorder the fp32 sums)."""
    w = S.WORKLOADS["paper_heads_fp16"]
    grid, spec, n = w["grid"], w["heads"], w["N"]
    g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec)
    pos = S.sports_scene(300_000).frames(range(4))[:n]
    tables = S.hash_tables(grid, seed=11, scale=1.0)
    weights = S.heads_weights(spec, seed=12, bias_scale=0.3)
    P, T, W = dev(pos), dev(tables), dev(weights)
    out = sp.heads_fwd(g, h, P, T, W, latent=True, raw=True)
    idx = np.random.default_rng(13).choice(n, 400, replace=False)
    want = hd.decode_forward(pos[idx], tables, weights, grid, spec)
    for k in ("scale", "rot", "sh", "opacity", "cov"):
        tol.absolute(host(out[k])[idx], want[k], tol.FP16_ATOL, k + " (1M launch, sampled)")
    widths = dict(S.HEADS_OUT_WIDTHS, sh=spec.sh_dim)
    G = {k: torch.randn((n, wd), device="cuda", generator=torch.Generator("cuda").manual_seed(14)) * 1e-2
         for k, wd in widths.items()}
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda")
    gw = torch.zeros(spec.n_params(), device="cuda")
    sp.heads_bwd(g, h, P, T, W, G, gt, gw, latent=out["latent"], raw=out["raw"])
    gt2, gw2 = torch.zeros_like(gt), torch.zeros_like(gw)
    half = n // 2
    for a, b in ((0, half), (half, n)):
        sp.heads_bwd(g, h, P[a:b], T, W, {k: v[a:b] for k, v in G.items()}, gt2, gw2, latent=out["latent"][a:b],
                     raw=out["raw"][a:b])
    torch.cuda.synchronize()
    tol.normwise(host(gt2), host(gt), 1e-4, "grad_tables by halves", tol.table_levels(grid.L, 1 << grid.log2_T, grid.F))
    tol.normwise(host(gw2), host(gw), 1e-4, "grad_weights by halves")


def test_heads_table_size_2_23(sp):
    """SPIN-4DGS section 4, Table 5: T = 2^23 entries per level, the paper's
    best setting (16 x 2^23 x 4 fp16 = 1 GiB of tables, 2 GiB of fp32
    gradients).  Forward on sampled rows of a 200k-position launch; the
    backward of a 3001-position launch, tensor-core and SIMT forms, level by
    level against the oracle's per-level scatter (its whole fp64 gradient
    would be 4 GiB)."""
    grid = dataclasses.replace(S.GRID_PAPER, log2_T=23)
    spec = S.HEADS_PAPER
    g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec)
    tables = S.hash_tables(grid, seed=21, scale=1.0)
    weights = S.heads_weights(spec, seed=22, bias_scale=0.3)
    T, W = dev(tables), dev(weights)
    n = 200_000
    pos = S.sports_scene(300_000).frames(range(4))[:n]
    out = sp.heads_fwd(g, h, dev(pos), T, W, latent=True)
    idx = np.sort(np.random.default_rng(23).choice(n, 500, replace=False))
    want = hd.decode_forward(pos[idx], tables, weights, grid, spec)
    for k in ("scale", "rot", "sh", "opacity", "cov"):
        tol.absolute(host(out[k])[idx], want[k], tol.FP16_ATOL, k + " (T = 2^23, sampled)")
    res, xt = dec._prepare(pos[idx], grid, False)
    tol.elementwise(host(out["latent"])[idx], want["z"], tol.FP32_RTOL, "latent (T = 2^23)",
                    tol.column_groups(grid.L * grid.F), rho=mag.encode_mag(xt, tables, res, grid.log2_T))
    del out
    nb = 3001
    pb = pos[:nb]
    widths = dict(S.HEADS_OUT_WIDTHS, sh=spec.sh_dim)
    grads = S.upstream_grads(nb, widths, 1e-2, seed=24)
    P, G = dev(pb), {k: dev(v) for k, v in grads.items()}
    saved = sp.heads_fwd(g, h, P, T, W, latent=True, raw=True)
    res, xt, dz, ww = hd.latent_backward(pb, tables, weights, grid, spec, grads)
    mxt, mres, mdz, mw = mag.heads_latent_mag(pb, tables, weights, grid, spec, grads)
    for form in ("tensor-core", "SIMT"):
        gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda")
        gw = torch.zeros(spec.n_params(), device="cuda")
        if form == "tensor-core":
            sp.heads_bwd(g, h, P, T, W, G, gt, gw, latent=saved["latent"], raw=saved["raw"])
        else:
            sp.heads_bwd(g, h, P, T, W, G, gt, gw)
        blocks, o = [], 0
        for head in range(4):
            hb = tol.weight_blocks(spec.layer_shapes(head), "head %d " % head, o)
            blocks += hb
            o = hb[-1][1].stop
        tol.elementwise(host(gw), ww, tol.FP16_GRAD_RTOL, form + " grad_weights (T = 2^23)", blocks, rho=mw)
        for l in range(grid.L):
            wl = hashgrid.scatter_table_grad_level(dz, xt, res, grid.log2_T, l, grid.F)
            tol.elementwise(host(gt[l]), wl, tol.FP16_GRAD_RTOL, "%s grad_tables (T = 2^23) level %d" % (form, l),
                            rho=mag.table_mag_level(mdz, mxt, mres, grid.log2_T, l, grid.F))
        del gt, gw
        torch.cuda.empty_cache()
