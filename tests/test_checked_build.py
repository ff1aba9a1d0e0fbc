"""The checked build (libspin4d_checked.so): the same decoder compiled with
device-side bounds checks on every hash-table index and HexPlane cell.

On the CPU: it exports the same entry points and says it is checked.  On a
B200: in-range workloads (decoder forward and backward, the paper's heads,
HexPlane forward and backward) run through it in a child process, match the
oracle, and leave no bounds error behind.  No test drives an index out of
range: the host validation admits no such input, and a test that plants a
mistake plants it in the oracle, on the CPU."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "spatiotemporal_neural_field_b200")


def _exports(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    return set(re.findall(r" T (spin4d_\w+)", out))


def test_checked_library_exports_the_decoder_and_says_so():
    from spatiotemporal_neural_field_b200 import build
    build.build()
    plain, checked = os.path.join(PKG, "libspin4d.so"), os.path.join(PKG, "libspin4d_checked.so")
    assert _exports(plain) == _exports(checked)
    assert ctypes.CDLL(checked).spin4d_checked_build() == 1
    assert ctypes.CDLL(plain).spin4d_checked_build() == 0


CHILD = r"""
import sys
sys.path.insert(0, %r)
import numpy as np
import torch
from oracle import decoder as dec, hexplane as hp, heads as hd
from spatiotemporal_neural_field_b200 import spin4d as sp, synthetic as S
from tests import tol
assert sp.lib.spin4d_checked_build() == 1, sp._LIB_PATH
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
sp.check_device_errors(clear=True)
# the sports decoder, forward and backward (tensor-core kernels)
w = S.WORKLOADS["sports_frame_fp16"]
grid, mlp = w["grid"], w["mlp"]
n = 20011
pos = S.sports_scene(300_000).frame(75)[:n]
tables, weights = S.hash_tables(grid, scale=1.0), S.mlp_weights(mlp, bias_scale=0.5)
g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
out = sp.decode_fwd(g, m, dev(pos), dev(tables), dev(weights))
want = dec.decode_forward(pos, tables, weights, grid, mlp)
for k in ("scale", "rot", "rgb", "opacity", "cov"):
    tol.absolute(out[k].cpu().numpy(), want[k], tol.FP16_ATOL, k)
grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, 1e-2)
gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device="cuda")
gw = torch.zeros(mlp.n_params(), device="cuda")
sp.decode_bwd(g, m, dev(pos), dev(tables), dev(weights), {k: dev(v) for k, v in grads.items()}, gt, gw)
# the stress grid (dense and hashed levels, F = 4) and the encoder alone
ws = S.WORKLOADS["stress_fp16_gate"]
gs = sp.grid_from_spec(ws["grid"])
ps = S.stress_positions(8009)
sp.encode_fwd(gs, dev(ps), dev(S.hash_tables(ws["grid"], scale=1.0)))
# the paper's heads, forward and tensor-core backward
gp, hh = sp.grid_from_spec(S.GRID_PAPER), sp.heads_from_spec(S.HEADS_PAPER)
tp, wp = dev(S.hash_tables(S.GRID_PAPER, scale=1.0)), dev(S.heads_weights(S.HEADS_PAPER, bias_scale=0.3))
P = dev(pos[:3001])
fo = sp.heads_fwd(gp, hh, P, tp, wp, latent=True, raw=True)
hg = {k: torch.randn((3001, wd), device="cuda") * 1e-2 for k, wd in dict(S.HEADS_OUT_WIDTHS, sh=48).items()}
gtp = torch.zeros((16, 1 << 21, 4), device="cuda")
gwp = torch.zeros(S.HEADS_PAPER.n_params(), device="cuda")
sp.heads_bwd(gp, hh, P, tp, wp, hg, gtp, gwp, latent=fo["latent"], raw=fo["raw"])
# HexPlane forward and backward
hx = S.HEX
inp = S.hexplane_inputs(2053)
planes, hw = S.hexplane_planes(hx), S.hexplane_weights(hx, bias_scale=0.5)
h = sp.hex_from_spec(hx)
I = {k: dev(v) for k, v in inp.items()}
ho = sp.hexplane_fwd(h, I, dev(planes), dev(hw))
hwant = hp.forward(inp, planes, hw, hx)
tol.elementwise(ho["sh"].cpu().numpy(), hwant["sh"], 1e-4, "hexplane sh")
hgr = S.upstream_grads(2053, S.HEX_OUT_WIDTHS, 1.0)
gpl = torch.zeros(hx.n_plane_floats(), device="cuda")
gwh = torch.zeros(hx.n_params(), device="cuda")
sp.hexplane_bwd(h, I, dev(planes), dev(hw), {k: dev(v) for k, v in hgr.items()}, gpl, gwh)
torch.cuda.synchronize()
sp.check_device_errors(clear=False)     # raises on a failed bounds check or a timed-out wait
print("CHECKED_OK", sp.lib.spin4d_checked_build())
""" % ROOT


@pytest.mark.gpu
def test_checked_build_runs_in_range_workloads_clean():
    env = dict(os.environ, SPIN4D_CHECKED="1")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, cwd=ROOT, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert "CHECKED_OK 1" in r.stdout
