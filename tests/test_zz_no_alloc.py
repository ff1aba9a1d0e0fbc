"""The allocation-free backward entry point (B200 only).

spin4d_decode_bwd_noalloc serves callers that cannot allocate device memory:
it runs the same backward pass as spin4d_decode_bwd but takes its scratch
from an array built into the library instead of a caller workspace.  This
file is collected last so that a run stopping at the first failure has run
every other test before it; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

from spatiotemporal_neural_field_b200 import synthetic as S
from tests import tol

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

# Only the fp32 atomic accumulation order can differ between the two entry
# points (same kernels, same inputs): the GPU-vs-GPU bound the other tests use.
CONSISTENCY_RTOL = 1e-4


@pytest.fixture(scope="module")
def sp():
    from spatiotemporal_neural_field_b200 import spin4d
    return spin4d


def _case(name, n):
    w = S.WORKLOADS[name]
    grid, mlp = w["grid"], w["mlp"]
    if name == "tiny_fp32":
        pos = S.uniform_positions(n)
    else:
        frame = S.sports_scene(300_000).frame(75)
        pos = frame[np.random.default_rng(5).choice(len(frame), n, replace=False)]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    grads = S.upstream_grads(n, S.DECODE_OUT_WIDTHS, 1e-2 if grid.dtype == "f16" else 1.0)
    return (grid, mlp, dev(pos), dev(S.hash_tables(grid, scale=1.0)), dev(S.mlp_weights(mlp, bias_scale=0.5)),
            {k: dev(v) for k, v in grads.items()})


@pytest.mark.parametrize("name,n", [("sports_frame_fp16", 50_021), ("tiny_fp32", 4099)])
def test_noalloc_backward_matches_workspace_backward_twice(sp, name, n):
    grid, mlp, P, T, W, G = _case(name, n)
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    shape = (grid.L, 1 << grid.log2_T, grid.F)
    ref_t = torch.zeros(shape, dtype=torch.float32, device="cuda")
    ref_w = torch.zeros(mlp.n_params(), dtype=torch.float32, device="cuda")
    sp.decode_bwd(g, m, P, T, W, G, ref_t, ref_w)
    for _ in range(2):   # two calls in a row: the shared scratch must not carry state
        gt = torch.zeros(shape, dtype=torch.float32, device="cuda")
        gw = torch.zeros(mlp.n_params(), dtype=torch.float32, device="cuda")
        sp.decode_bwd_noalloc(g, m, P, T, W, G, gt, gw)
        torch.cuda.synchronize()
        tol.normwise(gt.cpu().numpy(), ref_t.cpu().numpy(), CONSISTENCY_RTOL, "grad_tables")
        tol.normwise(gw.cpu().numpy(), ref_w.cpu().numpy(), CONSISTENCY_RTOL, "grad_weights")


def test_noalloc_rejects_scratch_beyond_its_size(sp):
    """A shape whose weight-gradient scratch exceeds the built-in array is
    refused before any launch.  Every data pointer is NULL: should the size
    check ever let the call through, the backward's own argument checks
    refuse it before launching anything."""
    g = sp.grid_desc(8, 8, 12, "f32", 4, 32, 4, 32, 0.0, 1.0)          # latent width 64
    m = sp.mlp_desc(64, 128, 4, "f32")                                 # ~58k weights
    need = sp.decode_bwd_workspace(g, m, 1_000_000)
    assert sp.NOALLOC_SCRATCH_BYTES == sp.lib.spin4d_decode_bwd_noalloc_scratch_bytes()
    assert need > sp.NOALLOC_SCRATCH_BYTES
    st = sp.lib.spin4d_decode_bwd_noalloc(ctypes.byref(g), ctypes.byref(m), None, 1_000_000, None, None, None, None,
                                          ctypes.byref(sp.OutputGrads()), None, None, None)
    assert st == sp.ERR_INVALID
