"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, computes the same host-side grid constants as the
oracle, rejects bad arguments before any launch, and honours the host
fault-injection hook."""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spin4d.h")
PROBE_HEADER = os.path.join(ROOT, "include", "spin4d_probe.h")


@pytest.fixture(scope="module")
def sp():
    from spatiotemporal_neural_field_b200 import build
    build.build()
    from spatiotemporal_neural_field_b200 import spin4d
    return spin4d


def declared_functions(header=HEADER):
    src = open(header).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(spin4d_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(sp):
    names = declared_functions()
    assert len(names) >= 17
    for n in names:
        assert hasattr(sp.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", sp._LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (spin4d_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(sp.EXPORTED) == set(names)
    assert not any("probe" in n or "selftest" in n for n in exported), "measurement tools in the decoder library"


def test_probe_library_exports_its_header(sp):
    """The measurement probes and the self-test live in their own library."""
    from spatiotemporal_neural_field_b200 import probe as pr
    names = declared_functions(PROBE_HEADER)
    assert len(names) == 7
    out = subprocess.run(["nm", "-D", "--defined-only", pr._LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (spin4d_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(pr.EXPORTED) == set(names)


def test_grid_init_matches_oracle_resolutions(sp):
    from oracle import hashgrid as hg
    from spatiotemporal_neural_field_b200 import synthetic as S
    for spec in (S.GRID_TINY, S.GRID_SPORTS, S.GRID_STRESS):
        g = sp.grid_from_spec(spec)
        want = hg.grid_resolutions(spec.L, spec.nmin_s, spec.nmax_s, spec.nmin_t, spec.nmax_t)
        assert np.array_equal(np.array(g.resolutions()), want)
        assert g.L == spec.L and g.F == spec.F and g.log2_T == spec.log2_T


def test_param_counts(sp):
    from spatiotemporal_neural_field_b200 import synthetic as S
    for spec in (S.MLP_TINY, S.MLP_SPORTS, S.MLP_STRESS):
        assert sp.mlp_param_count(sp.mlp_from_spec(spec)) == spec.n_params()
        assert S.mlp_weights(spec).size == spec.n_params()
    h = sp.hex_from_spec(S.HEX)
    assert sp.hexplane_plane_count(h) == S.HEX.n_plane_floats()
    assert sp.hexplane_param_count(h) == S.HEX.n_params()


FAKE = 1 << 20      # 16-byte aligned, never dereferenced: every call below returns before a launch


def _outs(sp):
    return sp.Outputs(FAKE, FAKE, FAKE, FAKE, FAKE, None)


def test_invalid_arguments_rejected_on_host(sp):
    from spatiotemporal_neural_field_b200 import synthetic as S
    lib = sp.lib
    g = sp.grid_from_spec(S.GRID_SPORTS)
    m = sp.mlp_from_spec(S.MLP_SPORTS)
    ref = ctypes.byref
    # negative N, null and misaligned pointers
    assert lib.spin4d_decode_fwd(ref(g), ref(m), FAKE, -1, FAKE, FAKE, None, _outs(sp), None) == sp.ERR_INVALID
    assert lib.spin4d_decode_fwd(ref(g), ref(m), None, 10, FAKE, FAKE, None, _outs(sp), None) == sp.ERR_INVALID
    assert lib.spin4d_decode_fwd(ref(g), ref(m), FAKE + 4, 10, FAKE, FAKE, None, _outs(sp), None) == sp.ERR_INVALID
    assert lib.spin4d_encode_fwd(ref(g), FAKE, 10, FAKE + 2, FAKE, None) == sp.ERR_INVALID
    # N == 0 is a valid no-op
    assert lib.spin4d_decode_fwd(ref(g), ref(m), None, 0, None, None, None, sp.Outputs(), None) == sp.OK
    assert lib.spin4d_encode_fwd(ref(g), None, 0, None, None, None) == sp.OK
    # descriptor errors
    bad = sp.grid_from_spec(S.GRID_SPORTS)
    bad.F = 3
    assert lib.spin4d_encode_fwd(ref(bad), FAKE, 10, FAKE, FAKE, None) == sp.ERR_INVALID
    bad = sp.grid_from_spec(S.GRID_SPORTS)
    bad.res[2][1] = 1
    assert lib.spin4d_encode_fwd(ref(bad), FAKE, 10, FAKE, FAKE, None) == sp.ERR_INVALID
    bad = sp.grid_from_spec(S.GRID_SPORTS)
    bad.t_max = bad.t_min
    assert lib.spin4d_encode_fwd(ref(bad), FAKE, 10, FAKE, FAKE, None) == sp.ERR_INVALID
    m2 = sp.mlp_from_spec(S.MLP_SPORTS)
    m2.in_dim = 31                         # must equal L*F
    assert lib.spin4d_decode_fwd(ref(g), ref(m2), FAKE, 10, FAKE, FAKE, None, _outs(sp), None) == sp.ERR_INVALID
    m3 = sp.mlp_desc(32, 64, 2, "f16", gate=True, tau=0.02)
    assert lib.spin4d_decode_fwd(ref(g), ref(m3), FAKE, 10, FAKE, FAKE, None, _outs(sp), None) == sp.ERR_INVALID
    m4 = sp.mlp_desc(32, 64, 2, "f16", gate=True, tau=0.0)
    assert lib.spin4d_decode_fwd(ref(g), ref(m4), FAKE, 10, FAKE, FAKE, FAKE, _outs(sp), None) == sp.ERR_INVALID
    # bwd: too small a workspace
    go = sp.OutputGrads()
    assert lib.spin4d_decode_bwd(ref(g), ref(m), FAKE, 1000, FAKE, FAKE, None, None, ref(go), FAKE, FAKE, FAKE, 16,
                                 None) == sp.ERR_INVALID
    # misaligned saved latent
    assert lib.spin4d_decode_fwd(ref(g), ref(m), FAKE, 10, FAKE, FAKE, None,
                                 sp.Outputs(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4), None) == sp.ERR_INVALID
    # extra gradients: the struct must be given, members aligned, the gate gradient only for a gated decoder
    assert lib.spin4d_decode_bwd_ext(ref(g), ref(m), FAKE, 10, FAKE, FAKE, None, None, ref(go), FAKE, FAKE, None,
                                     FAKE, 1 << 30, None) == sp.ERR_INVALID
    ex = sp.ExtraGrads(FAKE + 2, None)
    assert lib.spin4d_decode_bwd_ext(ref(g), ref(m), FAKE, 10, FAKE, FAKE, None, None, ref(go), FAKE, FAKE, ref(ex),
                                     FAKE, 1 << 30, None) == sp.ERR_INVALID
    ex = sp.ExtraGrads(None, FAKE)
    assert lib.spin4d_decode_bwd_ext(ref(g), ref(m), FAKE, 10, FAKE, FAKE, None, None, ref(go), FAKE, FAKE, ref(ex),
                                     FAKE, 1 << 30, None) == sp.ERR_INVALID
    # ordering
    assert lib.spin4d_morton_order_workspace(0) == 0
    assert lib.spin4d_morton_order_workspace(1000) > 0
    assert lib.spin4d_morton_order(ref(g), FAKE, 10, FAKE, FAKE, FAKE, 16, None) == sp.ERR_INVALID   # workspace
    assert lib.spin4d_morton_order(ref(g), FAKE + 8, 10, FAKE, FAKE, FAKE, 1 << 30, None) == sp.ERR_INVALID
    assert lib.spin4d_morton_order(ref(g), FAKE, -1, FAKE, FAKE, FAKE, 1 << 30, None) == sp.ERR_INVALID
    assert lib.spin4d_morton_order(ref(g), None, 0, None, None, None, 0, None) == sp.OK
    assert lib.spin4d_permute_rows(FAKE, 10, FAKE, FAKE, 10, 6, None) == sp.ERR_INVALID       # row bytes
    assert lib.spin4d_permute_rows(FAKE, 10, FAKE, FAKE, 10, 8, None) == sp.ERR_INVALID       # src == dst
    assert lib.spin4d_permute_rows(None, 0, None, None, 0, 8, None) == sp.OK
    # the paper's decoder
    hs = sp.heads_desc(64)
    assert sp.heads_param_count(hs) == S.HEADS_PAPER.n_params()
    gp4 = sp.grid_from_spec(S.GRID_PAPER)
    assert lib.spin4d_heads_fwd(ref(gp4), ref(sp.heads_desc(63)), FAKE, 10, FAKE, FAKE,
                                sp.HeadsOutputs(FAKE, FAKE, FAKE, FAKE, FAKE, None), None, 0, None) == sp.ERR_INVALID
    assert lib.spin4d_heads_fwd(ref(gp4), ref(sp.heads_desc(64, hidden=128)), FAKE, 10, FAKE, FAKE,
                                sp.HeadsOutputs(FAKE, FAKE, FAKE, FAKE, FAKE, None), None, 0, None) == sp.ERR_UNSUPPORTED
    assert lib.spin4d_heads_fwd(ref(gp4), ref(hs), FAKE, 10, FAKE, FAKE,
                                sp.HeadsOutputs(FAKE, FAKE + 4, FAKE, FAKE, FAKE, None), None, 0, None) == sp.ERR_INVALID
    # the backward's workspace covers the tensor-core kernel's padded slot (12480 floats per head,
    # one CTA) even where the SIMT kernel's packed slots are smaller
    assert lib.spin4d_heads_bwd_workspace(ref(gp4), ref(hs), 1) >= 4 * 12480 * 4
    assert lib.spin4d_heads_bwd_workspace(ref(gp4), ref(hs), 0) == 0
    # the split forward's workspace: 64 fp16 per position; misaligned or short is rejected
    assert lib.spin4d_heads_fwd_workspace(ref(gp4), ref(hs), 10) == 10 * 128
    # only the tensor-core configuration (fp16 weights, hidden 64, 48 SH rows) asks for one
    assert lib.spin4d_heads_fwd_workspace(ref(gp4), ref(sp.heads_desc(64, sh_dim=32)), 10) == 0
    assert lib.spin4d_heads_fwd_workspace(ref(gp4), ref(sp.heads_desc(64, hidden=32)), 10) == 0
    assert lib.spin4d_heads_fwd_workspace(ref(gp4), ref(sp.heads_desc(64, w_dtype="f32")), 10) == 0
    assert lib.spin4d_heads_fwd(ref(gp4), ref(hs), FAKE, 10, FAKE, FAKE,
                                sp.HeadsOutputs(FAKE, FAKE, FAKE, FAKE, FAKE, None), FAKE, 10 * 128 - 1,
                                None) == sp.ERR_INVALID
    assert lib.spin4d_heads_fwd(ref(gp4), ref(hs), FAKE, 10, FAKE, FAKE,
                                sp.HeadsOutputs(FAKE, FAKE, FAKE, FAKE, FAKE, None), FAKE + 16, 10 * 128,
                                None) == sp.ERR_INVALID
    assert lib.spin4d_heads_fwd(ref(gp4), ref(sp.heads_desc(64, hidden=62)), FAKE, 10, FAKE, FAKE,
                                sp.HeadsOutputs(FAKE, FAKE, FAKE, FAKE, FAKE, None), None, 0, None) == sp.ERR_UNSUPPORTED
    # grouped Adam: ends must increase to n
    grp = (sp.AdamGroup * 2)(sp.AdamGroup(60, 1e-3), sp.AdamGroup(50, 1e-4))
    assert lib.spin4d_adam_step_groups(FAKE, None, FAKE, FAKE, FAKE, 100, grp, 2, 1, 0.9, 0.99, 1e-15, 0, None,
                                       None) == sp.ERR_INVALID
    grp = (sp.AdamGroup * 2)(sp.AdamGroup(60, 1e-3), sp.AdamGroup(90, 1e-4))
    assert lib.spin4d_adam_step_groups(FAKE, None, FAKE, FAKE, FAKE, 100, grp, 2, 1, 0.9, 0.99, 1e-15, 0, None,
                                       None) == sp.ERR_INVALID
    # adam
    assert lib.spin4d_adam_step(FAKE, None, FAKE, FAKE, FAKE, 100, 0, 1e-3, 0.9, 0.99, 1e-15, 0, None,
                                None) == sp.ERR_INVALID
    assert lib.spin4d_adam_step(FAKE, None, FAKE, FAKE, FAKE, 100, 1, 1e-3, 1.0, 0.99, 1e-15, 0, None,
                                None) == sp.ERR_INVALID
    assert lib.spin4d_grid_init(None, 4, 2, 12, 0, 4, 32, 4, 32, 0.0, 1.0) == sp.ERR_INVALID
    assert sp.lib.spin4d_status_string(sp.ERR_INVALID) == b"invalid argument"


def test_unsupported_hexplane_shape(sp):
    lib = sp.lib
    h = sp.hex_desc(channels=16)
    inp = [FAKE] * 2
    assert lib.spin4d_hexplane_fwd(ctypes.byref(h), FAKE, FAKE, 10, FAKE, FAKE, FAKE, FAKE, FAKE,
                                   sp.HexOutputs(FAKE, FAKE, FAKE, FAKE, FAKE, None), None) == sp.ERR_UNSUPPORTED
    # supported shape, misaligned saved latent for the backward
    h = sp.hex_desc()
    go = sp.HexOutputGrads()
    assert lib.spin4d_hexplane_bwd(ctypes.byref(h), FAKE, FAKE, 10, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4,
                                   ctypes.byref(go), FAKE, FAKE, FAKE, 1 << 40, None) == sp.ERR_INVALID
    # the saved activations: none, no latent, a misaligned h1
    def saved(x):
        return lib.spin4d_hexplane_bwd_saved(ctypes.byref(h), FAKE, FAKE, 10, FAKE, FAKE, FAKE, FAKE, x, None,
                                             ctypes.byref(go), FAKE, FAKE, FAKE, 1 << 40, None)
    assert saved(None) == sp.ERR_INVALID
    assert saved(ctypes.byref(sp.HexSaved(None, FAKE))) == sp.ERR_INVALID
    assert saved(ctypes.byref(sp.HexSaved(FAKE, FAKE + 4))) == sp.ERR_INVALID
    # misaligned SH rows in the forward (canonical or output)
    assert lib.spin4d_hexplane_fwd(ctypes.byref(h), FAKE, FAKE, 10, FAKE, FAKE, FAKE, FAKE, FAKE + 4,
                                   sp.HexOutputs(FAKE, FAKE, FAKE, FAKE, FAKE, None, None), None) == sp.ERR_INVALID
    assert lib.spin4d_hexplane_fwd(ctypes.byref(h), FAKE, FAKE, 10, FAKE, FAKE, FAKE, FAKE, FAKE,
                                   sp.HexOutputs(FAKE, FAKE, FAKE, FAKE + 4, FAKE, None, None), None) == sp.ERR_INVALID
    # a misaligned saved h1 in the forward
    assert lib.spin4d_hexplane_fwd(ctypes.byref(h), FAKE, FAKE, 10, FAKE, FAKE, FAKE, FAKE, FAKE,
                                   sp.HexOutputs(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE + 4), None) == sp.ERR_INVALID


def test_fault_injection_hook_in_subprocess(sp):
    code = r"""
import ctypes, sys
sys.path.insert(0, %r)
from spatiotemporal_neural_field_b200 import spin4d as sp, synthetic as S
g = sp.grid_from_spec(S.GRID_SPORTS); m = sp.mlp_from_spec(S.MLP_SPORTS)
F = 1 << 20
r1 = sp.lib.spin4d_decode_fwd(ctypes.byref(g), ctypes.byref(m), F, 10, F, F, None, sp.Outputs(F, F, F, F, F, None), None)
r2 = sp.lib.spin4d_encode_fwd(ctypes.byref(g), F, -1, F, F, None)
print(r1, r2)
""" % ROOT
    env = dict(os.environ, SPIN4D_FAULT="spin4d_decode_fwd")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr
    r1, r2 = map(int, out.stdout.split())
    assert r1 == -5          # injected after validation, before any launch
    assert r2 == -1          # other entry points unaffected (still validated)


def test_learning_rate_schedule_matches_oracle(sp):
    from oracle import heads as hd
    for args in ((8e-3, 1e-7, 100, 1100), (1e-3, 1e-7, 0, 40000), (3e-5, 1e-7, 500, 500)):
        for step in (1, 2, 50, 99, 100, 101, 600, 1099, 1100, 1101, 40000, 50000):
            assert abs(sp.lr_warmup_cosine(step, *args) - hd.lr_warmup_cosine(step, *args)) <= 1e-12 * args[0]


def test_render_arguments_rejected_on_host(sp):
    """Every argument of the renderer is checked before a launch."""
    from spatiotemporal_neural_field_b200 import synthetic as S
    lib, ref = sp.lib, ctypes.byref
    cam = sp.camera_from_spec(S.orbit_camera(64, 48))
    desc = sp.render_desc(sh_degree=3)
    need = lib.spin4d_render_state_bytes(100, 64, 48, 4096)
    assert need > 0
    assert lib.spin4d_render_state_bytes(100, 0, 48, 4096) == 0
    assert lib.spin4d_render_state_bytes(-1, 64, 48, 4096) == 0
    assert lib.spin4d_render_state_bytes(100, 64, 48, -5) == 0

    def fwd(c=cam, d=desc, n=100, state=FAKE, nbytes=need, cap=4096, image=FAKE):
        return lib.spin4d_render_fwd(ref(c), ref(d), n, FAKE, FAKE, FAKE, FAKE, image, None, state, nbytes, cap,
                                     None)

    def bad_cam(**kw):
        c = sp.camera_from_spec(S.orbit_camera(64, 48))
        for k, v in kw.items():
            setattr(c, k, v)
        return c

    def bad_desc(**kw):
        d = sp.render_desc(sh_degree=3)
        for k, v in kw.items():
            setattr(d, k, v)
        return d

    assert fwd(c=bad_cam(width=0)) == sp.ERR_INVALID
    assert fwd(c=bad_cam(fx=0.0)) == sp.ERR_INVALID
    assert fwd(c=bad_cam(z_near=0.0)) == sp.ERR_INVALID
    assert fwd(d=bad_desc(sh_degree=4)) == sp.ERR_INVALID
    assert fwd(d=bad_desc(alpha_max=1.0)) == sp.ERR_INVALID
    assert fwd(d=bad_desc(alpha_min=0.99)) == sp.ERR_INVALID      # not below alpha_max
    assert fwd(d=bad_desc(t_stop=1.0)) == sp.ERR_INVALID
    assert fwd(d=bad_desc(lowpass=-1.0)) == sp.ERR_INVALID
    assert fwd(d=bad_desc(mean_stride=5)) == sp.ERR_INVALID
    assert fwd(d=bad_desc(reserved=1)) == sp.ERR_INVALID
    assert fwd(n=-1) == sp.ERR_INVALID
    assert fwd(nbytes=need - 1) == sp.ERR_INVALID                  # state too small
    assert fwd(state=FAKE + 16) == sp.ERR_INVALID                  # state not 256-byte aligned
    assert fwd(image=None) == sp.ERR_INVALID
    assert lib.spin4d_render_bwd(ref(cam), ref(desc), 100, FAKE, FAKE, FAKE, FAKE, None, FAKE, need, 4096,
                                 None, None, None, None, None) == sp.ERR_INVALID   # no upstream gradient


def test_l2_window_arguments_rejected_on_host(sp):
    """The opt-in L2 window refuses the legacy stream, a NULL base and an
    empty range before touching the device."""
    applied = ctypes.c_size_t(0)
    assert sp.lib.spin4d_l2_window_set(None, 1 << 20, 1 << 20, ctypes.byref(applied)) == sp.ERR_INVALID
    assert sp.lib.spin4d_l2_window_set(1, None, 1 << 20, ctypes.byref(applied)) == sp.ERR_INVALID
    assert sp.lib.spin4d_l2_window_set(1, 1 << 20, 0, ctypes.byref(applied)) == sp.ERR_INVALID
    assert sp.lib.spin4d_l2_window_clear(None) == sp.ERR_INVALID


def test_hexplane_empty_batch_is_a_no_op(sp):
    """N = 0 returns success before any pointer is looked at or any launch,
    for the forward and every backward entry point."""
    lib = sp.lib
    h = sp.hex_desc()
    go = sp.HexOutputGrads()
    out = sp.HexOutputs(None, None, None, None, None, None, None)
    assert lib.spin4d_hexplane_fwd(ctypes.byref(h), None, None, 0, None, None, None, None, None, out, None) == 0
    assert lib.spin4d_hexplane_bwd(ctypes.byref(h), None, None, 0, None, None, None, None, None, None,
                                   ctypes.byref(go), None, None, None, 0, None) == 0
    saved = sp.HexSaved(FAKE, FAKE)
    assert lib.spin4d_hexplane_bwd_saved(ctypes.byref(h), None, None, 0, None, None, None, None, ctypes.byref(saved),
                                         None, ctypes.byref(go), None, None, None, 0, None) == 0
    assert lib.spin4d_hexplane_bwd_workspace(ctypes.byref(h), 0) == 0
