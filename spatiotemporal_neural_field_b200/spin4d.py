"""Thin ctypes binding of ``libspin4d.so`` (declared in ``include/spin4d.h``).

Argument marshalling only: every step of the decoder runs in the library's
CUDA kernels.  torch is used for device memory and the current stream.  If
the library is missing the import fails loudly; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

# SPIN4D_CHECKED=1 selects the build with device-side bounds checks
_LIB_NAME = "libspin4d_checked.so" if os.environ.get("SPIN4D_CHECKED") == "1" else "libspin4d.so"
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), _LIB_NAME)
if not os.path.exists(_LIB_PATH):
    raise ImportError("%s is not built (run `python -m spatiotemporal_neural_field_b200.build` "
                      "or __graft_entry__.build()); spin4d has no CPU fallback" % _LIB_NAME)
lib = ctypes.CDLL(_LIB_PATH)

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_NONFINITE, ERR_INJECTED, ERR_TIMEOUT, ERR_BOUNDS = (
    0, -1, -2, -3, -4, -5, -6, -7)
F32, F16 = 0, 1
INPUT_NORMALISED = 1
MAX_LEVELS = 16
HEAD_ROWS = 11

c_i32, c_i64, c_f32, c_u32, c_vp, c_sz = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_uint32,
                                          ctypes.c_void_p, ctypes.c_size_t)


class GridDesc(ctypes.Structure):
    _fields_ = [("L", c_i32), ("F", c_i32), ("log2_T", c_i32), ("table_dtype", c_i32),
                ("res", (c_i32 * 4) * MAX_LEVELS), ("t_min", c_f32), ("t_max", c_f32),
                ("flags", c_u32), ("reserved", c_i32)]

    def resolutions(self):
        return [[self.res[l][d] for d in range(4)] for l in range(self.L)]


class MlpDesc(ctypes.Structure):
    _fields_ = [("in_dim", c_i32), ("hidden", c_i32), ("n_hidden", c_i32), ("w_dtype", c_i32),
                ("gate", c_i32), ("tau", c_f32)]


class Outputs(ctypes.Structure):
    _fields_ = [("scale", c_vp), ("rot", c_vp), ("rgb", c_vp), ("opacity", c_vp), ("cov", c_vp),
                ("latent", c_vp)]


class OutputGrads(ctypes.Structure):
    _fields_ = [("scale", c_vp), ("rot", c_vp), ("rgb", c_vp), ("opacity", c_vp), ("cov", c_vp)]


class ExtraGrads(ctypes.Structure):
    _fields_ = [("pos", c_vp), ("gate_cr", c_vp)]


class HexDesc(ctypes.Structure):
    _fields_ = [("n_scales", c_i32), ("scales", c_i32 * 4), ("time_res", c_i32), ("channels", c_i32),
                ("n_frames", c_i32), ("hidden", c_i32), ("n_hidden", c_i32)]


class HexOutputs(ctypes.Structure):
    _fields_ = [("mu", c_vp), ("rot", c_vp), ("scale", c_vp), ("sh", c_vp), ("cov", c_vp), ("latent", c_vp),
                ("hidden", c_vp)]


class HexSaved(ctypes.Structure):
    _fields_ = [("latent", c_vp), ("hidden", c_vp)]


class HexOutputGrads(ctypes.Structure):
    _fields_ = [("mu", c_vp), ("rot", c_vp), ("scale", c_vp), ("sh", c_vp), ("cov", c_vp)]


class HexGate(ctypes.Structure):
    _fields_ = [("cr", c_vp), ("tau", c_f32), ("grad_cr", c_vp)]


class HeadsDesc(ctypes.Structure):
    _fields_ = [("in_dim", c_i32), ("hidden", c_i32), ("sh_dim", c_i32), ("w_dtype", c_i32)]


class HeadsOutputs(ctypes.Structure):
    _fields_ = [("scale", c_vp), ("rot", c_vp), ("sh", c_vp), ("opacity", c_vp), ("cov", c_vp), ("latent", c_vp),
                ("raw", c_vp)]


class HeadsOutputGrads(ctypes.Structure):
    _fields_ = [("scale", c_vp), ("rot", c_vp), ("sh", c_vp), ("opacity", c_vp), ("cov", c_vp)]


class AdamGroup(ctypes.Structure):
    _fields_ = [("end", c_i64), ("lr", c_f32)]


class Camera(ctypes.Structure):
    _fields_ = [("view", c_f32 * 12), ("fx", c_f32), ("fy", c_f32), ("cx", c_f32), ("cy", c_f32),
                ("width", c_i32), ("height", c_i32), ("z_near", c_f32)]


class RenderDesc(ctypes.Structure):
    _fields_ = [("sh_degree", c_i32), ("lowpass", c_f32), ("alpha_max", c_f32), ("alpha_min", c_f32),
                ("t_stop", c_f32), ("background", c_f32 * 3), ("mean_stride", c_i32), ("reserved", c_i32)]


P = ctypes.POINTER
_SIGS = {
    "spin4d_grid_init": (c_i32, [P(GridDesc), c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_f32, c_f32]),
    "spin4d_mlp_param_count": (c_i64, [P(MlpDesc)]),
    "spin4d_encode_fwd": (c_i32, [P(GridDesc), c_vp, c_i64, c_vp, c_vp, c_vp]),
    "spin4d_decode_fwd": (c_i32, [P(GridDesc), P(MlpDesc), c_vp, c_i64, c_vp, c_vp, c_vp, Outputs, c_vp]),
    "spin4d_decode_bwd_workspace": (c_sz, [P(GridDesc), P(MlpDesc), c_i64]),
    "spin4d_decode_bwd": (c_i32, [P(GridDesc), P(MlpDesc), c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, P(OutputGrads),
                                  c_vp, c_vp, c_vp, c_sz, c_vp]),
    "spin4d_decode_bwd_ext": (c_i32, [P(GridDesc), P(MlpDesc), c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, P(OutputGrads),
                                      c_vp, c_vp, P(ExtraGrads), c_vp, c_sz, c_vp]),
    "spin4d_decode_bwd_noalloc_scratch_bytes": (c_sz, []),
    "spin4d_decode_bwd_noalloc": (c_i32, [P(GridDesc), P(MlpDesc), c_vp, c_i64, c_vp, c_vp, c_vp, c_vp,
                                          P(OutputGrads), c_vp, c_vp, c_vp]),
    "spin4d_cov_assemble": (c_i32, [c_vp, c_vp, c_i64, c_vp, c_vp]),
    "spin4d_heads_param_count": (c_i64, [P(HeadsDesc)]),
    "spin4d_heads_fwd_workspace": (c_sz, [P(GridDesc), P(HeadsDesc), c_i64]),
    "spin4d_heads_fwd": (c_i32, [P(GridDesc), P(HeadsDesc), c_vp, c_i64, c_vp, c_vp, HeadsOutputs, c_vp, c_sz,
                                 c_vp]),
    "spin4d_heads_bwd_workspace": (c_sz, [P(GridDesc), P(HeadsDesc), c_i64]),
    "spin4d_heads_bwd": (c_i32, [P(GridDesc), P(HeadsDesc), c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, P(HeadsOutputGrads),
                                 c_vp, c_vp, c_vp, c_sz, c_vp]),
    "spin4d_adam_step_groups": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, P(AdamGroup), c_i32, c_i32, c_f32,
                                        c_f32, c_f32, c_i32, c_vp, c_vp]),
    "spin4d_lr_warmup_cosine": (ctypes.c_double, [c_i64, ctypes.c_double, ctypes.c_double, c_i64, c_i64]),
    "spin4d_adam_step": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i32, c_f32, c_f32, c_f32, c_f32, c_i32,
                                 c_vp, c_vp]),
    "spin4d_hexplane_plane_count": (c_i64, [P(HexDesc)]),
    "spin4d_hexplane_param_count": (c_i64, [P(HexDesc)]),
    "spin4d_hexplane_fwd": (c_i32, [P(HexDesc), c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, HexOutputs, c_vp]),
    "spin4d_hexplane_fwd_gated": (c_i32, [P(HexDesc), c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, P(HexGate),
                                          HexOutputs, c_vp]),
    "spin4d_hexplane_bwd_gated": (c_i32, [P(HexDesc), c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                          P(HexGate), P(HexOutputGrads), c_vp, c_vp, c_vp, c_sz, c_vp]),
    "spin4d_hexplane_bwd_saved": (c_i32, [P(HexDesc), c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, P(HexSaved),
                                          P(HexGate), P(HexOutputGrads), c_vp, c_vp, c_vp, c_sz, c_vp]),
    "spin4d_hexplane_bwd_workspace": (c_sz, [P(HexDesc), c_i64]),
    "spin4d_hexplane_bwd": (c_i32, [P(HexDesc), c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                    P(HexOutputGrads), c_vp, c_vp, c_vp, c_sz, c_vp]),
    "spin4d_debug_corners": (c_i32, [P(GridDesc), c_vp, c_i64, c_vp, c_vp, c_vp]),
    "spin4d_check_device_errors": (c_i32, [c_i32]),
    "spin4d_morton_order_workspace": (c_sz, [c_i64]),
    "spin4d_morton_order": (c_i32, [P(GridDesc), c_vp, c_i64, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "spin4d_permute_rows": (c_i32, [c_vp, c_i64, c_vp, c_vp, c_i64, c_i64, c_vp]),
    "spin4d_render_state_bytes": (c_sz, [c_i64, c_i32, c_i32, c_i64]),
    "spin4d_render_fwd": (c_i32, [P(Camera), P(RenderDesc), c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz,
                                  c_i64, c_vp]),
    "spin4d_render_bwd": (c_i32, [P(Camera), P(RenderDesc), c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_i64,
                                  c_vp, c_vp, c_vp, c_vp, c_vp]),
    "spin4d_checked_build": (c_i32, []),
    "spin4d_l2_window_set": (c_i32, [c_vp, c_vp, c_sz, P(c_sz)]),
    "spin4d_l2_window_clear": (c_i32, [c_vp]),
    "spin4d_status_string": (ctypes.c_char_p, [c_i32]),
    "spin4d_last_cuda_error": (c_i32, []),
    "spin4d_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


class Spin4dError(RuntimeError):
    def __init__(self, call: str, status: int):
        msg = lib.spin4d_status_string(status).decode()
        if status == ERR_CUDA:
            msg += " (cudaError %d)" % lib.spin4d_last_cuda_error()
        super().__init__("%s failed: %s [%d]" % (call, msg, status))
        self.status = status


def _check(call: str, status: int) -> None:
    if status != OK:
        raise Spin4dError(call, status)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


_DT = {"f32": F32, "f16": F16, torch.float32: F32, torch.float16: F16}


# ---------------------------------------------------------------------------
# Descriptors
# ---------------------------------------------------------------------------
def grid_desc(L: int, F: int, log2_T: int, dtype, nmin_s: int, nmax_s: int, nmin_t: int, nmax_t: int,
              t_min: float, t_max: float, normalised_input: bool = False) -> GridDesc:
    g = GridDesc()
    _check("spin4d_grid_init", lib.spin4d_grid_init(ctypes.byref(g), L, F, log2_T, _DT[dtype], nmin_s, nmax_s,
                                                    nmin_t, nmax_t, t_min, t_max))
    if normalised_input:
        g.flags |= INPUT_NORMALISED
    return g


def grid_from_spec(spec, normalised_input: bool = False) -> GridDesc:
    return grid_desc(spec.L, spec.F, spec.log2_T, spec.dtype, spec.nmin_s, spec.nmax_s, spec.nmin_t,
                     spec.nmax_t, spec.t_min, spec.t_max, normalised_input)


def mlp_desc(in_dim: int, hidden: int, n_hidden: int, dtype, gate: bool = False, tau: float = 0.02) -> MlpDesc:
    return MlpDesc(in_dim, hidden, n_hidden, _DT[dtype], 1 if gate else 0, tau)


def mlp_from_spec(spec) -> MlpDesc:
    return mlp_desc(spec.in_dim, spec.hidden, spec.n_hidden, spec.dtype, spec.gate, spec.tau)


def mlp_param_count(m: MlpDesc) -> int:
    return int(lib.spin4d_mlp_param_count(ctypes.byref(m)))


def hex_desc(scales=(64, 128, 256), time_res: int = 75, channels: int = 32, n_frames: int = 150,
             hidden: int = 64, n_hidden: int = 2) -> HexDesc:
    h = HexDesc()
    h.n_scales = len(scales)
    for i, s in enumerate(scales):
        h.scales[i] = s
    h.time_res, h.channels, h.n_frames, h.hidden, h.n_hidden = time_res, channels, n_frames, hidden, n_hidden
    return h


def hex_from_spec(spec) -> HexDesc:
    return hex_desc(spec.scales, spec.time_res, spec.channels, spec.n_frames, spec.hidden, spec.n_hidden)


# ---------------------------------------------------------------------------
# Calls
# ---------------------------------------------------------------------------
def encode_fwd(g: GridDesc, pos: torch.Tensor, tables: torch.Tensor, z: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    N = pos.shape[0]
    if z is None:
        z = torch.empty((N, g.L * g.F), dtype=torch.float32, device=pos.device)
    _check("spin4d_encode_fwd", lib.spin4d_encode_fwd(ctypes.byref(g), _ptr(pos), N, _ptr(tables), _ptr(z),
                                                      _stream(stream)))
    return z


def alloc_outputs(N: int, device, latent_dim: int = 0) -> Dict[str, torch.Tensor]:
    """Output tensors; latent_dim = L*F also allocates the saved latent z."""
    out = {k: torch.empty((N, w), dtype=torch.float32, device=device)
           for k, w in (("scale", 3), ("rot", 4), ("rgb", 3), ("opacity", 1), ("cov", 6))}
    if latent_dim:
        out["latent"] = torch.empty((N, latent_dim), dtype=torch.float32, device=device)
    return out


def decode_fwd(g: GridDesc, m: MlpDesc, pos: torch.Tensor, tables: torch.Tensor, weights: torch.Tensor,
               gate_cr: Optional[torch.Tensor] = None, out: Optional[Dict[str, torch.Tensor]] = None,
               stream=None) -> Dict[str, torch.Tensor]:
    N = pos.shape[0]
    if out is None:
        out = alloc_outputs(N, pos.device)
    o = Outputs(*(_ptr(out.get(k)) for k in ("scale", "rot", "rgb", "opacity", "cov", "latent")))
    _check("spin4d_decode_fwd", lib.spin4d_decode_fwd(ctypes.byref(g), ctypes.byref(m), _ptr(pos), N, _ptr(tables),
                                                      _ptr(weights), _ptr(gate_cr), o, _stream(stream)))
    return out


def decode_bwd_workspace(g: GridDesc, m: MlpDesc, N: int) -> int:
    return int(lib.spin4d_decode_bwd_workspace(ctypes.byref(g), ctypes.byref(m), N))


def decode_bwd(g: GridDesc, m: MlpDesc, pos, tables, weights, grads: Dict[str, torch.Tensor],
               grad_tables: torch.Tensor, grad_weights: torch.Tensor, gate_cr=None,
               workspace: Optional[torch.Tensor] = None, latent: Optional[torch.Tensor] = None,
               grad_pos: Optional[torch.Tensor] = None, grad_gate: Optional[torch.Tensor] = None,
               stream=None) -> None:
    """latent: the z saved by decode_fwd for the same positions (optional);
    grad_pos: N x 3 fp32 accumulating the position gradient (optional);
    grad_gate: N x 2 fp32 accumulating the gradient w.r.t. the gate's (c, r)
    (optional, gated decoders)."""
    N = pos.shape[0]
    need = decode_bwd_workspace(g, m, N)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=pos.device)
    go = OutputGrads(*(_ptr(grads.get(k)) for k in ("scale", "rot", "rgb", "opacity", "cov")))
    common = (ctypes.byref(g), ctypes.byref(m), _ptr(pos), N, _ptr(tables), _ptr(weights), _ptr(gate_cr),
              _ptr(latent), ctypes.byref(go), _ptr(grad_tables), _ptr(grad_weights))
    if grad_pos is None and grad_gate is None:
        _check("spin4d_decode_bwd", lib.spin4d_decode_bwd(*common, _ptr(workspace), workspace.numel(),
                                                          _stream(stream)))
    else:
        extra = ExtraGrads(_ptr(grad_pos), _ptr(grad_gate))
        _check("spin4d_decode_bwd_ext", lib.spin4d_decode_bwd_ext(*common, ctypes.byref(extra), _ptr(workspace),
                                                                  workspace.numel(), _stream(stream)))


# the size of the library's built-in scratch, as the library was compiled
NOALLOC_SCRATCH_BYTES = int(lib.spin4d_decode_bwd_noalloc_scratch_bytes())


def decode_bwd_noalloc(g: GridDesc, m: MlpDesc, pos, tables, weights, grads: Dict[str, torch.Tensor],
                       grad_tables: torch.Tensor, grad_weights: torch.Tensor, gate_cr=None,
                       latent: Optional[torch.Tensor] = None, stream=None) -> None:
    """decode_bwd using the library's built-in scratch instead of a caller
    workspace (for hosts that cannot allocate device memory).  Calls that
    overlap on the GPU race on that scratch."""
    go = OutputGrads(*(_ptr(grads.get(k)) for k in ("scale", "rot", "rgb", "opacity", "cov")))
    _check("spin4d_decode_bwd_noalloc",
           lib.spin4d_decode_bwd_noalloc(ctypes.byref(g), ctypes.byref(m), _ptr(pos), pos.shape[0], _ptr(tables),
                                         _ptr(weights), _ptr(gate_cr), _ptr(latent), ctypes.byref(go),
                                         _ptr(grad_tables), _ptr(grad_weights), _stream(stream)))


def cov_assemble(scale: torch.Tensor, rot: torch.Tensor, cov: Optional[torch.Tensor] = None, stream=None):
    N = scale.shape[0]
    if cov is None:
        cov = torch.empty((N, 6), dtype=torch.float32, device=scale.device)
    _check("spin4d_cov_assemble", lib.spin4d_cov_assemble(_ptr(scale), _ptr(rot), N, _ptr(cov), _stream(stream)))
    return cov


def adam_step(params, grad, m, v, step: int, lr: float, b1: float, b2: float, eps: float,
              params_work: Optional[torch.Tensor] = None, zero_grad: bool = False,
              nonfinite_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    _check("spin4d_adam_step", lib.spin4d_adam_step(_ptr(params), _ptr(params_work), _ptr(grad), _ptr(m), _ptr(v),
                                                    params.numel(), step, lr, b1, b2, eps, 1 if zero_grad else 0,
                                                    _ptr(nonfinite_flag), _stream(stream)))


def adam_step_groups(params, grad, m, v, step: int, groups, b1: float, b2: float, eps: float,
                     params_work: Optional[torch.Tensor] = None, zero_grad: bool = False,
                     nonfinite_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """groups: [(end, lr), ...] with increasing ends, the last = params.numel()."""
    arr = (AdamGroup * len(groups))(*[AdamGroup(int(e), float(lr)) for e, lr in groups])
    _check("spin4d_adam_step_groups", lib.spin4d_adam_step_groups(
        _ptr(params), _ptr(params_work), _ptr(grad), _ptr(m), _ptr(v), params.numel(), arr, len(groups), step, b1, b2,
        eps, 1 if zero_grad else 0, _ptr(nonfinite_flag), _stream(stream)))


def lr_warmup_cosine(step: int, lr_max: float, lr_min: float, warmup: int, total: int) -> float:
    return float(lib.spin4d_lr_warmup_cosine(step, lr_max, lr_min, warmup, total))


# ---- the paper's four-head decoder ----
HEADS_KEYS = ("scale", "rot", "sh", "opacity", "cov")


def heads_desc(in_dim: int, hidden: int = 64, sh_dim: int = 48, w_dtype: str = "f16") -> HeadsDesc:
    return HeadsDesc(in_dim, hidden, sh_dim, F16 if w_dtype == "f16" else F32)


def heads_from_spec(spec) -> HeadsDesc:
    return heads_desc(spec.in_dim, spec.hidden, spec.sh_dim, spec.dtype)


def heads_param_count(h: HeadsDesc) -> int:
    return int(lib.spin4d_heads_param_count(ctypes.byref(h)))


def heads_fwd(g: GridDesc, h: HeadsDesc, pos, tables, weights, out=None, latent: bool = False, raw: bool = False,
              stream=None, workspace="auto"):
    """Outputs dict; with latent / raw it also holds z (N x in_dim) and the
    raw scale, rotation and opacity head outputs (N x 8) for heads_bwd.
    workspace: "auto" allocates what spin4d_heads_fwd_workspace asks for,
    None passes none (the fused kernel), or a uint8 device tensor."""
    N = pos.shape[0]
    if isinstance(workspace, str):
        need = lib.spin4d_heads_fwd_workspace(ctypes.byref(g), ctypes.byref(h), N)
        workspace = torch.empty(need, dtype=torch.uint8, device=pos.device) if need else None
    widths = {"scale": 3, "rot": 4, "sh": h.sh_dim, "opacity": 1, "cov": 6}
    if out is None:
        out = {k: torch.empty((N, w), dtype=torch.float32, device=pos.device) for k, w in widths.items()}
        if latent:
            out["latent"] = torch.empty((N, h.in_dim), dtype=torch.float32, device=pos.device)
        if raw:
            out["raw"] = torch.empty((N, 8), dtype=torch.float32, device=pos.device)
    o = HeadsOutputs(*(_ptr(out[k]) for k in HEADS_KEYS), _ptr(out.get("latent")), _ptr(out.get("raw")))
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("spin4d_heads_fwd", lib.spin4d_heads_fwd(ctypes.byref(g), ctypes.byref(h), _ptr(pos), N, _ptr(tables),
                                                    _ptr(weights), o, _ptr(workspace), ws_bytes, _stream(stream)))
    return out


def heads_bwd(g: GridDesc, h: HeadsDesc, pos, tables, weights, grads, grad_tables, grad_weights, latent=None,
              workspace=None, stream=None, raw=None) -> None:
    """grad_tables and grad_weights += the gradients of sum_k <grads[k], output_k>.
    latent and raw are the forward's saved z and raw head outputs (optional);
    with both, the paper's configuration runs on the tensor cores.  The
    workspace (uint8 device tensor) is allocated when not given."""
    N = pos.shape[0]
    if workspace is None:
        need = int(lib.spin4d_heads_bwd_workspace(ctypes.byref(g), ctypes.byref(h), N))
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=pos.device)
    go = HeadsOutputGrads(*(_ptr(grads.get(k)) for k in HEADS_KEYS))
    _check("spin4d_heads_bwd", lib.spin4d_heads_bwd(ctypes.byref(g), ctypes.byref(h), _ptr(pos), N, _ptr(tables),
                                                    _ptr(weights), _ptr(latent), _ptr(raw), ctypes.byref(go),
                                                    _ptr(grad_tables),
                                                    _ptr(grad_weights), _ptr(workspace), workspace.numel(),
                                                    _stream(stream)))


def hexplane_plane_count(h: HexDesc) -> int:
    return int(lib.spin4d_hexplane_plane_count(ctypes.byref(h)))


def hexplane_param_count(h: HexDesc) -> int:
    return int(lib.spin4d_hexplane_param_count(ctypes.byref(h)))


HEX_KEYS = (("mu", 3), ("rot", 4), ("scale", 3), ("sh", 48), ("cov", 6))


def hexplane_fwd(h: HexDesc, inp: Dict[str, torch.Tensor], planes, weights, out=None, stream=None,
                 gate_cr: Optional[torch.Tensor] = None, tau: float = 0.02):
    """With ``gate_cr`` (N x 2 window centre and half-width) the energy-flow
    window gates the deformation (spin4d_hexplane_fwd_gated)."""
    N = inp["mu"].shape[0]
    if out is None:
        out = {k: torch.empty((N, w), dtype=torch.float32, device=planes.device) for k, w in HEX_KEYS}
    o = HexOutputs(*(_ptr(out[k]) for k, _ in HEX_KEYS), _ptr(out.get("latent")), _ptr(out.get("hidden")))
    common = (ctypes.byref(h), _ptr(inp["mu"]), _ptr(inp["frame"]), N, _ptr(planes), _ptr(weights),
              _ptr(inp["q_can"]), _ptr(inp["logs_can"]), _ptr(inp["sh_can"]))
    if gate_cr is None:
        _check("spin4d_hexplane_fwd", lib.spin4d_hexplane_fwd(*common, o, _stream(stream)))
    else:
        gate = HexGate(_ptr(gate_cr), tau, None)
        _check("spin4d_hexplane_fwd_gated", lib.spin4d_hexplane_fwd_gated(*common, ctypes.byref(gate), o,
                                                                          _stream(stream)))
    return out


def hexplane_bwd_workspace(h: HexDesc, N: int) -> int:
    return int(lib.spin4d_hexplane_bwd_workspace(ctypes.byref(h), N))


def hexplane_bwd(h: HexDesc, inp, planes, weights, grads, grad_planes, grad_weights, workspace=None, latent=None,
                 stream=None, gate_cr: Optional[torch.Tensor] = None, tau: float = 0.02,
                 grad_cr: Optional[torch.Tensor] = None, hidden: Optional[torch.Tensor] = None):
    """With ``gate_cr`` the backward of the windowed deformation
    (spin4d_hexplane_bwd_gated); ``grad_cr`` (N x 2) += d loss / d(c, r).
    ``hidden`` (the forward's saved h1, with ``latent``) selects
    spin4d_hexplane_bwd_saved."""
    N = inp["mu"].shape[0]
    if workspace is None:
        workspace = torch.empty(max(hexplane_bwd_workspace(h, N), 1), dtype=torch.uint8, device=planes.device)
    go = HexOutputGrads(*(_ptr(grads.get(k)) for k, _ in HEX_KEYS))
    common = (ctypes.byref(h), _ptr(inp["mu"]), _ptr(inp["frame"]), N, _ptr(planes), _ptr(weights),
              _ptr(inp["q_can"]), _ptr(inp["logs_can"]), _ptr(inp["sh_can"]), _ptr(latent))
    tail = (ctypes.byref(go), _ptr(grad_planes), _ptr(grad_weights), _ptr(workspace), workspace.numel(),
            _stream(stream))
    gate = None if gate_cr is None else HexGate(_ptr(gate_cr), tau, _ptr(grad_cr))
    if hidden is not None:
        saved = HexSaved(_ptr(latent), _ptr(hidden))
        _check("spin4d_hexplane_bwd_saved",
               lib.spin4d_hexplane_bwd_saved(*common[:-2], ctypes.byref(saved),
                                             ctypes.byref(gate) if gate is not None else None, *tail))
    elif gate is None:
        _check("spin4d_hexplane_bwd", lib.spin4d_hexplane_bwd(*common, *tail))
    else:
        _check("spin4d_hexplane_bwd_gated", lib.spin4d_hexplane_bwd_gated(*common, ctypes.byref(gate), *tail))


def debug_corners(g: GridDesc, pos: torch.Tensor, stream=None):
    N = pos.shape[0]
    idx = torch.empty((N, g.L, 16), dtype=torch.int32, device=pos.device)
    frac = torch.empty((N, g.L, 4), dtype=torch.float32, device=pos.device)
    _check("spin4d_debug_corners", lib.spin4d_debug_corners(ctypes.byref(g), _ptr(pos), N, _ptr(idx), _ptr(frac),
                                                            _stream(stream)))
    return idx, frac


def check_device_errors(clear: bool = True) -> None:
    """Synchronous: raises if a kernel's bounded device wait ran out."""
    _check("spin4d_check_device_errors", lib.spin4d_check_device_errors(1 if clear else 0))


def morton_order(g: GridDesc, pos: torch.Tensor, workspace: Optional[torch.Tensor] = None, stream=None):
    """(sorted 30-bit Z-order keys, permutation), both N int32 holding uint32 values."""
    N = pos.shape[0]
    keys = torch.empty(N, dtype=torch.int32, device=pos.device)
    perm = torch.empty(N, dtype=torch.int32, device=pos.device)
    need = int(lib.spin4d_morton_order_workspace(N))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=pos.device)
    _check("spin4d_morton_order", lib.spin4d_morton_order(ctypes.byref(g), _ptr(pos), N, _ptr(keys), _ptr(perm),
                                                          _ptr(workspace), workspace.numel(), _stream(stream)))
    return keys, perm


def permute_rows(src: torch.Tensor, perm: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """out[i] = src[perm[i]] along the first dimension (contiguous tensors)."""
    N = perm.shape[0]
    if out is None:
        out = torch.empty((N,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    row_bytes = src[0].numel() * src.element_size() if src.dim() > 1 else src.element_size()
    _check("spin4d_permute_rows", lib.spin4d_permute_rows(_ptr(src), src.shape[0], _ptr(out), _ptr(perm), N,
                                                          row_bytes, _stream(stream)))
    return out


def l2_window_set(stream, buf: torch.Tensor, nbytes: Optional[int] = None) -> int:
    """Keeps ``buf`` (or its first ``nbytes``) persisting in L2 for the
    kernels launched on ``stream`` (a torch.cuda.Stream, not the default
    stream); returns the window's size in bytes."""
    applied = c_sz(0)
    n = buf.numel() * buf.element_size() if nbytes is None else nbytes
    _check("spin4d_l2_window_set", lib.spin4d_l2_window_set(_stream(stream), _ptr(buf), n, ctypes.byref(applied)))
    return int(applied.value)


def l2_window_clear(stream) -> None:
    _check("spin4d_l2_window_clear", lib.spin4d_l2_window_clear(_stream(stream)))


def version() -> str:
    return lib.spin4d_version().decode()


# ---------------------------------------------------------------------------
# Rendering (EWA projection + tile alpha compositing)
# ---------------------------------------------------------------------------
def camera(view, fx: float, fy: float, cx: float, cy: float, width: int, height: int,
           z_near: float = 0.2) -> Camera:
    """view: 3 x 4 world -> camera [R | t] (nested sequence or array)."""
    flat = [float(v) for row in view for v in row]
    if len(flat) != 12:
        raise ValueError("view must be 3 x 4")
    return Camera((c_f32 * 12)(*flat), fx, fy, cx, cy, int(width), int(height), z_near)


def camera_from_spec(spec) -> Camera:
    return camera(spec.view, spec.fx, spec.fy, spec.cx, spec.cy, spec.width, spec.height, spec.z_near)


def render_desc(sh_degree: int = 3, lowpass: float = 0.3, alpha_max: float = 0.99, alpha_min: float = 1.0 / 255.0,
                t_stop: float = 1e-4, background=(0.0, 0.0, 0.0), mean_stride: int = 3) -> RenderDesc:
    return RenderDesc(sh_degree, lowpass, alpha_max, alpha_min, t_stop, (c_f32 * 3)(*background), mean_stride, 0)


class RenderState:
    """Caller-owned state between ``render_fwd`` and ``render_bwd``."""

    def __init__(self, N: int, width: int, height: int, max_pairs: int, device):
        need = int(lib.spin4d_render_state_bytes(N, width, height, max_pairs))
        if need == 0:
            raise ValueError("invalid render sizes")
        self.N, self.width, self.height, self.max_pairs = N, width, height, max_pairs
        self.buf = torch.empty(need, dtype=torch.uint8, device=device)

    def pairs_needed(self) -> int:
        """(Gaussian, tile) pairs the last forward needed; synchronises."""
        return int(self.buf[:8].view(torch.int64).item())

    def pairs_kept(self) -> int:
        return int(self.buf[8:12].view(torch.int32).item())


def default_max_pairs(N: int, width: int, height: int) -> int:
    return max(16 * N, ((width + 15) // 16) * ((height + 15) // 16), 1 << 16)


def render_fwd(cam: Camera, desc: RenderDesc, means, cov, opacity, colours, image=None, final_T=None,
               state: Optional[RenderState] = None, stream=None):
    """Forward render; returns (image 3 x H x W, state).  Asynchronous: check
    ``state.pairs_needed() <= state.max_pairs`` (or use ``render``)."""
    N = means.shape[0]
    dev = means.device
    if state is None:
        state = RenderState(N, cam.width, cam.height, default_max_pairs(N, cam.width, cam.height), dev)
    if image is None:
        image = torch.empty((3, cam.height, cam.width), dtype=torch.float32, device=dev)
    _check("spin4d_render_fwd", lib.spin4d_render_fwd(ctypes.byref(cam), ctypes.byref(desc), N, _ptr(means),
                                                      _ptr(cov), _ptr(opacity), _ptr(colours), _ptr(image),
                                                      _ptr(final_T), _ptr(state.buf), state.buf.numel(),
                                                      state.max_pairs, _stream(stream)))
    return image, state


def render(cam: Camera, desc: RenderDesc, means, cov, opacity, colours, final_T=None,
           state: Optional[RenderState] = None, stream=None):
    """Forward render that grows the pair capacity until the frame fits
    (one host synchronisation per attempt)."""
    image, state = render_fwd(cam, desc, means, cov, opacity, colours, final_T=final_T, state=state, stream=stream)
    need = state.pairs_needed()
    if need > state.max_pairs:
        state = RenderState(means.shape[0], cam.width, cam.height, need, means.device)
        image, state = render_fwd(cam, desc, means, cov, opacity, colours, image=image, final_T=final_T,
                                  state=state, stream=stream)
    return image, state


def render_bwd(cam: Camera, desc: RenderDesc, means, cov, opacity, colours, grad_image, state: RenderState,
               grad_means=None, grad_cov=None, grad_opacity=None, grad_colours=None, stream=None):
    """Accumulates the render's gradients into the given tensors (allocating
    zeroed ones for those left None); returns them as a dict."""
    N = means.shape[0]
    dev = means.device
    z = lambda shape: torch.zeros(shape, dtype=torch.float32, device=dev)   # noqa: E731
    grad_means = z((N, 3)) if grad_means is None else grad_means
    grad_cov = z((N, 6)) if grad_cov is None else grad_cov
    grad_opacity = z((N,)) if grad_opacity is None else grad_opacity
    grad_colours = z(tuple(colours.shape)) if grad_colours is None else grad_colours
    _check("spin4d_render_bwd", lib.spin4d_render_bwd(ctypes.byref(cam), ctypes.byref(desc), N, _ptr(means),
                                                      _ptr(cov), _ptr(opacity), _ptr(colours), _ptr(grad_image),
                                                      _ptr(state.buf), state.buf.numel(), state.max_pairs,
                                                      _ptr(grad_means), _ptr(grad_cov), _ptr(grad_opacity),
                                                      _ptr(grad_colours), _stream(stream)))
    return dict(mu=grad_means, cov=grad_cov, opacity=grad_opacity, colours=grad_colours)
