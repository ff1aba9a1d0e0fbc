"""Seeded synthetic inputs for the SPIN-4DGS attribute decoder.

This module only draws data: positions, initial parameters and upstream
gradients, from numpy's PCG64 generator.  It holds none of the decoder's
arithmetic (no normalisation, no hashing, no resolutions, no interpolation,
no network).  Both the CUDA path and the CPU oracle receive exactly these
arrays, so it is the one module the two sides share.

Workloads (all seeded, default seed 0):

* ``tiny_fp32``      - 4096 positions, xyz ~ U[-1,1]^3, t ~ U[0,1].
* ``sports_frame``   - one frame (t = 75 of 150) of a fast-motion sports-like
  scene: 80 % static points ~ U[-1,1]^3 and 20 % in 8 rigid Gaussian blobs
  (sigma 0.03) whose centres fly ballistic arcs under gravity with specular
  bounces, moving at most 0.1 box units per frame.  This stands in for the
  CMU Panoptic Sports scenes (150 frames at 30 FPS, large inter-frame
  displacement) named in *Implicit 4D Gaussian Splatting for Fast Motion with
  Large Inter-Frame Displacements*, section 4 "Datasets".
* ``sports_sequence`` - all 150 frames of the same scene, frame-major.
* ``hexplane``       - canonical Gaussians mu ~ U[-1,1]^3, frame k ~ U{0..149}.
* ``stress``         - positions of the sports scene with a random frame per
  position, plus per-Gaussian temporal-window centres and half-widths.

Parameter initialisation follows section 3.3 of the same page (scale bias -5,
rotation bias (1,0,0,0), opacity bias logit(0.1), colour without special
initialisation) with Xavier-uniform weights and U(+-1e-4) hash tables.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np

HEAD_ROWS = 11          # scale 3, rotation 4, rgb 3, opacity 1
HEX_HEAD_ROWS = 58      # d_mu 3, d_q 4, d_logs 3, d_sh 48
HEX_CHANNELS = 32
HEX_SCALES = (64, 128, 256)
HEX_TIME_RES = 75
N_FRAMES = 150


@dataclasses.dataclass(frozen=True)
class GridSpec:
    """Sizes of a 4D multiresolution hash grid (no derived quantities)."""
    L: int
    F: int
    log2_T: int
    nmin_s: int
    nmax_s: int
    nmin_t: int
    nmax_t: int
    dtype: str                 # "f32" or "f16" table storage
    t_min: float
    t_max: float


@dataclasses.dataclass(frozen=True)
class MlpSpec:
    in_dim: int
    hidden: int
    n_hidden: int
    dtype: str                 # "f32" or "f16" weight storage
    gate: bool = False
    tau: float = 0.02

    def layer_shapes(self) -> List[Tuple[int, int]]:
        """(out, in) of each linear layer: trunk layers, then the 11-row head."""
        shapes = []
        d = self.in_dim
        for _ in range(self.n_hidden):
            shapes.append((self.hidden, d))
            d = self.hidden
        shapes.append((HEAD_ROWS, d))
        return shapes

    def n_params(self) -> int:
        return sum(o * i + o for o, i in self.layer_shapes())


@dataclasses.dataclass(frozen=True)
class HexSpec:
    hidden: int = 64
    n_hidden: int = 2
    channels: int = HEX_CHANNELS
    scales: Tuple[int, ...] = HEX_SCALES
    time_res: int = HEX_TIME_RES
    n_frames: int = N_FRAMES

    @property
    def in_dim(self) -> int:
        return len(self.scales) * 6 * self.channels

    def layer_shapes(self) -> List[Tuple[int, int]]:
        shapes = []
        d = self.in_dim
        for _ in range(self.n_hidden):
            shapes.append((self.hidden, d))
            d = self.hidden
        shapes.append((HEX_HEAD_ROWS, d))
        return shapes

    def n_params(self) -> int:
        return sum(o * i + o for o, i in self.layer_shapes())

    def plane_shapes(self) -> List[Tuple[int, int]]:
        """(rows, cols) of each plane, scale-major, planes XY XZ YZ XT YT ZT.

        A plane over axes (a, b) is stored [rows = res_b][cols = res_a][C]."""
        out = []
        for m in self.scales:
            out += [(m, m), (m, m), (m, m),
                    (self.time_res, m), (self.time_res, m), (self.time_res, m)]
        return out

    def n_plane_floats(self) -> int:
        return sum(r * c for r, c in self.plane_shapes()) * self.channels


# ---------------------------------------------------------------------------
# Workload table.  Keys name the workload by what it is.
# ---------------------------------------------------------------------------
GRID_TINY = GridSpec(L=4, F=2, log2_T=12, nmin_s=4, nmax_s=32, nmin_t=4, nmax_t=32,
                     dtype="f32", t_min=0.0, t_max=1.0)
MLP_TINY = MlpSpec(in_dim=8, hidden=32, n_hidden=1, dtype="f32")

GRID_SPORTS = GridSpec(L=16, F=2, log2_T=19, nmin_s=16, nmax_s=2048, nmin_t=8, nmax_t=150,
                       dtype="f16", t_min=0.0, t_max=float(N_FRAMES - 1))
MLP_SPORTS = MlpSpec(in_dim=32, hidden=64, n_hidden=2, dtype="f16")

GRID_STRESS = GridSpec(L=16, F=4, log2_T=22, nmin_s=16, nmax_s=2048, nmin_t=8, nmax_t=150,
                       dtype="f16", t_min=0.0, t_max=float(N_FRAMES - 1))
MLP_STRESS = MlpSpec(in_dim=64, hidden=128, n_hidden=2, dtype="f16", gate=True, tau=0.02)

HEX = HexSpec()


@dataclasses.dataclass(frozen=True)
class HeadsSpec:
    """The paper's decoder: four heads (scale, rotation, SH colour, opacity),
    each a three-layer MLP in_dim -> hidden -> hidden -> rows."""
    in_dim: int
    hidden: int = 64
    sh_dim: int = 48
    dtype: str = "f16"

    def head_rows(self) -> Tuple[int, int, int, int]:
        return (3, 4, self.sh_dim, 1)

    def layer_shapes(self, head: int) -> List[Tuple[int, int]]:
        return [(self.hidden, self.in_dim), (self.hidden, self.hidden), (self.head_rows()[head], self.hidden)]

    def n_params(self) -> int:
        return sum(o * i + o for h in range(4) for o, i in self.layer_shapes(h))


# The paper's configuration (SPIN-4DGS section 4): hidden 64, L = 16, F = 4,
# hash tables of 2^21 entries; resolutions as the sports grid (the page gives
# none).
GRID_PAPER = GridSpec(L=16, F=4, log2_T=21, nmin_s=16, nmax_s=2048, nmin_t=8, nmax_t=150,
                      dtype="f16", t_min=0.0, t_max=float(N_FRAMES - 1))
HEADS_PAPER = HeadsSpec(in_dim=64)
GRID_TINY4 = GridSpec(L=4, F=4, log2_T=12, nmin_s=4, nmax_s=32, nmin_t=4, nmax_t=32,
                      dtype="f32", t_min=0.0, t_max=1.0)
HEADS_TINY = HeadsSpec(in_dim=16, hidden=16, sh_dim=12, dtype="f32")

WORKLOADS: Dict[str, dict] = {
    "tiny_fp32": dict(N=4096, grid=GRID_TINY, mlp=MLP_TINY, grad_std=1.0),
    "sports_frame_fp16": dict(N=300_000, grid=GRID_SPORTS, mlp=MLP_SPORTS, frame=75),
    "sports_train_fp16": dict(N=N_FRAMES * 300_000, batch=1_000_000, grid=GRID_SPORTS,
                              mlp=MLP_SPORTS, grad_std=1e-2, lr=1e-3, betas=(0.9, 0.99),
                              eps=1e-15),
    "hexplane_fp32": dict(N=500_000, hex=HEX, grad_std=1.0),
    "stress_fp16_gate": dict(N=4_000_000, grid=GRID_STRESS, mlp=MLP_STRESS, grad_std=1.0),
    # the paper's decoder: one 1M-position training launch of sports frames 0-3
    "paper_heads_fp16": dict(N=1_000_000, grid=GRID_PAPER, heads=HEADS_PAPER, grad_std=1e-2),
}


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f16":
        return a.astype(np.float16)
    if dtype == "f32":
        return a.astype(np.float32)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Positions
# ---------------------------------------------------------------------------
def uniform_positions(n: int, seed: int = 0, t_lo: float = 0.0, t_hi: float = 1.0) -> np.ndarray:
    """N x 4 float32 (x, y, z, t): xyz ~ U[-1,1]^3, t ~ U[t_lo, t_hi]."""
    g = rng(seed)
    p = np.empty((n, 4), np.float32)
    p[:, :3] = g.uniform(-1.0, 1.0, size=(n, 3))
    p[:, 3] = g.uniform(t_lo, t_hi, size=n)
    return p


@dataclasses.dataclass
class SportsScene:
    """A fixed synthetic scene; ``frame(k)`` returns the positions at frame k."""
    static: np.ndarray            # (n_static, 3)
    offsets: np.ndarray           # (n_clusters, per_cluster, 3) rigid blob offsets
    centres: np.ndarray           # (n_frames, n_clusters, 3) blob centre per frame

    @property
    def n_per_frame(self) -> int:
        return self.static.shape[0] + self.offsets.shape[0] * self.offsets.shape[1]

    def frame(self, k: int) -> np.ndarray:
        n = self.n_per_frame
        p = np.empty((n, 4), np.float32)
        ns = self.static.shape[0]
        p[:ns, :3] = self.static
        moving = self.centres[k][:, None, :] + self.offsets
        p[ns:, :3] = moving.reshape(-1, 3)
        p[:, 3] = float(k)
        return p

    def frames(self, ks) -> np.ndarray:
        return np.concatenate([self.frame(int(k)) for k in ks], axis=0)

    def max_displacement(self) -> float:
        d = np.linalg.norm(np.diff(self.centres, axis=0), axis=-1)
        return float(d.max())


def sports_scene(n_per_frame: int = 300_000, seed: int = 0, n_clusters: int = 8,
                 sigma: float = 0.03, n_frames: int = N_FRAMES, gravity: float = 0.002,
                 speed_range=(0.02, 0.08), vmax: float = 0.1, wall: float = 0.9) -> SportsScene:
    """80 % static background, 20 % in rigid blobs on bouncing ballistic paths."""
    g = rng(seed)
    n_moving = n_per_frame // 5
    per = n_moving // n_clusters
    n_static = n_per_frame - per * n_clusters
    static = g.uniform(-1.0, 1.0, size=(n_static, 3)).astype(np.float32)
    offsets = g.normal(0.0, sigma, size=(n_clusters, per, 3)).astype(np.float32)
    p = g.uniform(-0.5, 0.5, size=(n_clusters, 3))
    d = g.normal(size=(n_clusters, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    v = d * g.uniform(speed_range[0], speed_range[1], size=(n_clusters, 1))
    centres = np.empty((n_frames, n_clusters, 3))
    for k in range(n_frames):
        centres[k] = p
        v = v + np.array([0.0, -gravity, 0.0])
        sp = np.linalg.norm(v, axis=1, keepdims=True)
        v = np.where(sp > vmax, v * (vmax / np.maximum(sp, 1e-30)), v)
        p = p + v
        for ax in range(3):          # specular bounce off the walls
            hi = p[:, ax] > wall
            lo = p[:, ax] < -wall
            p[hi, ax] = 2 * wall - p[hi, ax]
            p[lo, ax] = -2 * wall - p[lo, ax]
            v[hi | lo, ax] = -v[hi | lo, ax]
    return SportsScene(static=static, offsets=offsets, centres=centres.astype(np.float32))


def stress_positions(n: int, seed: int = 0) -> np.ndarray:
    """Sports-scene positions with an independent random frame per position."""
    scene = sports_scene(300_000, seed)
    g = rng(seed + 101)
    frames = g.integers(0, N_FRAMES, size=n)
    slot = g.integers(0, scene.n_per_frame, size=n)
    ns = scene.static.shape[0]
    per = scene.offsets.shape[1]
    p = np.empty((n, 4), np.float32)
    is_static = slot < ns
    p[is_static, :3] = scene.static[slot[is_static]]
    m = ~is_static
    ms = slot[m] - ns
    cl, j = ms // per, ms % per
    p[m, :3] = scene.centres[frames[m], cl] + scene.offsets[cl, j]
    p[:, 3] = frames.astype(np.float32)
    return p


def gate_params(n: int, seed: int = 0) -> np.ndarray:
    """N x 2 float32 (c, r): window centre ~ U(0,1), half-width ~ U(0.05, 0.5)."""
    g = rng(seed + 202)
    cr = np.empty((n, 2), np.float32)
    cr[:, 0] = g.uniform(0.0, 1.0, size=n)
    cr[:, 1] = g.uniform(0.05, 0.5, size=n)
    return cr


# ---------------------------------------------------------------------------
# Parameters
# ---------------------------------------------------------------------------
def hash_tables(grid: GridSpec, seed: int = 0, scale: float = 1e-4) -> np.ndarray:
    """L x T x F tables ~ U(-scale, scale), stored in the grid's dtype."""
    g = rng(seed + 303)
    t = g.uniform(-scale, scale, size=(grid.L, 1 << grid.log2_T, grid.F))
    return _store(t, grid.dtype)


def _xavier(g: np.random.Generator, out_dim: int, in_dim: int) -> np.ndarray:
    bound = math.sqrt(6.0 / (in_dim + out_dim))
    return g.uniform(-bound, bound, size=(out_dim, in_dim))


HEAD_BIAS = np.array([-5.0, -5.0, -5.0,          # scale: exp(-5) ~ 0.0067
                      1.0, 0.0, 0.0, 0.0,        # rotation (w, x, y, z)
                      0.0, 0.0, 0.0,             # colour: no special init
                      math.log(0.1 / 0.9)])      # opacity: logit(0.1) ~ -2.197


def mlp_weights(mlp: MlpSpec, seed: int = 0, head_bias: bool = True,
                bias_scale: float = 0.0) -> np.ndarray:
    """Packed weight vector: per layer W[out][in] row-major, then b[out].

    Trunk layers are Xavier-uniform with zero bias (or U(+-bias_scale) when
    bias_scale > 0, used by parity cases that must exercise the bias path).
    The head is four Xavier-uniform blocks (fan_out 3/4/3/1) with the
    page's bias initialisation."""
    g = rng(seed + 404)
    parts = []
    shapes = mlp.layer_shapes()
    for li, (o, i) in enumerate(shapes):
        if li < len(shapes) - 1:
            W = _xavier(g, o, i)
            b = g.uniform(-bias_scale, bias_scale, size=o) if bias_scale > 0 else np.zeros(o)
        else:
            W = np.concatenate([_xavier(g, 3, i), _xavier(g, 4, i),
                                _xavier(g, 3, i), _xavier(g, 1, i)], axis=0)
            b = HEAD_BIAS.copy() if head_bias else g.uniform(-1, 1, size=o)
            if bias_scale > 0:
                b = b + g.uniform(-bias_scale, bias_scale, size=o)
        parts += [W.reshape(-1), b]
    return _store(np.concatenate(parts), mlp.dtype)


# Final-layer biases of the paper's heads (section 3.3): scale -5, rotation
# (1, 0, 0, 0), SH colour none, opacity logit(0.1).
HEADS_BIAS = ([-5.0, -5.0, -5.0], [1.0, 0.0, 0.0, 0.0], None, [math.log(0.1 / 0.9)])


def heads_weights(spec: HeadsSpec, seed: int = 0, bias_scale: float = 0.0) -> np.ndarray:
    """Packed weights of the four heads in order (scale, rotation, SH,
    opacity), each [W1 b1 W2 b2 W3 b3] with W[out][in] row-major:
    Xavier-uniform weights, hidden biases zero, final biases as the page
    initialises them; U(+-bias_scale) added to every bias when > 0."""
    g = rng(seed + 909)
    parts = []
    for h in range(4):
        shapes = spec.layer_shapes(h)
        for li, (o, i) in enumerate(shapes):
            W = _xavier(g, o, i)
            b = np.zeros(o)
            if li == 2 and HEADS_BIAS[h] is not None:
                b = np.array(HEADS_BIAS[h], np.float64)
            if bias_scale > 0:
                b = b + g.uniform(-bias_scale, bias_scale, size=o)
            parts += [W.reshape(-1), b]
    return _store(np.concatenate(parts), spec.dtype)


HEADS_OUT_WIDTHS = {"scale": 3, "rot": 4, "sh": 48, "opacity": 1, "cov": 6}


def hexplane_planes(hx: HexSpec, seed: int = 0, lo: float = 0.1, hi: float = 0.5) -> np.ndarray:
    """All planes packed scale-major, plane-major, [rows][cols][C], fp32."""
    g = rng(seed + 505)
    return g.uniform(lo, hi, size=hx.n_plane_floats()).astype(np.float32)


def hexplane_weights(hx: HexSpec, seed: int = 0, bias_scale: float = 0.0) -> np.ndarray:
    """Packed fp32 weights: trunk Xavier (zero bias), then geometry head
    (10 rows: d_mu 3, d_q 4, d_logs 3) and appearance head (48 rows) Xavier
    with zero bias, stacked as one 58-row layer."""
    g = rng(seed + 606)
    parts = []
    shapes = hx.layer_shapes()
    for li, (o, i) in enumerate(shapes):
        if li < len(shapes) - 1:
            W = _xavier(g, o, i)
        else:
            W = np.concatenate([_xavier(g, 10, i), _xavier(g, 48, i)], axis=0)
        b = g.uniform(-bias_scale, bias_scale, size=o) if bias_scale > 0 else np.zeros(o)
        parts += [W.reshape(-1), b]
    return np.concatenate(parts).astype(np.float32)


def hexplane_inputs(n: int, seed: int = 0) -> Dict[str, np.ndarray]:
    """Canonical Gaussians: mu ~ U[-1,1]^3, frame ~ U{0..149}, random unit
    quaternion, log-scale ~ U(ln 0.005, ln 0.05), SH ~ N(0, 0.1^2)."""
    g = rng(seed + 707)
    mu = g.uniform(-1.0, 1.0, size=(n, 3)).astype(np.float32)
    frame = g.integers(0, N_FRAMES, size=n).astype(np.int32)
    q = g.normal(size=(n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    logs = g.uniform(math.log(0.005), math.log(0.05), size=(n, 3))
    sh = g.normal(0.0, 0.1, size=(n, 48))
    return dict(mu=mu, frame=frame, q_can=q.astype(np.float32),
                logs_can=logs.astype(np.float32), sh_can=sh.astype(np.float32))


def upstream_grads(n: int, widths: Dict[str, int], std: float, seed: int = 0) -> Dict[str, np.ndarray]:
    """Upstream gradients ~ N(0, std^2), one float32 array per output."""
    g = rng(seed + 808)
    return {k: g.normal(0.0, std, size=(n, w)).astype(np.float32) for k, w in widths.items()}


DECODE_OUT_WIDTHS = {"scale": 3, "rot": 4, "rgb": 3, "opacity": 1, "cov": 6}
HEX_OUT_WIDTHS = {"mu": 3, "rot": 4, "scale": 3, "sh": 48, "cov": 6}


# ---------------------------------------------------------------------------
# Rendering inputs
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class CameraSpec:
    """A pinhole camera: view is the 3 x 4 world -> camera matrix [R | t]
    (camera looking along +z, y down the image), intrinsics in pixels."""
    view: Tuple[Tuple[float, ...], ...]
    fx: float
    fy: float
    cx: float
    cy: float
    width: int
    height: int
    z_near: float = 0.2


def orbit_camera(width: int = 640, height: int = 360, focal: float = 560.0, distance: float = 2.8,
                 azimuth_deg: float = 30.0, elevation_deg: float = 15.0, z_near: float = 0.2) -> CameraSpec:
    """A camera on a sphere of radius ``distance`` around the origin, looking
    at it (the Panoptic Sports cameras ring the dome at 640 x 360)."""
    az, el = math.radians(azimuth_deg), math.radians(elevation_deg)
    eye = distance * np.array([math.cos(el) * math.sin(az), -math.sin(el), -math.cos(el) * math.cos(az)])
    fwd = -eye / np.linalg.norm(eye)
    up = np.array([0.0, -1.0, 0.0])
    right = np.cross(up, fwd)
    right /= np.linalg.norm(right)
    down = np.cross(fwd, right)
    R = np.stack([right, down, fwd])                # rows: camera x, y, z axes in world coordinates
    t = -R @ eye
    view = np.concatenate([R, t[:, None]], axis=1).astype(np.float32)
    return CameraSpec(view=tuple(map(tuple, view.tolist())), fx=float(focal), fy=float(focal),
                      cx=width / 2.0, cy=height / 2.0, width=int(width), height=int(height), z_near=float(z_near))


def random_spd(n: int, sigmas: np.ndarray, g: np.random.Generator) -> np.ndarray:
    """n x 6 packed (xx, xy, xz, yy, yz, zz) symmetric positive-definite
    matrices U diag(sigmas^2) U^T, U a random orthogonal matrix (QR of a
    normal matrix)."""
    U, _ = np.linalg.qr(g.normal(size=(n, 3, 3)))
    M = U * (sigmas ** 2)[:, None, :]
    S = M @ np.transpose(U, (0, 2, 1))
    return np.stack([S[:, 0, 0], S[:, 0, 1], S[:, 0, 2], S[:, 1, 1], S[:, 1, 2], S[:, 2, 2]], axis=1)


def render_scene(n: int, seed: int = 0, positions: Optional[np.ndarray] = None, sh_degree: int = 3,
                 scale_factor: float = 1.0, opacity_lo: float = 0.05) -> Dict[str, np.ndarray]:
    """Attributes shaped like a trained scene: per-axis standard deviations
    log-normal (sigma 0.4) around ``scale_factor`` x the mean distance to the
    3 nearest neighbours (the initial scale 3D Gaussian Splatting gives each
    point, so dense regions get small Gaussians), random orientations,
    opacity = sigmoid(N(0, 2^2)) floored at ``opacity_lo``, SH coefficients
    with the degree-0 term U(0.4, 3.2) and the higher ones N(0, 0.1^2)
    (sh_degree -1: RGB U(0.05, 1)).  Positions default to frame 75 of the
    sports scene."""
    from scipy.spatial import cKDTree
    g = rng(seed + 909)
    if positions is None:
        positions = sports_scene(n, seed).frame(75)
    mu = np.ascontiguousarray(positions[:, :3], np.float32)
    n = mu.shape[0]
    k = min(3, n - 1)
    if k >= 1:
        dist, _ = cKDTree(mu.astype(np.float64)).query(mu.astype(np.float64), k=k + 1)
        s0 = scale_factor * np.maximum(dist[:, 1:].mean(axis=1), 1e-6)
    else:
        s0 = np.full(n, scale_factor * 0.1)
    sig = s0[:, None] * np.exp(g.normal(0.0, 0.4, size=(n, 3)))
    cov = random_spd(n, sig, g).astype(np.float32)
    op = 1.0 / (1.0 + np.exp(-g.normal(0.0, 2.0, size=n)))
    op = np.maximum(op, opacity_lo).astype(np.float32)
    if sh_degree < 0:
        col = g.uniform(0.05, 1.0, size=(n, 3)).astype(np.float32)
    else:
        K = (sh_degree + 1) ** 2
        col = g.normal(0.0, 0.1, size=(n, K, 3))
        col[:, 0, :] = g.uniform(0.4, 3.2, size=(n, 3))
        col = col.reshape(n, 3 * K).astype(np.float32)
    return dict(mu=mu, cov=cov, opacity=op, colours=col)


def image_grads(cam: CameraSpec, std: float = 1.0, seed: int = 0) -> np.ndarray:
    """3 x H x W float32 upstream image gradients ~ N(0, std^2)."""
    g = rng(seed + 1010)
    return g.normal(0.0, std, size=(3, cam.height, cam.width)).astype(np.float32)
