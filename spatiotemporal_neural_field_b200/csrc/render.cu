// EWA projection and tile-based alpha compositing of the decoded Gaussians
// (SPIN-4DGS section 3.1: Eq. 1 Gaussian, Eq. 3 Sigma_2D = J W Sigma W^T J^T,
// Eq. 4 front-to-back blending C = sum_i c_i a_i prod_{j<i} (1 - a_j)).
//
// Forward, all on one stream, no host synchronisation (graph-capturable;
// every kernel after the projection is a programmatic dependent launch of
// the one before it, see pdl.cuh):
//  1. project_kernel, one thread per Gaussian: camera transform, Eq. 3 with
//     the screen-space filter, conic, colour from the spherical harmonics,
//     the box of pixels its support can reach and the 16x16 tiles it spans.
//  2. Stable radix sort of the Gaussians by depth (the fp32 bits of a
//     positive depth order like the values).
//  3. Tile counts in depth order, their exclusive scan, then emit_pairs
//     writes (tile, Gaussian) pairs: Gaussians in depth order, so a stable
//     sort of the pairs by tile (ceil(tile bits / 8) passes) leaves every
//     tile's list in depth order, ties by Gaussian index.
//  4. tile_ranges_kernel marks each tile's run; rasterise_fwd runs one
//     256-thread CTA per tile, stages batches of 256 Gaussians in shared
//     memory, skips per warp the Gaussians whose support box misses the
//     warp's 8x4 block, and blends the rest into its pixels, leaving early
//     once every pixel's transmittance is spent.
// Backward: rasterise_bwd walks each pixel's list back to front, recovering
// the transmittance by division, sums each Gaussian's screen-space gradient
// over the warp's 32 pixels with a transposing shuffle reduction and adds it
// with one atomic per value;
// project_bwd_kernel chains it through the projection to the mean,
// covariance, opacity and colour inputs.
//
// The per-pixel arithmetic of the support test and alpha is written with
// explicit round-to-nearest intrinsics so the forward and backward kernels
// take bit-identical decisions.
#include <math.h>

#include <algorithm>

#include "host.h"
#include "pdl.cuh"
#include "radix.cuh"

namespace spin4d {
namespace {

constexpr int kTileSide = 16;
constexpr float kSupportD2 = 9.0f;    // 3-sigma ellipse

struct Cam {
  float R[9], t[3];
  float fx, fy, cx, cy;
  float campos[3];
  int W, H;
  float z_near;
};

struct Blend {
  int sh_degree, n_coef, mean_stride;
  float lowpass, alpha_max, alpha_min, t_stop;
  float bg[3];
  float log_amin;
  int tiles_x, tiles_y;
};

// ---------------------------------------------------------------------------
// real spherical harmonics up to degree 3, index l*l + l + m, no
// Condon-Shortley phase; the polynomial forms on the unit sphere
// ---------------------------------------------------------------------------
constexpr float kY0 = 0.28209479177387814f;    // 1 / (2 sqrt(pi))
constexpr float kY1 = 0.48860251190291992f;    // sqrt(3 / (4 pi))
constexpr float kY2a = 1.0925484305920792f;    // sqrt(15 / pi) / 2
constexpr float kY2b = 0.31539156525252005f;   // sqrt(5 / pi) / 4
constexpr float kY2c = 0.54627421529603959f;   // sqrt(15 / pi) / 4
constexpr float kY3a = 0.59004358992664352f;   // sqrt(35 / (2 pi)) / 4
constexpr float kY3b = 2.8906114426405538f;    // sqrt(105 / pi) / 2
constexpr float kY3c = 0.45704579946446572f;   // sqrt(21 / (2 pi)) / 4
constexpr float kY3d = 0.37317633259011540f;   // sqrt(7 / pi) / 4
constexpr float kY3e = 1.4453057213202769f;    // sqrt(105 / pi) / 4

__device__ __forceinline__ void sh_basis(int deg, float x, float y, float z, float* Y) {
  Y[0] = kY0;
  if (deg < 1) return;
  Y[1] = kY1 * y;
  Y[2] = kY1 * z;
  Y[3] = kY1 * x;
  if (deg < 2) return;
  const float xx = x * x, yy = y * y, zz = z * z;
  Y[4] = kY2a * x * y;
  Y[5] = kY2a * y * z;
  Y[6] = kY2b * (3.0f * zz - 1.0f);
  Y[7] = kY2a * x * z;
  Y[8] = kY2c * (xx - yy);
  if (deg < 3) return;
  Y[9] = kY3a * y * (3.0f * xx - yy);
  Y[10] = kY3b * x * y * z;
  Y[11] = kY3c * y * (5.0f * zz - 1.0f);
  Y[12] = kY3d * z * (5.0f * zz - 3.0f);
  Y[13] = kY3c * x * (5.0f * zz - 1.0f);
  Y[14] = kY3e * z * (xx - yy);
  Y[15] = kY3a * x * (xx - 3.0f * yy);
}

// g += w * grad Y_k (gradient of the polynomial form in R^3)
__device__ __forceinline__ void sh_grad_acc(int k, float w, float x, float y, float z, float* g) {
  switch (k) {
    case 1: g[1] += w * kY1; break;
    case 2: g[2] += w * kY1; break;
    case 3: g[0] += w * kY1; break;
    case 4: g[0] += w * kY2a * y; g[1] += w * kY2a * x; break;
    case 5: g[1] += w * kY2a * z; g[2] += w * kY2a * y; break;
    case 6: g[2] += w * kY2b * 6.0f * z; break;
    case 7: g[0] += w * kY2a * z; g[2] += w * kY2a * x; break;
    case 8: g[0] += w * kY2c * 2.0f * x; g[1] -= w * kY2c * 2.0f * y; break;
    case 9: g[0] += w * kY3a * 6.0f * x * y; g[1] += w * kY3a * 3.0f * (x * x - y * y); break;
    case 10: g[0] += w * kY3b * y * z; g[1] += w * kY3b * x * z; g[2] += w * kY3b * x * y; break;
    case 11: g[1] += w * kY3c * (5.0f * z * z - 1.0f); g[2] += w * kY3c * 10.0f * y * z; break;
    case 12: g[2] += w * kY3d * (15.0f * z * z - 3.0f); break;
    case 13: g[0] += w * kY3c * (5.0f * z * z - 1.0f); g[2] += w * kY3c * 10.0f * x * z; break;
    case 14: g[0] += w * kY3e * 2.0f * x * z; g[1] -= w * kY3e * 2.0f * y * z; g[2] += w * kY3e * (x * x - y * y); break;
    case 15: g[0] += w * kY3a * 3.0f * (x * x - y * y); g[1] -= w * kY3a * 6.0f * x * y; break;
    default: break;
  }
}

// ---------------------------------------------------------------------------
// projection of one Gaussian (Eq. 3)
// ---------------------------------------------------------------------------
struct Proj {
  float xc[3];
  float T0[3], T1[3];   // rows of J W
  float S[6];           // Sigma packed (xx, xy, xz, yy, yz, zz)
  float M0[3], M1[3];   // rows of (J W) Sigma
  float A, B, C, det;   // filtered Sigma_2D = [[A, B], [B, C]]
  float mx, my;
  bool visible;
};

__device__ __forceinline__ void project_one(const Cam& c, float lowpass, const float* __restrict__ mu,
                                            const float* __restrict__ cov, Proj& p) {
  const float m0 = __ldg(mu), m1 = __ldg(mu + 1), m2 = __ldg(mu + 2);
#pragma unroll
  for (int r = 0; r < 3; ++r) p.xc[r] = c.R[3 * r] * m0 + c.R[3 * r + 1] * m1 + c.R[3 * r + 2] * m2 + c.t[r];
  const float x = p.xc[0], y = p.xc[1], z = p.xc[2];
  p.visible = z > c.z_near;
  const float zs = p.visible ? z : 1.0f;
  const float iz = 1.0f / zs;
  const float j00 = c.fx * iz, j02 = -c.fx * x * iz * iz;
  const float j11 = c.fy * iz, j12 = -c.fy * y * iz * iz;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    p.T0[k] = j00 * c.R[k] + j02 * c.R[6 + k];
    p.T1[k] = j11 * c.R[3 + k] + j12 * c.R[6 + k];
  }
#pragma unroll
  for (int k = 0; k < 6; ++k) p.S[k] = __ldg(cov + k);
  const float* S = p.S;
  // Sigma rows: (S0 S1 S2), (S1 S3 S4), (S2 S4 S5)
  p.M0[0] = p.T0[0] * S[0] + p.T0[1] * S[1] + p.T0[2] * S[2];
  p.M0[1] = p.T0[0] * S[1] + p.T0[1] * S[3] + p.T0[2] * S[4];
  p.M0[2] = p.T0[0] * S[2] + p.T0[1] * S[4] + p.T0[2] * S[5];
  p.M1[0] = p.T1[0] * S[0] + p.T1[1] * S[1] + p.T1[2] * S[2];
  p.M1[1] = p.T1[0] * S[1] + p.T1[1] * S[3] + p.T1[2] * S[4];
  p.M1[2] = p.T1[0] * S[2] + p.T1[1] * S[4] + p.T1[2] * S[5];
  p.A = p.M0[0] * p.T0[0] + p.M0[1] * p.T0[1] + p.M0[2] * p.T0[2] + lowpass;
  p.B = p.M0[0] * p.T1[0] + p.M0[1] * p.T1[1] + p.M0[2] * p.T1[2];
  p.C = p.M1[0] * p.T1[0] + p.M1[1] * p.T1[1] + p.M1[2] * p.T1[2] + lowpass;
  p.det = p.A * p.C - p.B * p.B;
  p.mx = c.fx * x * iz + c.cx;
  p.my = c.fy * y * iz + c.cy;
  p.visible = p.visible && p.det > 0.0f && isfinite(p.det) && isfinite(p.mx) && isfinite(p.my) && isfinite(p.A) &&
              isfinite(p.C);
}

__device__ __forceinline__ void view_dir(const Cam& c, const float* __restrict__ mu, float d[3], float& nv) {
  const float v0 = __ldg(mu) - c.campos[0], v1 = __ldg(mu + 1) - c.campos[1], v2 = __ldg(mu + 2) - c.campos[2];
  nv = sqrtf(v0 * v0 + v1 * v1 + v2 * v2);
  const float inv = 1.0f / fmaxf(nv, 1e-30f);
  d[0] = v0 * inv;
  d[1] = v1 * inv;
  d[2] = v2 * inv;
}

constexpr int kProjThreads = 128;   // Gaussians per projection tile

// Colour rows of DEG (3 (DEG+1)^2 floats; DEG -1: 3) of one tile of
// Gaussians, staged through shared memory so global reads and writes are
// coalesced; padded by one float so each thread's row sits in its own banks.
template <int DEG>
struct ColourTile {
  static constexpr int kRow = DEG < 0 ? 3 : 3 * (DEG + 1) * (DEG + 1);
  static constexpr int kPitch = kRow + 1;
  static constexpr bool kStaged = DEG >= 0;
};

template <int DEG>
__device__ __forceinline__ void stage_rows(const float* __restrict__ src, int64_t n0, int nb, float* sm) {
  constexpr int R = ColourTile<DEG>::kRow, P = ColourTile<DEG>::kPitch;
  const float* g = src + n0 * R;
  for (int e = threadIdx.x; e < nb * R; e += kProjThreads) sm[(e / R) * P + e % R] = __ldg(g + e);
}

template <int DEG>
__global__ void __launch_bounds__(kProjThreads) project_kernel(
    Cam c, Blend b, int64_t N, const float* __restrict__ means, const float* __restrict__ cov,
    const float* __restrict__ opacity, const float* __restrict__ colours, float4* __restrict__ conic_o,
    float4* __restrict__ xy, float4* __restrict__ rgb, uint2* __restrict__ rect, uint32_t* __restrict__ ntiles,
    uint32_t* __restrict__ dkey) {
  pdl_wait();
  pdl_release();
  using CT = ColourTile<DEG>;
  constexpr int K = DEG < 0 ? 1 : (DEG + 1) * (DEG + 1);
  __shared__ float s_col[CT::kStaged ? kProjThreads * CT::kPitch : 1];
  for (int64_t n0 = (int64_t)blockIdx.x * kProjThreads; n0 < N; n0 += (int64_t)gridDim.x * kProjThreads) {
    const int nb = (int)min((int64_t)kProjThreads, N - n0);
    if (CT::kStaged) {
      __syncthreads();
      stage_rows<DEG>(colours, n0, nb, s_col);
      __syncthreads();
    }
    const int64_t n = n0 + threadIdx.x;
    if (threadIdx.x >= nb) continue;
    const float* mu = means + n * b.mean_stride;
    Proj p;
    project_one(c, b.lowpass, mu, cov + 6 * n, p);
    const float o = __ldg(opacity + n);
    uint32_t nt = 0, key = 0xFFFFFFFFu;
    float4 co = make_float4(0.f, 0.f, 0.f, 0.f), col = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 m = make_float4(0.f, 0.f, 0.f, 0.f);
    uint2 r = make_uint2(0u, 0u);
    // a Gaussian whose opacity is below alpha_min is skipped at every pixel
    if (p.visible && o >= b.alpha_min) {
      const float inv = 1.0f / p.det;
      co = make_float4(p.C * inv, -p.B * inv, p.A * inv, o);
      // support: d^2 <= 9 and o exp(-d^2/2) >= alpha_min; a slightly larger
      // box than the exact one keeps it a superset under fp32 rounding
      float r2 = kSupportD2;
      if (b.alpha_min > 0.0f) r2 = fminf(r2, 2.0f * (logf(o) - b.log_amin));
      r2 = r2 * 1.0001f + 0.01f;
      const float rx = sqrtf(r2 * p.A) + 0.01f, ry = sqrtf(r2 * p.C) + 0.01f;
      m = make_float4(p.mx, p.my, rx, ry);
      // pixel i is sampled at i + 1/2
      const int i0 = max((int)ceilf(fmaxf(p.mx - rx - 0.5f, -1.0f)), 0);
      const int i1 = min((int)floorf(fminf(p.mx + rx - 0.5f, (float)c.W)), c.W - 1);
      const int j0 = max((int)ceilf(fmaxf(p.my - ry - 0.5f, -1.0f)), 0);
      const int j1 = min((int)floorf(fminf(p.my + ry - 0.5f, (float)c.H)), c.H - 1);
      if (i0 <= i1 && j0 <= j1) {
        const uint32_t tx0 = i0 / kTileSide, tx1 = i1 / kTileSide, ty0 = j0 / kTileSide, ty1 = j1 / kTileSide;
        nt = (tx1 - tx0 + 1) * (ty1 - ty0 + 1);
        r = make_uint2(tx0 | (tx1 << 16), ty0 | (ty1 << 16));
        key = __float_as_uint(p.xc[2]);   // z > z_near > 0
      }
      if (DEG < 0) {
        const float* cc = colours + 3 * n;
        col = make_float4(__ldg(cc), __ldg(cc + 1), __ldg(cc + 2), 0.f);
      } else {
        float d[3], nv, Y[16];
        view_dir(c, mu, d, nv);
        sh_basis(DEG, d[0], d[1], d[2], Y);
        const float* k = s_col + threadIdx.x * CT::kPitch;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int i = 0; i < K; ++i) {
          s0 += Y[i] * k[3 * i];
          s1 += Y[i] * k[3 * i + 1];
          s2 += Y[i] * k[3 * i + 2];
        }
        col = make_float4(fmaxf(s0, 0.f), fmaxf(s1, 0.f), fmaxf(s2, 0.f), 0.f);
      }
    }
    conic_o[n] = co;
    xy[n] = m;
    rgb[n] = col;
    rect[n] = r;
    ntiles[n] = nt;
    dkey[n] = key;
  }
}

// cnt[k] = tile count of the k-th nearest Gaussian; header[0..1] += their
// exact 64-bit total (the 32-bit scan that follows may wrap; see emit_pairs)
__global__ void counts_in_order(const uint32_t* __restrict__ perm, const uint32_t* __restrict__ ntiles, int64_t N,
                                uint32_t* __restrict__ cnt, uint32_t* __restrict__ header) {
  pdl_wait();
  pdl_release();
  uint64_t local = 0;
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < N; k += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t c = ntiles[perm[k]];
    cnt[k] = c;
    local += c;
  }
  for (int s = 16; s > 0; s >>= 1) local += __shfl_xor_sync(0xffffffffu, local, s);
  if ((threadIdx.x & 31) == 0 && local) atomicAdd(reinterpret_cast<unsigned long long*>(header), local);
}

// header[2] = pairs that will be written: all of them when they fit, the
// first `cap` when they do not, none when the total overflows 32 bits (the
// scan's offsets would then wrap and could leave slots unwritten).
__global__ void clamp_pair_count(uint32_t* header, uint32_t cap) {
  pdl_wait();
  pdl_release();
  const uint64_t need = *reinterpret_cast<const unsigned long long*>(header);
  header[2] = need > 0xFFFFFFFFull ? 0u : (need > cap ? cap : (uint32_t)need);
}

// The pairs of the k-th nearest Gaussian at offs[k] .. offs[k] + cnt[k] - 1,
// those below cap only.
__global__ void emit_pairs(const uint32_t* __restrict__ perm, const uint32_t* __restrict__ cnt,
                           const uint32_t* __restrict__ offs, const uint2* __restrict__ rect, int64_t N, int tiles_x,
                           const uint32_t* __restrict__ header, uint32_t* __restrict__ pair_tile,
                           uint32_t* __restrict__ pair_id) {
  pdl_wait();
  pdl_release();
  const uint32_t kept = header[2];
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < N; k += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t c = cnt[k];
    if (c == 0) continue;
    const uint32_t g = perm[k];
    const uint2 r = rect[g];
    const uint32_t tx0 = r.x & 0xFFFFu, tx1 = r.x >> 16, ty0 = r.y & 0xFFFFu, ty1 = r.y >> 16;
    uint64_t o = offs[k];
    for (uint32_t ty = ty0; ty <= ty1 && o < kept; ++ty)
      for (uint32_t tx = tx0; tx <= tx1 && o < kept; ++tx, ++o) {
        pair_tile[o] = ty * (uint32_t)tiles_x + tx;
        pair_id[o] = g;
      }
  }
}

__global__ void tile_ranges_kernel(const uint32_t* __restrict__ tile, const uint32_t* __restrict__ header,
                                   int64_t cap, uint32_t n_tiles, uint2* __restrict__ ranges) {
  pdl_wait();
  pdl_release();
  const int64_t n = min((int64_t)header[2], cap);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t t = tile[i];
    if (t >= n_tiles) continue;   // never taken: every kept slot holds a tile of this image
    if (i == 0 || tile[i - 1] != t) ranges[t].x = (uint32_t)i;
    if (i == n - 1 || tile[i + 1] != t) ranges[t].y = (uint32_t)(i + 1);
  }
}

// d^2 = [dx dy] conic [dx dy]^T and G = exp(-d^2/2), rounding pinned
__device__ __forceinline__ float mahalanobis2(float4 co, float dx, float dy) {
  const float t = __fmul_rn(co.z, __fmul_rn(dy, dy));
  const float u = __fmaf_rn(__fmul_rn(__fmul_rn(2.0f, co.y), dx), dy, t);
  return __fmaf_rn(__fmul_rn(co.x, dx), dx, u);
}

// Rasterisers: one CTA of kRastThreads per 16x16 tile, one pixel a thread;
// each warp owns an 8x4 block ((warp & 1, warp >> 1) in a 2x4 grid of
// blocks), lane (lane & 7, lane >> 3) in it, and skips as a whole the
// Gaussians whose support box misses its block.
constexpr int kRastThreads = 256;
constexpr int kFewLanes = 10;   // backward: up to this many blending lanes add directly, more reduce first

struct TileGeom {
  int px, py;                   // the lane's pixel
  float wx0, wx1, wy0, wy1;     // the warp block's pixel centres, for the box test
};

__device__ __forceinline__ TileGeom tile_geom(const Blend& b) {
  const int tile = blockIdx.x;
  const int tx = tile % b.tiles_x, ty = tile / b.tiles_x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bx = tx * kTileSide + (warp & 1) * 8, by = ty * kTileSide + (warp >> 1) * 4;
  TileGeom g;
  g.px = bx + (lane & 7);
  g.py = by + (lane >> 3);
  g.wx0 = (float)bx + 0.5f;
  g.wx1 = (float)bx + 7.5f;
  g.wy0 = (float)by + 0.5f;
  g.wy1 = (float)by + 3.5f;
  return g;
}

// warp-uniform: the Gaussian's support box (centre m.xy, half-widths m.zw) misses the warp's block
__device__ __forceinline__ bool box_misses(const float4& m, const TileGeom& g) {
  return m.x + m.z < g.wx0 || m.x - m.z > g.wx1 || m.y + m.w < g.wy0 || m.y - m.w > g.wy1;
}

// Bit w set when the Gaussian's support box (centre m.xy, half-widths m.zw)
// reaches warp w's block of this tile (pixel centres bx + 0.5 .. bx + 7.5,
// by + 0.5 .. by + 3.5 for block (w & 1, w >> 1)); computed once per batch
// entry, so each warp then tests one bit.
__device__ __forceinline__ uint32_t block_mask(const float4& m, const Blend& b) {
  const int tile = blockIdx.x;
  const float x0 = (float)((tile % b.tiles_x) * kTileSide), y0 = (float)((tile / b.tiles_x) * kTileSide);
  const float lx = m.x - m.z, hx = m.x + m.z, ly = m.y - m.w, hy = m.y + m.w;
  uint32_t cols = 0, rows = 0;
#pragma unroll
  for (int c = 0; c < 2; ++c)
    if (hx >= x0 + 8.0f * c + 0.5f && lx <= x0 + 8.0f * c + 7.5f) cols |= 1u << c;
#pragma unroll
  for (int r = 0; r < 4; ++r)
    if (hy >= y0 + 4.0f * r + 0.5f && ly <= y0 + 4.0f * r + 3.5f) rows |= 1u << r;
  uint32_t mask = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w)
    if (((cols >> (w & 1)) & 1u) && ((rows >> (w >> 1)) & 1u)) mask |= 1u << w;
  return mask;
}

struct FwdPix {
  float fx, fy, T, c0, c1, c2;
  uint32_t last;
  bool done;
};

__device__ __forceinline__ void blend_step(FwdPix& q, const float4& co, const float4& m, const float4& cc,
                                           const Blend& b, uint32_t idx) {
  const float dx = __fsub_rn(q.fx, m.x), dy = __fsub_rn(q.fy, m.y);
  const float d2 = mahalanobis2(co, dx, dy);
  if (d2 > kSupportD2) return;
  const float a = fminf(b.alpha_max, __fmul_rn(co.w, __expf(__fmul_rn(-0.5f, d2))));
  if (a < b.alpha_min) return;
  const float Tn = __fmul_rn(q.T, __fsub_rn(1.0f, a));
  if (Tn < b.t_stop) {
    q.done = true;
    return;
  }
  const float w = a * q.T;
  q.c0 += cc.x * w;
  q.c1 += cc.y * w;
  q.c2 += cc.z * w;
  q.T = Tn;
  q.last = idx;
}

__device__ __forceinline__ void store_pixel(const FwdPix& q, int px, int py, int W, int H, const Blend& b,
                                            float* __restrict__ image, float* __restrict__ final_T,
                                            uint32_t* __restrict__ n_contrib, float* __restrict__ final_T_out) {
  if (px >= W || py >= H) return;
  const int64_t pix = (int64_t)py * W + px;
  const int64_t plane = (int64_t)W * H;
  image[pix] = q.c0 + q.T * b.bg[0];
  image[plane + pix] = q.c1 + q.T * b.bg[1];
  image[2 * plane + pix] = q.c2 + q.T * b.bg[2];
  final_T[pix] = q.T;
  n_contrib[pix] = q.last;
  if (final_T_out) final_T_out[pix] = q.T;
}

__global__ void __launch_bounds__(kRastThreads) rasterise_fwd(Blend b, int W, int H, const uint2* __restrict__ ranges,
                                                             const uint32_t* __restrict__ pair_id,
                                                             const float4* __restrict__ conic_o,
                                                             const float4* __restrict__ xy,
                                                             const float4* __restrict__ rgb, float* __restrict__ image,
                                                             float* __restrict__ final_T,
                                                             uint32_t* __restrict__ n_contrib,
                                                             float* __restrict__ final_T_out) {
  pdl_wait();
  pdl_release();
  __shared__ float4 s_co[kRastThreads];
  __shared__ float4 s_xy[kRastThreads];
  __shared__ float4 s_rgb[kRastThreads];
  __shared__ uint8_t s_mask[kRastThreads];
  const TileGeom g = tile_geom(b);
  const uint32_t wbit = 1u << (threadIdx.x >> 5);
  FwdPix q{(float)g.px + 0.5f, (float)g.py + 0.5f, 1.0f, 0.f, 0.f, 0.f, 0u, !(g.px < W && g.py < H)};
  const uint2 range = ranges[blockIdx.x];
  for (uint32_t base = range.x; base < range.y; base += kRastThreads) {
    // also the barrier that frees the previous batch's shared memory
    if (__syncthreads_count(q.done) == kRastThreads) break;
    const uint32_t i = base + threadIdx.x;
    if (i < range.y) {
      const uint32_t id = pair_id[i];
      s_co[threadIdx.x] = conic_o[id];
      const float4 m = xy[id];
      s_xy[threadIdx.x] = m;
      s_rgb[threadIdx.x] = rgb[id];
      s_mask[threadIdx.x] = (uint8_t)block_mask(m, b);
    }
    __syncthreads();
    const int cnt = (int)min((uint32_t)kRastThreads, range.y - base);
    for (int j = 0; j < cnt && !q.done; ++j) {
      if (!(s_mask[j] & wbit)) continue;   // the same for the whole warp
      blend_step(q, s_co[j], s_xy[j], s_rgb[j], b, base - range.x + j + 1);
    }
  }
  store_pixel(q, g.px, g.py, W, H, b, image, final_T, n_contrib, final_T_out);
}

// Sums each of v[0..15] over the warp with 16 shuffles instead of 80: every
// level hands half of the values to the partner lane and keeps the other
// half.  Lane L (and L ^ 1) ends with the total of value (L >> 1) & 15.
__device__ __forceinline__ float warp_transpose_sum16(float (&v)[16], int lane) {
#pragma unroll
  for (int lvl = 0; lvl < 4; ++lvl) {
    const int off = 16 >> lvl, half = 8 >> lvl;
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

struct BwdPix {
  float fx, fy, T, S, Tf, gbg, g0, g1, g2;
  uint32_t last;
};

__device__ __forceinline__ BwdPix bwd_pixel(int px, int py, int W, int H, const Blend& b,
                                            const float* __restrict__ final_T, const uint32_t* __restrict__ n_contrib,
                                            const float* __restrict__ grad_image) {
  BwdPix q{(float)px + 0.5f, (float)py + 0.5f, 1.0f, 0.f, 1.0f, 0.f, 0.f, 0.f, 0.f, 0u};
  if (px < W && py < H) {
    const int64_t pix = (int64_t)py * W + px, plane = (int64_t)W * H;
    q.T = final_T[pix];
    q.last = n_contrib[pix];
    q.g0 = grad_image[pix];
    q.g1 = grad_image[plane + pix];
    q.g2 = grad_image[2 * plane + pix];
  }
  q.Tf = q.T;
  q.gbg = q.g0 * b.bg[0] + q.g1 * b.bg[1] + q.g2 * b.bg[2];
  return q;
}

// One pixel's share of Gaussian j's screen-space gradient, added to v:
// (d x, d y, d conic a, b, c, d opacity, d r, d g, d b).  The decisions are
// the forward's (same arithmetic); j beyond the pixel's last blended
// Gaussian is skipped.  Returns whether the pixel blended Gaussian j.
__device__ __forceinline__ bool grad_step(BwdPix& q, uint32_t jidx, const float4& co, const float4& m,
                                          const float4& cc, const Blend& b, float (&v)[16]) {
  if (jidx >= q.last) return false;
  const float dx = __fsub_rn(q.fx, m.x), dy = __fsub_rn(q.fy, m.y);
  const float d2 = mahalanobis2(co, dx, dy);
  if (d2 > kSupportD2) return false;
  const float G = __expf(__fmul_rn(-0.5f, d2));
  const float raw = __fmul_rn(co.w, G);
  const float a = fminf(b.alpha_max, raw);
  if (a < b.alpha_min) return false;
  const float oma = 1.0f - a;
  const float Ti = q.T / oma;             // transmittance before Gaussian j
  const float gc = q.g0 * cc.x + q.g1 * cc.y + q.g2 * cc.z;
  float ga = Ti * gc - (q.S + q.Tf * q.gbg) / oma;
  const float wgt = a * Ti;
  v[6] += q.g0 * wgt;
  v[7] += q.g1 * wgt;
  v[8] += q.g2 * wgt;
  q.S += gc * wgt;
  q.T = Ti;
  if (raw > b.alpha_max) ga = 0.0f;       // clamped: alpha does not move
  v[5] += ga * G;
  const float gd2 = -0.5f * ga * co.w * G;
  v[2] += gd2 * dx * dx;
  v[3] += gd2 * 2.0f * dx * dy;
  v[4] += gd2 * dy * dy;
  v[0] += -2.0f * gd2 * (co.x * dx + co.y * dy);
  v[1] += -2.0f * gd2 * (co.y * dx + co.z * dy);
  return true;
}

// gacc per Gaussian: 12 floats, the 9 of grad_step then 3 unused
__global__ void __launch_bounds__(kRastThreads) rasterise_bwd(Blend b, int W, int H, const uint2* __restrict__ ranges,
                                                             const uint32_t* __restrict__ pair_id,
                                                             const float4* __restrict__ conic_o,
                                                             const float4* __restrict__ xy,
                                                             const float4* __restrict__ rgb,
                                                             const float* __restrict__ final_T,
                                                             const uint32_t* __restrict__ n_contrib,
                                                             const float* __restrict__ grad_image,
                                                             float4* __restrict__ gacc) {
  pdl_release();   // the projection backward may launch; it waits for this grid in its pdl_wait
  __shared__ float4 s_co[kRastThreads];
  __shared__ float4 s_xy[kRastThreads];
  __shared__ float4 s_rgb[kRastThreads];
  __shared__ uint32_t s_id[kRastThreads];
  __shared__ uint32_t s_max;
  const TileGeom g = tile_geom(b);
  const int lane = threadIdx.x & 31;
  BwdPix q = bwd_pixel(g.px, g.py, W, H, b, final_T, n_contrib, grad_image);
  const uint2 range = ranges[blockIdx.x];
  if (threadIdx.x == 0) s_max = 0;
  __syncthreads();
  atomicMax(&s_max, q.last);
  __syncthreads();
  const uint32_t max_last = s_max;
  const uint32_t warp_last = __reduce_max_sync(0xffffffffu, q.last);
  for (uint32_t hi = max_last; hi > 0;) {
    const uint32_t lo = hi > (uint32_t)kRastThreads ? hi - kRastThreads : 0u;
    __syncthreads();
    const uint32_t i = lo + threadIdx.x;
    if (i < hi) {
      const uint32_t id = pair_id[range.x + i];
      s_id[threadIdx.x] = id;
      s_co[threadIdx.x] = conic_o[id];
      s_xy[threadIdx.x] = xy[id];
      s_rgb[threadIdx.x] = rgb[id];
    }
    __syncthreads();
    for (int j = (int)(hi - lo) - 1; j >= 0; --j) {
      const uint32_t jidx = lo + j;
      const float4 m = s_xy[j];
      // warp-uniform: the support box misses the block, or no lane got this far
      if (jidx >= warp_last || box_misses(m, g)) continue;
      float v[16] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const bool hit = grad_step(q, jidx, s_co[j], m, s_rgb[j], b, v);
      const uint32_t hits = __ballot_sync(0xffffffffu, hit);
      if (hits) {
        float* gq = reinterpret_cast<float*>(gacc + 3 * (int64_t)s_id[j]);
        if (__popc(hits) <= kFewLanes) {
          // a few lanes: each adds its own nine values (cheaper than the reduction)
          if (hit) {
#pragma unroll
            for (int k = 0; k < 9; ++k) atomicAdd(gq + k, v[k]);
          }
        } else {
          const float total = warp_transpose_sum16(v, lane);
          const int k = (lane >> 1) & 15;
          if ((lane & 1) == 0 && k < 9) atomicAdd(gq + k, total);
        }
      }
    }
    hi = lo;
  }
}

template <int DEG>
__global__ void __launch_bounds__(kProjThreads) project_bwd_kernel(
    Cam c, Blend b, int64_t N, const float* __restrict__ means, const float* __restrict__ cov,
    const float* __restrict__ opacity, const float* __restrict__ colours, const float4* __restrict__ gacc,
    float* __restrict__ grad_means, float* __restrict__ grad_cov, float* __restrict__ grad_opacity,
    float* __restrict__ grad_colours) {
  pdl_wait();
  pdl_release();
  using CT = ColourTile<DEG>;
  constexpr int K = DEG < 0 ? 1 : (DEG + 1) * (DEG + 1);
  // the tile's SH rows; each thread overwrites its own row with its SH
  // gradient, which is then added to grad_colours row-coalesced
  __shared__ float s_col[CT::kStaged ? kProjThreads * CT::kPitch : 1];
  for (int64_t n0 = (int64_t)blockIdx.x * kProjThreads; n0 < N; n0 += (int64_t)gridDim.x * kProjThreads) {
    const int nb = (int)min((int64_t)kProjThreads, N - n0);
    if (CT::kStaged) {
      __syncthreads();
      stage_rows<DEG>(colours, n0, nb, s_col);
      __syncthreads();
    }
    const int64_t n = n0 + threadIdx.x;
    bool live = threadIdx.x < nb;
    Proj p;
    float o = 0.f;
    const float* mu = means + n * b.mean_stride;
    if (live) {
      project_one(c, b.lowpass, mu, cov + 6 * n, p);
      o = __ldg(opacity + n);
      live = p.visible && o >= b.alpha_min;   // otherwise never blended: zero gradient
    }
    float* krow = s_col + threadIdx.x * CT::kPitch;
    if (live) {
      const float4 q0 = gacc[3 * n], q1 = gacc[3 * n + 1], q2 = gacc[3 * n + 2];
      const float gx = q0.x, gy = q0.y, ga = q0.z, gb = q0.w, gc = q1.x;
      const float grgb[3] = {q1.z, q1.w, q2.x};
      if (grad_opacity) grad_opacity[n] += q1.y;
      // conic (a, b, c) = (C, -B, A) / det, det = A C - B^2
      const float A = p.A, B = p.B, C = p.C;
      const float id = 1.0f / p.det, id2 = id * id;
      const float gA = (-ga * C * C + gb * B * C - gc * B * B) * id2;
      const float gB = (2.0f * ga * B * C + 2.0f * gc * A * B) * id2 - gb * (id + 2.0f * B * B * id2);
      const float gC = (-ga * B * B + gb * A * B - gc * A * A) * id2;
      // G2 = [[gA, gB/2], [gB/2, gC]]: dL/dSigma = T^T G2 T
      float U0[3], U1[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        U0[k] = gA * p.T0[k] + 0.5f * gB * p.T1[k];
        U1[k] = 0.5f * gB * p.T0[k] + gC * p.T1[k];
      }
      if (grad_cov) {
        float* gcv = grad_cov + 6 * n;
        gcv[0] += p.T0[0] * U0[0] + p.T1[0] * U1[0];
        gcv[1] += 2.0f * (p.T0[0] * U0[1] + p.T1[0] * U1[1]);
        gcv[2] += 2.0f * (p.T0[0] * U0[2] + p.T1[0] * U1[2]);
        gcv[3] += p.T0[1] * U0[1] + p.T1[1] * U1[1];
        gcv[4] += 2.0f * (p.T0[1] * U0[2] + p.T1[1] * U1[2]);
        gcv[5] += p.T0[2] * U0[2] + p.T1[2] * U1[2];
      }
      // dL/d(J W) = 2 G2 (J W) Sigma; dL/dJ = that times W^T
      float gT0[3], gT1[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        gT0[k] = 2.0f * (gA * p.M0[k] + 0.5f * gB * p.M1[k]);
        gT1[k] = 2.0f * (0.5f * gB * p.M0[k] + gC * p.M1[k]);
      }
      const float gJ00 = gT0[0] * c.R[0] + gT0[1] * c.R[1] + gT0[2] * c.R[2];
      const float gJ02 = gT0[0] * c.R[6] + gT0[1] * c.R[7] + gT0[2] * c.R[8];
      const float gJ11 = gT1[0] * c.R[3] + gT1[1] * c.R[4] + gT1[2] * c.R[5];
      const float gJ12 = gT1[0] * c.R[6] + gT1[1] * c.R[7] + gT1[2] * c.R[8];
      const float x = p.xc[0], y = p.xc[1], z = p.xc[2];
      const float iz = 1.0f / z, iz2 = iz * iz, iz3 = iz2 * iz;
      float gxc[3];
      gxc[0] = -c.fx * iz2 * gJ02 + gx * c.fx * iz;
      gxc[1] = -c.fy * iz2 * gJ12 + gy * c.fy * iz;
      gxc[2] = -c.fx * iz2 * gJ00 + 2.0f * c.fx * x * iz3 * gJ02 - c.fy * iz2 * gJ11 + 2.0f * c.fy * y * iz3 * gJ12 -
               gx * c.fx * x * iz2 - gy * c.fy * y * iz2;
      float gmu[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) gmu[k] = c.R[k] * gxc[0] + c.R[3 + k] * gxc[1] + c.R[6 + k] * gxc[2];
      if (DEG < 0) {
        if (grad_colours)
          for (int ch = 0; ch < 3; ++ch) grad_colours[3 * n + ch] += grgb[ch];
      } else {
        float d[3], nv, Y[16];
        view_dir(c, mu, d, nv);
        sh_basis(DEG, d[0], d[1], d[2], Y);
        float pre[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < K; ++i)
#pragma unroll
          for (int ch = 0; ch < 3; ++ch) pre[ch] += Y[i] * krow[3 * i + ch];
        float gp[3];
#pragma unroll
        for (int ch = 0; ch < 3; ++ch) gp[ch] = pre[ch] >= 0.0f ? grgb[ch] : 0.0f;
        float gd[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < K; ++i) {
          float w = 0.f;
#pragma unroll
          for (int ch = 0; ch < 3; ++ch) {
            w += gp[ch] * krow[3 * i + ch];
            krow[3 * i + ch] = Y[i] * gp[ch];   // this row now holds the SH gradient
          }
          sh_grad_acc(i, w, d[0], d[1], d[2], gd);
        }
        // d = v / |v|: dL/dv = (I - d d^T) dL/dd / |v|
        const float dot = gd[0] * d[0] + gd[1] * d[1] + gd[2] * d[2];
        const float inv = 1.0f / fmaxf(nv, 1e-30f);
#pragma unroll
        for (int k2 = 0; k2 < 3; ++k2) gmu[k2] += (gd[k2] - d[k2] * dot) * inv;
      }
      if (grad_means)
#pragma unroll
        for (int k2 = 0; k2 < 3; ++k2) grad_means[3 * n + k2] += gmu[k2];
    } else if (CT::kStaged && threadIdx.x < nb) {
#pragma unroll
      for (int i = 0; i < CT::kRow; ++i) krow[i] = 0.0f;
    }
    if (CT::kStaged && grad_colours) {
      __syncthreads();
      constexpr int R = CT::kRow, P = CT::kPitch;
      float* g = grad_colours + n0 * R;
      for (int e = threadIdx.x; e < nb * R; e += kProjThreads) g[e] += s_col[(e / R) * P + e % R];
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct StateLayout {
  size_t header, conic_o, xy, rgb, rect, ntiles, dkey, dkey_b, dperm, dperm_b, cnt, offs;
  size_t pair_tile, pair_id, pair_tile_b, pair_id_b, scratch, ranges, final_T, n_contrib, gacc, total;
};

int tiles_of(int side) { return (side + kTileSide - 1) / kTileSide; }

StateLayout state_layout(int64_t N, int W, int H, int64_t P) {
  using radix::align256;
  StateLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += align256(bytes);
    return at;
  };
  const size_t n = (size_t)std::max<int64_t>(N, 1), p = (size_t)std::max<int64_t>(P, 1);
  const size_t tiles = (size_t)tiles_of(W) * tiles_of(H);
  L.header = take(256);
  L.conic_o = take(n * 16);
  L.xy = take(n * 16);
  L.rgb = take(n * 16);
  L.rect = take(n * 8);
  L.ntiles = take(n * 4);
  L.dkey = take(n * 4);
  L.dkey_b = take(n * 4);
  L.dperm = take(n * 4);
  L.dperm_b = take(n * 4);
  L.cnt = take(n * 4);
  L.offs = take(n * 4);
  L.pair_tile = take(p * 4);
  L.pair_id = take(p * 4);
  L.pair_tile_b = take(p * 4);
  L.pair_id_b = take(p * 4);
  L.scratch = take(std::max({radix::scratch_bytes((int64_t)n), radix::scratch_bytes((int64_t)p),
                             radix::exclusive_scan_scratch((int64_t)n)}));
  L.ranges = take(tiles * 8);
  L.final_T = take((size_t)W * H * 4);
  L.n_contrib = take((size_t)W * H * 4);
  L.gacc = take(n * 48);
  L.total = o;
  return L;
}

int validate_render(const spin4d_camera* cam, const spin4d_render_desc* d, int64_t N, int64_t max_pairs) {
  if (!cam || !d) return SPIN4D_ERR_INVALID;
  if (cam->width < 1 || cam->height < 1 || cam->width > SPIN4D_MAX_IMAGE_SIDE ||
      cam->height > SPIN4D_MAX_IMAGE_SIDE)
    return SPIN4D_ERR_INVALID;
  for (int i = 0; i < 12; ++i)
    if (!isfinite(cam->view[i])) return SPIN4D_ERR_INVALID;
  if (!(cam->fx > 0.f) || !(cam->fy > 0.f) || !isfinite(cam->fx) || !isfinite(cam->fy) || !isfinite(cam->cx) ||
      !isfinite(cam->cy) || !(cam->z_near > 0.f) || !isfinite(cam->z_near))
    return SPIN4D_ERR_INVALID;
  if (d->sh_degree < -1 || d->sh_degree > 3 || !(d->lowpass >= 0.f) || !isfinite(d->lowpass) ||
      !(d->alpha_max > 0.f && d->alpha_max < 1.f) || !(d->alpha_min >= 0.f && d->alpha_min < d->alpha_max) ||
      !(d->t_stop >= 0.f && d->t_stop < 1.f) || (d->mean_stride != 3 && d->mean_stride != 4) || d->reserved != 0)
    return SPIN4D_ERR_INVALID;
  for (int i = 0; i < 3; ++i)
    if (!isfinite(d->background[i])) return SPIN4D_ERR_INVALID;
  if (N < 0 || N > SPIN4D_MAX_RENDER_GAUSSIANS || max_pairs < 0 || max_pairs > SPIN4D_MAX_RENDER_PAIRS)
    return SPIN4D_ERR_INVALID;
  return SPIN4D_OK;
}

void make_params(const spin4d_camera* cam, const spin4d_render_desc* d, Cam& c, Blend& b) {
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 3; ++j) c.R[3 * i + j] = cam->view[4 * i + j];
    c.t[i] = cam->view[4 * i + 3];
  }
  for (int j = 0; j < 3; ++j) {   // camera centre -R^T t, in double
    double s = 0.0;
    for (int i = 0; i < 3; ++i) s -= (double)cam->view[4 * i + j] * (double)cam->view[4 * i + 3];
    c.campos[j] = (float)s;
  }
  c.fx = cam->fx;
  c.fy = cam->fy;
  c.cx = cam->cx;
  c.cy = cam->cy;
  c.W = cam->width;
  c.H = cam->height;
  c.z_near = cam->z_near;
  b.sh_degree = d->sh_degree;
  b.n_coef = d->sh_degree < 0 ? 1 : (d->sh_degree + 1) * (d->sh_degree + 1);
  b.mean_stride = d->mean_stride;
  b.lowpass = d->lowpass;
  b.alpha_max = d->alpha_max;
  b.alpha_min = d->alpha_min;
  b.t_stop = d->t_stop;
  for (int i = 0; i < 3; ++i) b.bg[i] = d->background[i];
  b.log_amin = d->alpha_min > 0.f ? logf(d->alpha_min) : 0.f;
  b.tiles_x = tiles_of(cam->width);
  b.tiles_y = tiles_of(cam->height);
}

int tile_sort_passes(int n_tiles) {
  int bits = 0;
  while ((1 << bits) < n_tiles) ++bits;
  return (bits + 7) / 8;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

int check_inputs(int64_t N, const float* means, const float* cov, const float* opacity, const float* colours,
                 void* state, size_t state_bytes, size_t need) {
  if (N > 0 && (!means || !cov || !opacity || !colours)) return SPIN4D_ERR_INVALID;
  if (!state || !aligned(state, 256) || state_bytes < need) return SPIN4D_ERR_INVALID;
  if (N > 0 && (!aligned(means, 4) || !aligned(cov, 4) || !aligned(opacity, 4) || !aligned(colours, 4)))
    return SPIN4D_ERR_INVALID;
  return SPIN4D_OK;
}

}  // namespace
}  // namespace spin4d

using namespace spin4d;

extern "C" size_t spin4d_render_state_bytes(int64_t N, int width, int height, int64_t max_pairs) {
  if (N < 0 || N > SPIN4D_MAX_RENDER_GAUSSIANS || width < 1 || height < 1 || width > SPIN4D_MAX_IMAGE_SIDE ||
      height > SPIN4D_MAX_IMAGE_SIDE || max_pairs < 0 || max_pairs > SPIN4D_MAX_RENDER_PAIRS)
    return 0;
  return state_layout(N, width, height, max_pairs).total;
}

extern "C" int spin4d_render_fwd(const spin4d_camera* cam, const spin4d_render_desc* desc, int64_t N,
                                 const float* means, const float* cov, const float* opacity, const float* colours,
                                 float* image, float* final_T, void* state, size_t state_bytes, int64_t max_pairs,
                                 spin4d_stream_t stream) {
  SPIN4D_CHECK(validate_render(cam, desc, N, max_pairs));
  const StateLayout L = state_layout(N, cam->width, cam->height, max_pairs);
  SPIN4D_CHECK(check_inputs(N, means, cov, opacity, colours, state, state_bytes, L.total));
  if (!image || !aligned(image, 4) || (final_T && !aligned(final_T, 4))) return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_render_fwd")) return SPIN4D_ERR_INJECTED;
  cudaStream_t s = (cudaStream_t)stream;
  Cam c;
  Blend b;
  make_params(cam, desc, c, b);
  const int n_tiles = b.tiles_x * b.tiles_y;
  uint32_t* header = at<uint32_t>(state, L.header);
  SPIN4D_CHECK(cuda_status(cudaMemsetAsync(header, 0, 256, s)));
  SPIN4D_CHECK(cuda_status(cudaMemsetAsync(at<void>(state, L.ranges), 0, (size_t)n_tiles * 8, s)));
  uint32_t* pair_tile = at<uint32_t>(state, L.pair_tile);
  uint32_t* pair_id = at<uint32_t>(state, L.pair_id);
  if (N > 0) {
    const int blocks = persistent_blocks((N + 255) / 256, 8);
    const int pblocks = persistent_blocks((N + kProjThreads - 1) / kProjThreads, 8);
#define SPIN4D_PROJECT(DEG)                                                                                    \
  project_kernel<DEG><<<pblocks, kProjThreads, 0, s>>>(c, b, N, means, cov, opacity, colours,                \
                                                       at<float4>(state, L.conic_o), at<float4>(state, L.xy), \
                                                       at<float4>(state, L.rgb), at<uint2>(state, L.rect),    \
                                                       at<uint32_t>(state, L.ntiles), at<uint32_t>(state, L.dkey))
    switch (b.sh_degree) {
      case -1: SPIN4D_PROJECT(-1); break;
      case 0: SPIN4D_PROJECT(0); break;
      case 1: SPIN4D_PROJECT(1); break;
      case 2: SPIN4D_PROJECT(2); break;
      default: SPIN4D_PROJECT(3); break;
    }
#undef SPIN4D_PROJECT
    SPIN4D_CHECK(launch_status());
    uint32_t* dkey = at<uint32_t>(state, L.dkey);
    uint32_t* dperm = at<uint32_t>(state, L.dperm);
    radix::sort_pairs(dkey, dperm, at<uint32_t>(state, L.dkey_b), at<uint32_t>(state, L.dperm_b), true, N, nullptr, 4,
                      at<void>(state, L.scratch), s);
    uint32_t* cnt = at<uint32_t>(state, L.cnt);
    uint32_t* offs = at<uint32_t>(state, L.offs);
    launch_pdl(counts_in_order, blocks, 256, 0, s, dperm, at<uint32_t>(state, L.ntiles), N, cnt, header);
    launch_pdl(clamp_pair_count, 1, 1, 0, s, header, (uint32_t)max_pairs);
    radix::exclusive_scan(cnt, N, offs, at<void>(state, L.scratch), s);
    launch_pdl(emit_pairs, blocks, 256, 0, s, dperm, cnt, offs, at<uint2>(state, L.rect), N, b.tiles_x, header,
               pair_tile, pair_id);
    SPIN4D_CHECK(launch_status());
    const int passes = tile_sort_passes(n_tiles);
    if (passes > 0 && max_pairs > 0) {
      const bool in_place = radix::sort_pairs(pair_tile, pair_id, at<uint32_t>(state, L.pair_tile_b),
                                              at<uint32_t>(state, L.pair_id_b), false, max_pairs, header + 2, passes,
                                              at<void>(state, L.scratch), s);
      if (!in_place) {
        pair_tile = at<uint32_t>(state, L.pair_tile_b);
        pair_id = at<uint32_t>(state, L.pair_id_b);
      }
    }
    if (max_pairs > 0)
      launch_pdl(tile_ranges_kernel, persistent_blocks((max_pairs + 255) / 256, 8), 256, 0, s, pair_tile,
                 (const uint32_t*)header, max_pairs, (uint32_t)n_tiles, at<uint2>(state, L.ranges));
    SPIN4D_CHECK(launch_status());
  }
  launch_pdl(rasterise_fwd, n_tiles, kRastThreads, 0, s, b, c.W, c.H, (const uint2*)at<uint2>(state, L.ranges),
             (const uint32_t*)pair_id, (const float4*)at<float4>(state, L.conic_o),
             (const float4*)at<float4>(state, L.xy), (const float4*)at<float4>(state, L.rgb), image,
             at<float>(state, L.final_T), at<uint32_t>(state, L.n_contrib), final_T);
  return launch_status();
}

extern "C" int spin4d_render_bwd(const spin4d_camera* cam, const spin4d_render_desc* desc, int64_t N,
                                 const float* means, const float* cov, const float* opacity, const float* colours,
                                 const float* grad_image, void* state, size_t state_bytes, int64_t max_pairs,
                                 float* grad_means, float* grad_cov, float* grad_opacity, float* grad_colours,
                                 spin4d_stream_t stream) {
  SPIN4D_CHECK(validate_render(cam, desc, N, max_pairs));
  const StateLayout L = state_layout(N, cam->width, cam->height, max_pairs);
  SPIN4D_CHECK(check_inputs(N, means, cov, opacity, colours, state, state_bytes, L.total));
  if (!grad_image || !aligned(grad_image, 4)) return SPIN4D_ERR_INVALID;
  for (const float* g : {grad_means, grad_cov, grad_opacity, grad_colours})
    if (g && !aligned(g, 4)) return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_render_bwd")) return SPIN4D_ERR_INJECTED;
  if (N == 0) return SPIN4D_OK;
  cudaStream_t s = (cudaStream_t)stream;
  Cam c;
  Blend b;
  make_params(cam, desc, c, b);
  const int n_tiles = b.tiles_x * b.tiles_y;
  float4* gacc = at<float4>(state, L.gacc);
  SPIN4D_CHECK(cuda_status(cudaMemsetAsync(gacc, 0, (size_t)N * 48, s)));
  const int passes = tile_sort_passes(n_tiles);
  const bool in_b = passes > 0 && max_pairs > 0 && (passes % 2) == 1;
  const uint32_t* pair_id = at<uint32_t>(state, in_b ? L.pair_id_b : L.pair_id);
  rasterise_bwd<<<n_tiles, kRastThreads, 0, s>>>(b, c.W, c.H, at<uint2>(state, L.ranges), pair_id,
                                                at<float4>(state, L.conic_o), at<float4>(state, L.xy),
                                                at<float4>(state, L.rgb), at<float>(state, L.final_T),
                                                at<uint32_t>(state, L.n_contrib), grad_image, gacc);
  SPIN4D_CHECK(launch_status());
  const int pblocks = persistent_blocks((N + kProjThreads - 1) / kProjThreads, 8);
#define SPIN4D_PROJECT_BWD(DEG)                                                                                 \
  launch_pdl(project_bwd_kernel<DEG>, pblocks, kProjThreads, 0, s, c, b, N, means, cov, opacity, colours,          \
             (const float4*)gacc, grad_means, grad_cov, grad_opacity, grad_colours)
  switch (b.sh_degree) {
    case -1: SPIN4D_PROJECT_BWD(-1); break;
    case 0: SPIN4D_PROJECT_BWD(0); break;
    case 1: SPIN4D_PROJECT_BWD(1); break;
    case 2: SPIN4D_PROJECT_BWD(2); break;
    default: SPIN4D_PROJECT_BWD(3); break;
  }
#undef SPIN4D_PROJECT_BWD
  return launch_status();
}
