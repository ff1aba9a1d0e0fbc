// Device-side building blocks shared by the spin4d kernels.
//
// Normalisation (SPIN-4DGS section 3.3, Eq. 7-8) and the interpolation-cell
// decision run in fp32 with every operation explicitly rounded
// (__fmul_rn/__fadd_rn/__fdiv_rn/__fsqrt_rn) so that no fused multiply-add
// changes which grid cell a position falls into: the corner indices are an
// integer result and must not depend on compiler contraction choices.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "spin4d.h"

namespace spin4d {

constexpr uint32_t kPrimeY = 2654435761u;
constexpr uint32_t kPrimeZ = 805459861u;
constexpr uint32_t kPrimeT = 3674653429u;
constexpr int kHeadRows = 11;
constexpr float kScaleClip = 20.0f;
constexpr float kNormFloor = 1e-12f;

// Host-derived per-level constants, passed by value to every grid kernel.
struct GridParams {
  int L, F, log2_T, table_dtype;
  uint32_t mask;          // T - 1
  uint32_t dense_bits;    // bit l set when level l is indexed densely
  uint32_t flags;
  float t_min, span;      // span = fl32(t_max - t_min)
  int max_cell[SPIN4D_MAX_LEVELS][4];       // res - 2
  float scale[SPIN4D_MAX_LEVELS][4];        // (float)(res - 1)
  uint32_t stride[SPIN4D_MAX_LEVELS][4];    // dense strides 1, rx, rx*ry, rx*ry*rz
};

__device__ __forceinline__ float clamp01(float v) {
  // fmaxf(NaN, 0) = 0, so a NaN coordinate lands on 0 (same reading as the oracle).
  return fminf(fmaxf(v, 0.0f), 1.0f);
}

// Eq. 7 (Mip-NeRF contraction, then /4 + 1/2) and Eq. 8 (time), pinned order.
__device__ __forceinline__ void normalise_position(float4 p, const GridParams& g, float xt[4]) {
  if (g.flags & SPIN4D_INPUT_NORMALISED) {
    xt[0] = clamp01(p.x); xt[1] = clamp01(p.y); xt[2] = clamp01(p.z); xt[3] = clamp01(p.w);
    return;
  }
  float n2 = __fadd_rn(__fadd_rn(__fmul_rn(p.x, p.x), __fmul_rn(p.y, p.y)), __fmul_rn(p.z, p.z));
  float n = __fsqrt_rn(n2);
  float cx = p.x, cy = p.y, cz = p.z;
  if (!(n <= 1.0f)) {
    float k = __fsub_rn(2.0f, __fdiv_rn(1.0f, n));
    cx = __fmul_rn(k, __fdiv_rn(p.x, n));
    cy = __fmul_rn(k, __fdiv_rn(p.y, n));
    cz = __fmul_rn(k, __fdiv_rn(p.z, n));
  }
  xt[0] = clamp01(__fadd_rn(__fmul_rn(cx, 0.25f), 0.5f));
  xt[1] = clamp01(__fadd_rn(__fmul_rn(cy, 0.25f), 0.5f));
  xt[2] = clamp01(__fadd_rn(__fmul_rn(cz, 0.25f), 0.5f));
  xt[3] = clamp01(__fdiv_rn(__fsub_rn(p.w, g.t_min), g.span));
}

// The cell of a normalised position at level l: lower vertex and fraction.
__device__ __forceinline__ void level_cell(const float xt[4], const GridParams& g, int l,
                                           uint32_t base[4], float frac[4]) {
#pragma unroll
  for (int d = 0; d < 4; ++d) {
    float p = __fmul_rn(xt[d], g.scale[l][d]);
    int i = (int)floorf(p);
    i = min(max(i, 0), g.max_cell[l][d]);
    base[d] = (uint32_t)i;
    frac[d] = __fsub_rn(p, (float)i);   // exact
  }
}

// Table index of the 16 corners (bit d of c selects base_d + 1).
// ---------------------------------------------------------------------------
// Checked build (compiled with SPIN4D_CHECKED): device-side bounds checks on
// every table index and HexPlane cell.  A failed check records itself in this
// translation unit's bounds word and the access is redirected to a valid
// address (entry 0 of the level, the plane's first row): nothing traps, and
// spin4d_check_device_errors reports SPIN4D_ERR_BOUNDS.  Each translation
// unit registers a reader of its word with the library at load time.
// ---------------------------------------------------------------------------
#ifdef SPIN4D_CHECKED
static __device__ int g_bounds_error = 0;
__device__ __forceinline__ bool bounds_ok(bool ok) {
  if (!ok) atomicExch(&g_bounds_error, 1);
  return ok;
}
int register_bounds_word(int (*reader)(int clear));   // api.cu
static int read_bounds_word(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_bounds_error, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_bounds_error, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}
static const int g_bounds_registered = register_bounds_word(read_bounds_word);
#endif

__device__ __forceinline__ void level_indices(const uint32_t base[4], const GridParams& g, int l,
                                              uint32_t idx[16]) {
  if ((g.dense_bits >> l) & 1u) {
    const uint32_t sy = g.stride[l][1], sz = g.stride[l][2], st = g.stride[l][3];
    uint32_t b0 = base[0] + base[1] * sy + base[2] * sz + base[3] * st;
#pragma unroll
    for (int c = 0; c < 16; ++c)
      idx[c] = b0 + (c & 1) + ((c >> 1) & 1) * sy + ((c >> 2) & 1) * sz + ((c >> 3) & 1) * st;
  } else {
    uint32_t hx[2] = {base[0], base[0] + 1u};
    uint32_t hy0 = base[1] * kPrimeY, hz0 = base[2] * kPrimeZ, ht0 = base[3] * kPrimeT;
    uint32_t hy[2] = {hy0, hy0 + kPrimeY};
    uint32_t hz[2] = {hz0, hz0 + kPrimeZ};
    uint32_t ht[2] = {ht0, ht0 + kPrimeT};
#pragma unroll
    for (int c = 0; c < 16; ++c)
      idx[c] = (hx[c & 1] ^ hy[(c >> 1) & 1] ^ hz[(c >> 2) & 1] ^ ht[(c >> 3) & 1]) & g.mask;
  }
#ifdef SPIN4D_CHECKED
#pragma unroll
  for (int c = 0; c < 16; ++c)
    if (!bounds_ok(idx[c] <= g.mask)) idx[c] = 0;   // index < T
#endif
}

// Quadrilinear weights prod_d (bit_d ? w_d : 1 - w_d), fp32.
__device__ __forceinline__ void level_weights(const float frac[4], float w[16]) {
  float wx[2] = {1.0f - frac[0], frac[0]};
  float wy[2] = {1.0f - frac[1], frac[1]};
  float wz[2] = {1.0f - frac[2], frac[2]};
  float wt[2] = {1.0f - frac[3], frac[3]};
  float wxy[4], wzt[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    wxy[i] = wx[i & 1] * wy[i >> 1];
    wzt[i] = wz[i & 1] * wt[i >> 1];
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) w[c] = wxy[c & 3] * wzt[c >> 2];
}

// ---------------------------------------------------------------------------
// Table entry loads: F features of entry e, converted to fp32.
// ---------------------------------------------------------------------------
template <typename T, int F> struct Entry;

template <int F> struct Entry<float, F> {
  static __device__ __forceinline__ void load(const float* __restrict__ tab, uint32_t e, float v[F]) {
    const float* p = tab + (size_t)e * F;
    if constexpr (F == 1) {
      v[0] = __ldg(p);
    } else if constexpr (F == 2) {
      float2 a = __ldg(reinterpret_cast<const float2*>(p));
      v[0] = a.x; v[1] = a.y;
    } else {
#pragma unroll
      for (int q = 0; q < F / 4; ++q) {
        float4 a = __ldg(reinterpret_cast<const float4*>(p) + q);
        v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
      }
    }
  }
};

template <int F> struct Entry<__half, F> {
  static __device__ __forceinline__ void load(const __half* __restrict__ tab, uint32_t e, float v[F]) {
    const __half* p = tab + (size_t)e * F;
    if constexpr (F == 1) {
      v[0] = __half2float(__ldg(p));
    } else if constexpr (F == 2) {
      unsigned int u = __ldg(reinterpret_cast<const unsigned int*>(p));
      float2 a = __half22float2(*reinterpret_cast<__half2*>(&u));
      v[0] = a.x; v[1] = a.y;
    } else if constexpr (F == 4) {
      uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
      float2 a = __half22float2(*reinterpret_cast<__half2*>(&u.x));
      float2 b = __half22float2(*reinterpret_cast<__half2*>(&u.y));
      v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    } else {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
      unsigned int w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 a = __half22float2(*reinterpret_cast<__half2*>(&w4[q]));
        v[2 * q] = a.x; v[2 * q + 1] = a.y;
      }
    }
  }
};

// Encode one level: acc[f] = sum_c w_c * table_l[idx_c][f].
template <typename T, int F>
__device__ __forceinline__ void encode_level(const float xt[4], const GridParams& g, int l,
                                             const T* __restrict__ tables, float acc[F]) {
  uint32_t base[4];
  float frac[4];
  level_cell(xt, g, l, base, frac);
  uint32_t idx[16];
  level_indices(base, g, l, idx);
  float w[16];
  level_weights(frac, w);
  const T* tab = tables + ((size_t)l << g.log2_T) * F;
#pragma unroll
  for (int f = 0; f < F; ++f) acc[f] = 0.0f;
  float v[16][F];
#pragma unroll
  for (int c = 0; c < 16; ++c) Entry<T, F>::load(tab, idx[c], v[c]);
#pragma unroll
  for (int c = 0; c < 16; ++c)
#pragma unroll
    for (int f = 0; f < F; ++f) acc[f] = fmaf(w[c], v[c][f], acc[f]);
}

// Encode one level of an fp16 table, x-neighbours paired: corners c (x bit 0)
// and c+1 (x bit 1) usually fall in the same 16-byte group of G = 8/F entries
// (dense levels: consecutive entries; hashed levels: x enters the hash with
// prime 1, so x and x+1 differ only in the low bits unless a carry crosses
// the group).  One 16-byte load then serves both corners; only lanes whose
// pair straddles two groups issue a second load.  Four pairs per batch bound
// the registers held by loads in flight.
template <int F>
__device__ __forceinline__ uint32_t group_word(const uint4& v, uint32_t i) {
  // word holding entry i of the group (F = 2: one word per entry)
  return (i & 2u) ? ((i & 1u) ? v.w : v.z) : ((i & 1u) ? v.y : v.x);
}

template <int F>
__device__ __forceinline__ void accumulate_entry(const uint4& v, uint32_t i, float wgt, float acc[F]) {
  if constexpr (F == 2) {
    uint32_t u = group_word<F>(v, i);
    float2 a = __half22float2(*reinterpret_cast<__half2*>(&u));
    acc[0] = fmaf(wgt, a.x, acc[0]);
    acc[1] = fmaf(wgt, a.y, acc[1]);
  } else if constexpr (F == 4) {
    uint32_t u0 = (i & 1u) ? v.z : v.x, u1 = (i & 1u) ? v.w : v.y;
    float2 a = __half22float2(*reinterpret_cast<__half2*>(&u0));
    float2 b = __half22float2(*reinterpret_cast<__half2*>(&u1));
    acc[0] = fmaf(wgt, a.x, acc[0]);
    acc[1] = fmaf(wgt, a.y, acc[1]);
    acc[2] = fmaf(wgt, b.x, acc[2]);
    acc[3] = fmaf(wgt, b.y, acc[3]);
  }
}

template <int F>
__device__ __forceinline__ void encode_level_f16_paired(const float xt[4], const GridParams& g, int l,
                                                        const __half* __restrict__ tables, float acc[F]) {
  static_assert(F == 2 || F == 4, "paired gather covers F = 2 and 4");
  constexpr uint32_t G = 8 / F;   // entries per 16-byte group
  uint32_t base[4];
  float frac[4];
  level_cell(xt, g, l, base, frac);
  uint32_t idx[16];
  level_indices(base, g, l, idx);
  float w[16];
  level_weights(frac, w);
  const uint4* tab = reinterpret_cast<const uint4*>(tables + ((size_t)l << g.log2_T) * F);
#pragma unroll
  for (int f = 0; f < F; ++f) acc[f] = 0.0f;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint4 v0[4], v1[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int c = 2 * (4 * b + p);
      const uint32_t g0 = idx[c] / G, g1 = idx[c + 1] / G;
      v0[p] = __ldg(tab + g0);
      v1[p] = v0[p];
      if (g1 != g0) v1[p] = __ldg(tab + g1);
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int c = 2 * (4 * b + p);
      accumulate_entry<F>(v0[p], idx[c] % G, w[c], acc);
      accumulate_entry<F>(v1[p], idx[c + 1] % G, w[c + 1], acc);
    }
  }
}

// ---------------------------------------------------------------------------
// Position gradient (trainable Gaussian means).
// ---------------------------------------------------------------------------
// gx[d] += d<dz, z_l>/dx~_d for one level: inside the position's cell
// z_l = sum_c W_c e_c with W_c = prod_d (bit_d ? w_d : 1 - w_d) and
// w_d = x~_d (res_d - 1) - base_d, so the derivative is
// (res_d - 1) sum_c (dz . e_c) dW_c/dw_d,
// dW_c/dw_d = (bit_d ? 1 : -1) prod_{e != d} (bit_e ? w_e : 1 - w_e).
template <typename T, int F>
__device__ __forceinline__ void level_position_grad(const float xt[4], const GridParams& g, int l,
                                                    const T* __restrict__ tables, const float dz[F], float gx[4]) {
  uint32_t base[4];
  float frac[4];
  level_cell(xt, g, l, base, frac);
  uint32_t idx[16];
  level_indices(base, g, l, idx);
  const T* tab = tables + ((size_t)l << g.log2_T) * F;
  float s[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    float v[F];
    Entry<T, F>::load(tab, idx[c], v);
    float a = 0.0f;
#pragma unroll
    for (int f = 0; f < F; ++f) a = fmaf(dz[f], v[f], a);
    s[c] = a;
  }
#pragma unroll
  for (int d = 0; d < 4; ++d) {
    float acc = 0.0f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      float p = ((c >> d) & 1) ? s[c] : -s[c];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (e != d) p *= ((c >> e) & 1) ? frac[e] : 1.0f - frac[e];
      acc += p;
    }
    gx[d] = fmaf(acc, g.scale[l][d], gx[d]);
  }
}

// Gradient w.r.t. the raw spatial position from the gradient w.r.t. the
// normalised coordinates: Eq. 7's Jacobian, I/4 inside the unit ball and
// (g I + h mu mu^T)/4 outside with g = 2/n - 1/n^2, h = 2/n^4 - 2/n^3 (the
// contracted point 2 - 1/n along the ray of mu).  For normalised input, the
// clamp to [0, 1] alone: the gradient passes where the input was in range.
__device__ __forceinline__ void position_grad_chain(float4 p, const GridParams& g, const float gx[4], float out[3]) {
  if (g.flags & SPIN4D_INPUT_NORMALISED) {
    out[0] = (p.x >= 0.0f && p.x <= 1.0f) ? gx[0] : 0.0f;
    out[1] = (p.y >= 0.0f && p.y <= 1.0f) ? gx[1] : 0.0f;
    out[2] = (p.z >= 0.0f && p.z <= 1.0f) ? gx[2] : 0.0f;
    return;
  }
  const float n2 = __fadd_rn(__fadd_rn(__fmul_rn(p.x, p.x), __fmul_rn(p.y, p.y)), __fmul_rn(p.z, p.z));
  const float n = __fsqrt_rn(n2);
  if (n <= 1.0f) {
    out[0] = 0.25f * gx[0];
    out[1] = 0.25f * gx[1];
    out[2] = 0.25f * gx[2];
    return;
  }
  const float in = 1.0f / n;
  const float gg = in * (2.0f - in);                 // 2/n - 1/n^2
  const float hh = 2.0f * in * in * in * (in - 1.0f);   // 2/n^4 - 2/n^3
  const float dot = p.x * gx[0] + p.y * gx[1] + p.z * gx[2];
  out[0] = 0.25f * (gg * gx[0] + hh * dot * p.x);
  out[1] = 0.25f * (gg * gx[1] + hh * dot * p.y);
  out[2] = 0.25f * (gg * gx[2] + hh * dot * p.z);
}

// ---------------------------------------------------------------------------
// Scatter-add of the adjoint: grad_l[idx_c][f] += w_c * dz[f]  (fp32 atomics).
// ---------------------------------------------------------------------------
template <int F>
__device__ __forceinline__ void scatter_entry(float* __restrict__ grad, uint32_t e, float wgt,
                                              const float dz[F]) {
  float* p = grad + (size_t)e * F;
  if constexpr (F == 1) {
    atomicAdd(p, wgt * dz[0]);
  } else if constexpr (F == 2) {
    atomicAdd(reinterpret_cast<float2*>(p), make_float2(wgt * dz[0], wgt * dz[1]));
  } else {
#pragma unroll
    for (int q = 0; q < F / 4; ++q)
      atomicAdd(reinterpret_cast<float4*>(p) + q,
                make_float4(wgt * dz[4 * q], wgt * dz[4 * q + 1], wgt * dz[4 * q + 2], wgt * dz[4 * q + 3]));
  }
}

template <int F>
__device__ __forceinline__ void scatter_level(const float xt[4], const GridParams& g, int l,
                                              float* __restrict__ grad_tables, const float dz[F]) {
  uint32_t base[4];
  float frac[4];
  level_cell(xt, g, l, base, frac);
  uint32_t idx[16];
  level_indices(base, g, l, idx);
  float w[16];
  level_weights(frac, w);
  float* gl = grad_tables + ((size_t)l << g.log2_T) * F;
#pragma unroll
  for (int c = 0; c < 16; ++c) scatter_entry<F>(gl, idx[c], w[c], dz);
}

// ---------------------------------------------------------------------------
// Activations (Eq. 11), covariance (Eq. 2) and their adjoints, fp32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

__device__ __forceinline__ void quat_rotmat(const float q[4], float R[3][3]) {
  const float w = q[0], x = q[1], y = q[2], z = q[3];
  R[0][0] = 1.f - 2.f * (y * y + z * z);
  R[0][1] = 2.f * (x * y - w * z);
  R[0][2] = 2.f * (x * z + w * y);
  R[1][0] = 2.f * (x * y + w * z);
  R[1][1] = 1.f - 2.f * (x * x + z * z);
  R[1][2] = 2.f * (y * z - w * x);
  R[2][0] = 2.f * (x * z - w * y);
  R[2][1] = 2.f * (y * z + w * x);
  R[2][2] = 1.f - 2.f * (x * x + y * y);
}

// Sigma = (R S)(R S)^T packed (xx, xy, xz, yy, yz, zz).
__device__ __forceinline__ void covariance(const float s[3], const float q[4], float cov[6]) {
  float R[3][3];
  quat_rotmat(q, R);
  float M[3][3];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int k = 0; k < 3; ++k) M[i][k] = R[i][k] * s[k];
  const int I[6] = {0, 0, 0, 1, 1, 2}, J[6] = {0, 1, 2, 1, 2, 2};
#pragma unroll
  for (int p = 0; p < 6; ++p)
    cov[p] = M[I[p]][0] * M[J[p]][0] + M[I[p]][1] * M[J[p]][1] + M[I[p]][2] * M[J[p]][2];
}

// Adjoint of `covariance`: ds += d/ds, dq += d/dq of sum(gc * cov).
__device__ __forceinline__ void covariance_backward(const float s[3], const float q[4], const float gc[6],
                                                    float ds[3], float dq[4]) {
  float R[3][3];
  quat_rotmat(q, R);
  // symmetric G: packed off-diagonals count once, so half on each side
  float G[3][3] = {{gc[0], 0.5f * gc[1], 0.5f * gc[2]},
                   {0.5f * gc[1], gc[3], 0.5f * gc[4]},
                   {0.5f * gc[2], 0.5f * gc[4], gc[5]}};
  float M[3][3], dM[3][3], dR[3][3];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int k = 0; k < 3; ++k) M[i][k] = R[i][k] * s[k];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int k = 0; k < 3; ++k) dM[i][k] = 2.f * (G[i][0] * M[0][k] + G[i][1] * M[1][k] + G[i][2] * M[2][k]);
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    ds[k] += dM[0][k] * R[0][k] + dM[1][k] * R[1][k] + dM[2][k] * R[2][k];
#pragma unroll
    for (int i = 0; i < 3; ++i) dR[i][k] = dM[i][k] * s[k];
  }
  const float w = q[0], x = q[1], y = q[2], z = q[3];
  dq[0] += 2.f * (-z * dR[0][1] + y * dR[0][2] + z * dR[1][0] - x * dR[1][2] - y * dR[2][0] + x * dR[2][1]);
  dq[1] += 2.f * (y * dR[0][1] + z * dR[0][2] + y * dR[1][0] - 2.f * x * dR[1][1] - w * dR[1][2] +
                  z * dR[2][0] + w * dR[2][1] - 2.f * x * dR[2][2]);
  dq[2] += 2.f * (-2.f * y * dR[0][0] + x * dR[0][1] + w * dR[0][2] + x * dR[1][0] + z * dR[1][2] -
                  w * dR[2][0] + z * dR[2][1] - 2.f * y * dR[2][2]);
  dq[3] += 2.f * (-2.f * z * dR[0][0] - w * dR[0][1] + x * dR[0][2] + w * dR[1][0] - 2.f * z * dR[1][1] +
                  y * dR[1][2] + x * dR[2][0] + y * dR[2][1]);
}

// r = r^ / max(||r^||, 1e-12); returns ||r^||.
__device__ __forceinline__ float normalise_quat(const float rh[4], float r[4]) {
  float nrm = sqrtf(rh[0] * rh[0] + rh[1] * rh[1] + rh[2] * rh[2] + rh[3] * rh[3]);
  float inv = 1.0f / fmaxf(nrm, kNormFloor);
#pragma unroll
  for (int i = 0; i < 4; ++i) r[i] = rh[i] * inv;
  return nrm;
}

__device__ __forceinline__ void normalise_quat_backward(const float r[4], float nrm, const float gr[4],
                                                        float drh[4]) {
  if (nrm > kNormFloor) {
    float dot = r[0] * gr[0] + r[1] * gr[1] + r[2] * gr[2] + r[3] * gr[3];
    float inv = 1.0f / nrm;
#pragma unroll
    for (int i = 0; i < 4; ++i) drh[i] = (gr[i] - r[i] * dot) * inv;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) drh[i] = gr[i] / kNormFloor;
  }
}

// KineticGS double-sigmoid window on the normalised time.
__device__ __forceinline__ float temporal_gate(float t, float c, float r, float tau) {
  return sigmoidf_((t - (c - r)) / tau) * sigmoidf_(((c + r) - t) / tau);
}

// Gradient w.r.t. the window centre c and half-width r of the gate, given
// dloss/dw: w = a b with a = sigma((t - (c - r))/tau), b = sigma(((c + r) - t)/tau),
// dw/dc = a b (a - b)/tau and dw/dr = a b (2 - a - b)/tau.
__device__ __forceinline__ void temporal_gate_backward(float t, float c, float r, float tau, float dw, float out[2]) {
  const float a = sigmoidf_((t - (c - r)) / tau), b = sigmoidf_(((c + r) - t) / tau);
  const float k = dw * a * b / tau;
  out[0] = k * (a - b);
  out[1] = k * (2.0f - a - b);
}

// Decoded attributes of one Gaussian from its 11 head outputs.
struct Attr {
  float s[3], r[4], rgb[3], o, cov[6];
};

__device__ __forceinline__ void heads_forward(const float y[kHeadRows], float gate, Attr& a) {
#pragma unroll
  for (int i = 0; i < 3; ++i) a.s[i] = expf(fminf(y[i], kScaleClip));
  normalise_quat(y + 3, a.r);
#pragma unroll
  for (int i = 0; i < 3; ++i) a.rgb[i] = sigmoidf_(y[7 + i]);
  a.o = sigmoidf_(y[10]) * gate;
  covariance(a.s, a.r, a.cov);
}

// dy = d loss / d y for loss = <g, attributes>; g members may be zero.
struct AttrGrad {
  float s[3], r[4], rgb[3], o, cov[6];
};

__device__ __forceinline__ void heads_backward(const float y[kHeadRows], float gate, const AttrGrad& g,
                                               float dy[kHeadRows]) {
  float s[3], r[4];
#pragma unroll
  for (int i = 0; i < 3; ++i) s[i] = expf(fminf(y[i], kScaleClip));
  float nrm = normalise_quat(y + 3, r);
  float ds[3] = {g.s[0], g.s[1], g.s[2]};
  float dr[4] = {g.r[0], g.r[1], g.r[2], g.r[3]};
  covariance_backward(s, r, g.cov, ds, dr);
#pragma unroll
  for (int i = 0; i < 3; ++i) dy[i] = (y[i] <= kScaleClip) ? ds[i] * s[i] : 0.0f;
  normalise_quat_backward(r, nrm, dr, dy + 3);
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    float c = sigmoidf_(y[7 + i]);
    dy[7 + i] = g.rgb[i] * c * (1.0f - c);
  }
  float so = sigmoidf_(y[10]);
  dy[10] = g.o * gate * so * (1.0f - so);
}

// Floats between consecutive per-block slots of a weight-gradient workspace:
// n rounded up to a multiple of 4 so every slot starts 16-byte aligned (the
// slots are updated with vector accesses).
__host__ __device__ __forceinline__ size_t slot_stride(int n) { return ((size_t)n + 3) & ~(size_t)3; }

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// Sums over a warp: v[i] holds this lane's value of column i; on return the
// lane holds the sum over the warp's 32 lanes of column `lane`.  Each of the
// five exchange rounds halves the columns a lane is responsible for.
__device__ __forceinline__ float warp_column_sum(float v[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}


// Adds 32 consecutive floats to a workspace slot row with fp32 vector
// reductions.  Only this thread ever updates these elements, so the adds land
// in program order and the sum does not depend on scheduling.
__device__ __forceinline__ void slot_add32(float* dst, const float a[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) atomicAdd(d + q, make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]));
}

}  // namespace spin4d
