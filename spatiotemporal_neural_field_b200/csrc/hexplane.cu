// HexPlane encoder + two-branch deformation network, fp32 SIMT path
// (4D Gaussian Splatting reading notes, sections 3.1-3.2; covariance from
// SPIN-4DGS section 3.1, Eq. 2).
//
// Forward, one thread per Gaussian: the 18 bilinear plane samples (3 scales x
// XY XZ YZ XT YT ZT) are gathered 4 channels at a time (full 16-byte vectors
// of a channel-last plane row) and folded straight into the first layer's
// accumulators, so the 576-wide feature never leaves registers.
//
// Backward, one thread block per tile of 64 Gaussians: activations and deltas
// of the small layers sit in shared memory [feature][gaussian]; the first
// layer's weight gradient is reduced plane sample by plane sample (32 input
// features at a time, re-gathered), so shared memory never holds the whole
// 576-wide feature.  Weight gradients go to the block's workspace slot and
// are summed in a fixed order by a second kernel; plane gradients are
// scattered with fp32 vector atomics.
#include <cuda_bf16.h>
#include <string.h>

#include <cmath>
#include <stdlib.h>

#include <mutex>

#include "host.h"
#include "tc.cuh"

namespace spin4d {

// Set when a bounded wait of a HexPlane tensor-core kernel runs out.
__device__ int g_hex_device_error = 0;

int hex_device_error(int clear) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_hex_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_status(e);
  if (clear && v) {
    int zero = 0;
    e = cudaMemcpyToSymbol(g_hex_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_status(e);
  }
  return v ? SPIN4D_ERR_TIMEOUT : SPIN4D_OK;
}

constexpr int kHexC = 32;
constexpr int kHexH = 64;
constexpr int kHexHead = 58;
constexpr int kHexBwdBlock = 64;

struct HexParams {
  int n_samples;          // n_scales * 6
  int in_dim;             // n_samples * C
  float inv_frames;       // unused placeholder for layout stability
  float frames_m1;        // (float)(n_frames - 1)
  int axis_a[24], axis_b[24];
  int res_a[24], res_b[24];
  float scale_a[24], scale_b[24];
  int64_t off[24];        // float offset of each plane
  // KineticGS energy-flow window (NULL gate_cr: no window): w from the
  // per-Gaussian (c, r) on the normalised time, H(w) = [w >= 1/2] gates the
  // displacement, w scales the log-scale and SH offsets; gate_grad (N x 2,
  // may be NULL) receives d loss / d(c, r) in the backward
  const float* gate_cr;
  float* gate_grad;
  float gate_tau;
};

// The window weight w and the displacement gate H(w) of Gaussian n (1, 1
// without a window).
__device__ __forceinline__ void hex_window(const HexParams& hp, const int32_t* __restrict__ frame, int64_t n,
                                          float& w, float& hgate, float& t, float2& cr) {
  w = 1.0f;
  hgate = 1.0f;
  t = 0.0f;
  cr = make_float2(0.f, 0.f);
  if (!hp.gate_cr) return;
  t = clamp01(__fdiv_rn((float)__ldg(frame + n), hp.frames_m1));
  cr = __ldg(reinterpret_cast<const float2*>(hp.gate_cr) + n);
  w = temporal_gate(t, cr.x, cr.y, hp.gate_tau);
  hgate = w >= 0.5f ? 1.0f : 0.0f;
}

struct HexOutPtrs {
  float *mu, *rot, *scale, *sh, *cov;
};
struct HexGradPtrs {
  const float *mu, *rot, *scale, *sh, *cov;
};

__device__ __forceinline__ void hex_normalise(const float* __restrict__ mu, const int32_t* __restrict__ frame,
                                              int64_t n, const HexParams& hp, float xt[4]) {
#pragma unroll
  for (int d = 0; d < 3; ++d) xt[d] = clamp01(__fmul_rn(__fadd_rn(__ldg(mu + 3 * n + d), 1.0f), 0.5f));
  xt[3] = clamp01(__fdiv_rn((float)__ldg(frame + n), hp.frames_m1));
}

struct PlaneSample {
  int64_t o00, o01, o10, o11;   // float offsets of the 4 corners' channel rows
  float w00, w01, w10, w11;
};

// xt[a] by selects, so a runtime axis index keeps xt in registers.
__device__ __forceinline__ float pick_axis(const float xt[4], int a) {
  return a == 0 ? xt[0] : (a == 1 ? xt[1] : (a == 2 ? xt[2] : xt[3]));
}

__device__ __forceinline__ PlaneSample plane_sample(const float xt[4], const HexParams& hp, int k) {
  float pa = __fmul_rn(pick_axis(xt, hp.axis_a[k]), hp.scale_a[k]);
  float pb = __fmul_rn(pick_axis(xt, hp.axis_b[k]), hp.scale_b[k]);
  int ia = min(max((int)floorf(pa), 0), hp.res_a[k] - 2);
  int ib = min(max((int)floorf(pb), 0), hp.res_b[k] - 2);
  float wa = __fsub_rn(pa, (float)ia), wb = __fsub_rn(pb, (float)ib);
  PlaneSample s;
  const int64_t row = (int64_t)hp.res_a[k] * kHexC;
  s.o00 = hp.off[k] + ((int64_t)ib * hp.res_a[k] + ia) * kHexC;
#ifdef SPIN4D_CHECKED
  // the cell's four rows inside plane k
  if (!bounds_ok(ia >= 0 && ib >= 0 && ia + 1 < hp.res_a[k] && ib + 1 < hp.res_b[k])) s.o00 = hp.off[k];
#endif
  s.o01 = s.o00 + kHexC;
  s.o10 = s.o00 + row;
  s.o11 = s.o10 + kHexC;
  s.w00 = (1.0f - wa) * (1.0f - wb);
  s.w01 = wa * (1.0f - wb);
  s.w10 = (1.0f - wa) * wb;
  s.w11 = wa * wb;
  return s;
}

// The first corner's float offset and the bilinear fractions of sample k,
// computed exactly as plane_sample does.
__device__ __forceinline__ int64_t plane_corner(const float xt[4], const HexParams& hp, int k, float& wa, float& wb) {
  float pa = __fmul_rn(pick_axis(xt, hp.axis_a[k]), hp.scale_a[k]);
  float pb = __fmul_rn(pick_axis(xt, hp.axis_b[k]), hp.scale_b[k]);
  int ia = min(max((int)floorf(pa), 0), hp.res_a[k] - 2);
  int ib = min(max((int)floorf(pb), 0), hp.res_b[k] - 2);
  wa = __fsub_rn(pa, (float)ia);
  wb = __fsub_rn(pb, (float)ib);
#ifdef SPIN4D_CHECKED
  if (!bounds_ok(ia >= 0 && ib >= 0 && ia + 1 < hp.res_a[k] && ib + 1 < hp.res_b[k])) return hp.off[k];
#endif
  return hp.off[k] + ((int64_t)ib * hp.res_a[k] + ia) * kHexC;
}

__device__ __forceinline__ float4 sample4(const float* __restrict__ planes, const PlaneSample& s, int c4) {
  float4 a = __ldg(reinterpret_cast<const float4*>(planes + s.o00) + c4);
  float4 b = __ldg(reinterpret_cast<const float4*>(planes + s.o01) + c4);
  float4 c = __ldg(reinterpret_cast<const float4*>(planes + s.o10) + c4);
  float4 d = __ldg(reinterpret_cast<const float4*>(planes + s.o11) + c4);
  float4 r;
  r.x = s.w00 * a.x + s.w01 * b.x + s.w10 * c.x + s.w11 * d.x;
  r.y = s.w00 * a.y + s.w01 * b.y + s.w10 * c.y + s.w11 * d.y;
  r.z = s.w00 * a.z + s.w01 * b.z + s.w10 * c.z + s.w11 * d.z;
  r.w = s.w00 * a.w + s.w01 * b.w + s.w10 * c.w + s.w11 * d.w;
  return r;
}

__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }

// Forward through the trunk: h1 = relu(W1 z + b1), h2 = relu(W2 h1 + b2).
__device__ __forceinline__ void hex_trunk(const float xt[4], const HexParams& hp, const float* __restrict__ planes,
                                          const float* __restrict__ W, float h1[kHexH], float h2[kHexH]) {
  const int IN = hp.in_dim;
  const float* b1 = W + kHexH * IN;
#pragma unroll
  for (int o = 0; o < kHexH; ++o) h1[o] = __ldg(b1 + o);
  for (int k = 0; k < hp.n_samples; ++k) {
    PlaneSample s = plane_sample(xt, hp, k);
    const int fo = k * kHexC;
#pragma unroll 1
    for (int c4 = 0; c4 < kHexC / 4; ++c4) {
      float4 z4 = sample4(planes, s, c4);
#pragma unroll
      for (int o = 0; o < kHexH; ++o)
        h1[o] += dot4(__ldg(reinterpret_cast<const float4*>(W + (size_t)o * IN + fo) + c4), z4);
    }
  }
#pragma unroll
  for (int o = 0; o < kHexH; ++o) h1[o] = fmaxf(h1[o], 0.0f);
  const float* W2 = b1 + kHexH;
  const float* b2 = W2 + kHexH * kHexH;
#pragma unroll 4
  for (int o = 0; o < kHexH; ++o) {
    float acc = __ldg(b2 + o);
#pragma unroll
    for (int k4 = 0; k4 < kHexH / 4; ++k4) {
      float4 w = __ldg(reinterpret_cast<const float4*>(W2 + o * kHexH) + k4);
      acc += w.x * h1[4 * k4] + w.y * h1[4 * k4 + 1] + w.z * h1[4 * k4 + 2] + w.w * h1[4 * k4 + 3];
    }
    h2[o] = fmaxf(acc, 0.0f);
  }
}

__device__ __forceinline__ float head_row(const float* __restrict__ W3, int o, const float h2[kHexH]) {
  float acc = __ldg(W3 + kHexHead * kHexH + o);
#pragma unroll
  for (int k4 = 0; k4 < kHexH / 4; ++k4) {
    float4 w = __ldg(reinterpret_cast<const float4*>(W3 + o * kHexH) + k4);
    acc += w.x * h2[4 * k4] + w.y * h2[4 * k4 + 1] + w.z * h2[4 * k4 + 2] + w.w * h2[4 * k4 + 3];
  }
  return acc;
}

__device__ __forceinline__ const float* head_weights(const float* W, const HexParams& hp) {
  return W + kHexH * hp.in_dim + kHexH + kHexH * kHexH + kHexH;
}

__global__ void __launch_bounds__(128) hexplane_fwd_kernel(HexParams hp, const float* __restrict__ mu,
                                                           const int32_t* __restrict__ frame, int64_t N,
                                                           const float* __restrict__ planes,
                                                           const float* __restrict__ W,
                                                           const float* __restrict__ q_can,
                                                           const float* __restrict__ logs_can,
                                                           const float* __restrict__ sh_can, HexOutPtrs out) {
  const float* W3 = head_weights(W, hp);
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N; n += (int64_t)gridDim.x * blockDim.x) {
    float xt[4];
    hex_normalise(mu, frame, n, hp, xt);
    float h1[kHexH], h2[kHexH];
    hex_trunk(xt, hp, planes, W, h1, h2);
    float y[10];
#pragma unroll
    for (int o = 0; o < 10; ++o) y[o] = head_row(W3, o, h2);
    for (int o = 10; o < kHexHead; ++o) out.sh[48 * n + (o - 10)] = __ldg(sh_can + 48 * n + (o - 10)) + head_row(W3, o, h2);
    float qh[4], q[4], s[3], cov[6];
#pragma unroll
    for (int i = 0; i < 3; ++i) out.mu[3 * n + i] = __ldg(mu + 3 * n + i) + y[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) qh[i] = __ldg(q_can + 4 * n + i) + y[3 + i];
    normalise_quat(qh, q);
#pragma unroll
    for (int i = 0; i < 3; ++i) s[i] = expf(__ldg(logs_can + 3 * n + i) + y[7 + i]);
    covariance(s, q, cov);
    reinterpret_cast<float4*>(out.rot)[n] = make_float4(q[0], q[1], q[2], q[3]);
#pragma unroll
    for (int i = 0; i < 3; ++i) out.scale[3 * n + i] = s[i];
#pragma unroll
    for (int i = 0; i < 6; ++i) out.cov[6 * n + i] = cov[i];
  }
}

__device__ __forceinline__ float g_or0(const float* p, int64_t i) { return p ? __ldg(p + i) : 0.0f; }

// slot[p] += sum_t d[o][t] * a[k][t] for the (o, k) of this block's layer.
__device__ __forceinline__ void hex_block_wgrad(const float* d, const float* a, int n_out, int n_in, float* slot_w,
                                                float* slot_b) {
  const int nW = n_out * n_in;
  for (int p = threadIdx.x; p < nW + n_out; p += blockDim.x) {
    float s = 0.0f;
    if (p < nW) {
      const int o = p / n_in, k = p - o * n_in;
      for (int t = 0; t < kHexBwdBlock; ++t) s = fmaf(d[o * kHexBwdBlock + t], a[k * kHexBwdBlock + t], s);
      slot_w[p] += s;
    } else {
      const int o = p - nW;
      for (int t = 0; t < kHexBwdBlock; ++t) s += d[o * kHexBwdBlock + t];
      slot_b[o] += s;
    }
  }
}

__global__ void __launch_bounds__(kHexBwdBlock) hexplane_bwd_kernel(
    HexParams hp, const float* __restrict__ mu, const int32_t* __restrict__ frame, int64_t N,
    const float* __restrict__ planes, const float* __restrict__ W, const float* __restrict__ q_can,
    const float* __restrict__ logs_can, HexGradPtrs go, float* __restrict__ grad_planes, float* __restrict__ ws,
    int n_params) {
  extern __shared__ float hsm[];
  float* h1b = hsm;
  float* h2b = h1b + kHexH * kHexBwdBlock;
  float* dyb = h2b + kHexH * kHexBwdBlock;
  float* d2b = dyb + kHexHead * kHexBwdBlock;
  float* d1b = d2b + kHexH * kHexBwdBlock;
  float* zc = d1b + kHexH * kHexBwdBlock;
  const int IN = hp.in_dim;
  const int col = threadIdx.x;
  float* slot = ws + (size_t)blockIdx.x * slot_stride(n_params);
  for (int p = threadIdx.x; p < n_params; p += blockDim.x) slot[p] = 0.0f;
  const float* W2 = W + kHexH * IN + kHexH;
  const float* W3 = head_weights(W, hp);
  float* sW1 = slot;
  float* sb1 = slot + kHexH * IN;
  float* sW2 = sb1 + kHexH;
  float* sb2 = sW2 + kHexH * kHexH;
  float* sW3 = sb2 + kHexH;
  float* sb3 = sW3 + kHexHead * kHexH;

  for (int64_t n0 = (int64_t)blockIdx.x * kHexBwdBlock; n0 < N; n0 += (int64_t)gridDim.x * kHexBwdBlock) {
    const int64_t n = n0 + col;
    const bool valid = n < N;
    float xt[4] = {0.f, 0.f, 0.f, 0.f};
    // ---- A: forward, head adjoint ----
    if (valid) {
      hex_normalise(mu, frame, n, hp, xt);
      float h1[kHexH], h2[kHexH];
      hex_trunk(xt, hp, planes, W, h1, h2);
#pragma unroll
      for (int o = 0; o < kHexH; ++o) {
        h1b[o * kHexBwdBlock + col] = h1[o];
        h2b[o * kHexBwdBlock + col] = h2[o];
      }
      float y[10];
#pragma unroll
      for (int o = 0; o < 10; ++o) y[o] = head_row(W3, o, h2);
      float qh[4], q[4], s[3];
#pragma unroll
      for (int i = 0; i < 4; ++i) qh[i] = __ldg(q_can + 4 * n + i) + y[3 + i];
      float nrm = normalise_quat(qh, q);
#pragma unroll
      for (int i = 0; i < 3; ++i) s[i] = expf(__ldg(logs_can + 3 * n + i) + y[7 + i]);
      float gc[6], ds[3], dq[4], dqh[4];
#pragma unroll
      for (int i = 0; i < 6; ++i) gc[i] = g_or0(go.cov, 6 * n + i);
#pragma unroll
      for (int i = 0; i < 3; ++i) ds[i] = g_or0(go.scale, 3 * n + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) dq[i] = g_or0(go.rot, 4 * n + i);
      covariance_backward(s, q, gc, ds, dq);
      normalise_quat_backward(q, nrm, dq, dqh);
#pragma unroll
      for (int i = 0; i < 3; ++i) dyb[i * kHexBwdBlock + col] = g_or0(go.mu, 3 * n + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) dyb[(3 + i) * kHexBwdBlock + col] = dqh[i];
#pragma unroll
      for (int i = 0; i < 3; ++i) dyb[(7 + i) * kHexBwdBlock + col] = ds[i] * s[i];
      for (int i = 0; i < 48; ++i) dyb[(10 + i) * kHexBwdBlock + col] = g_or0(go.sh, 48 * n + i);
    } else {
      for (int o = 0; o < kHexH; ++o) h1b[o * kHexBwdBlock + col] = h2b[o * kHexBwdBlock + col] = 0.0f;
      for (int o = 0; o < kHexHead; ++o) dyb[o * kHexBwdBlock + col] = 0.0f;
    }
    __syncthreads();
    // ---- B: head weight gradient; C: delta of layer 2 ----
    hex_block_wgrad(dyb, h2b, kHexHead, kHexH, sW3, sb3);
    for (int k = 0; k < kHexH; ++k) {
      float s = 0.0f;
      for (int o = 0; o < kHexHead; ++o) s = fmaf(__ldg(W3 + o * kHexH + k), dyb[o * kHexBwdBlock + col], s);
      d2b[k * kHexBwdBlock + col] = h2b[k * kHexBwdBlock + col] > 0.0f ? s : 0.0f;
    }
    __syncthreads();
    // ---- D: layer-2 weight gradient; E: delta of layer 1 ----
    hex_block_wgrad(d2b, h1b, kHexH, kHexH, sW2, sb2);
    for (int k = 0; k < kHexH; ++k) {
      float s = 0.0f;
      for (int o = 0; o < kHexH; ++o) s = fmaf(__ldg(W2 + o * kHexH + k), d2b[o * kHexBwdBlock + col], s);
      d1b[k * kHexBwdBlock + col] = h1b[k * kHexBwdBlock + col] > 0.0f ? s : 0.0f;
    }
    __syncthreads();
    // layer-1 bias
    for (int o = threadIdx.x; o < kHexH; o += blockDim.x) {
      float s = 0.0f;
      for (int t = 0; t < kHexBwdBlock; ++t) s += d1b[o * kHexBwdBlock + t];
      sb1[o] += s;
    }
    // ---- F: per plane sample: re-gather z, scatter dz, reduce dW1 ----
    for (int k = 0; k < hp.n_samples; ++k) {
      const int fo = k * kHexC;
      if (valid) {
        PlaneSample s = plane_sample(xt, hp, k);
        for (int c4 = 0; c4 < kHexC / 4; ++c4) {
          float4 z4 = sample4(planes, s, c4);
          zc[(4 * c4 + 0) * kHexBwdBlock + col] = z4.x;
          zc[(4 * c4 + 1) * kHexBwdBlock + col] = z4.y;
          zc[(4 * c4 + 2) * kHexBwdBlock + col] = z4.z;
          zc[(4 * c4 + 3) * kHexBwdBlock + col] = z4.w;
          float4 dz = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int o = 0; o < kHexH; ++o) {
            float d = d1b[o * kHexBwdBlock + col];
            float4 w = __ldg(reinterpret_cast<const float4*>(W + (size_t)o * IN + fo) + c4);
            dz.x = fmaf(w.x, d, dz.x);
            dz.y = fmaf(w.y, d, dz.y);
            dz.z = fmaf(w.z, d, dz.z);
            dz.w = fmaf(w.w, d, dz.w);
          }
          float4* g00 = reinterpret_cast<float4*>(grad_planes + s.o00) + c4;
          float4* g01 = reinterpret_cast<float4*>(grad_planes + s.o01) + c4;
          float4* g10 = reinterpret_cast<float4*>(grad_planes + s.o10) + c4;
          float4* g11 = reinterpret_cast<float4*>(grad_planes + s.o11) + c4;
          atomicAdd(g00, make_float4(s.w00 * dz.x, s.w00 * dz.y, s.w00 * dz.z, s.w00 * dz.w));
          atomicAdd(g01, make_float4(s.w01 * dz.x, s.w01 * dz.y, s.w01 * dz.z, s.w01 * dz.w));
          atomicAdd(g10, make_float4(s.w10 * dz.x, s.w10 * dz.y, s.w10 * dz.z, s.w10 * dz.w));
          atomicAdd(g11, make_float4(s.w11 * dz.x, s.w11 * dz.y, s.w11 * dz.z, s.w11 * dz.w));
        }
      } else {
        for (int c = 0; c < kHexC; ++c) zc[c * kHexBwdBlock + col] = 0.0f;
      }
      __syncthreads();
      for (int p = threadIdx.x; p < kHexH * kHexC; p += blockDim.x) {
        const int o = p / kHexC, c = p - o * kHexC;
        float s = 0.0f;
        for (int t = 0; t < kHexBwdBlock; ++t) s = fmaf(d1b[o * kHexBwdBlock + t], zc[c * kHexBwdBlock + t], s);
        sW1[(size_t)o * IN + fo + c] += s;
      }
      __syncthreads();
    }
  }
}

__global__ void hex_reduce_slots(const float* __restrict__ ws, int n_slots, int n_params, float* __restrict__ out) {
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < n_params; p += gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int c = 0; c < n_slots; ++c) s += ws[(size_t)c * slot_stride(n_params) + p];
    out[p] += s;
  }
}

// ---------------------------------------------------------------------------
// Forward and backward on the tensor cores, fp32-accurate: bf16x3 split.
//
// Every operand x is split into three bf16 parts, x0 = bf16(x),
// x1 = bf16(x - x0), x2 = bf16(x - x0 - x1), so |x - (x0 + x1 + x2)| is below
// 2^-26 |x|.  A product keeps the six terms x_i.y_j with i + j <= 2: x0.y0 in
// one TMEM accumulator and the five smaller terms in a second one (the
// tensor core aligns addends to the running sum and truncates, so the small
// terms must not share the big one's accumulator); the dropped terms are
// below 2^-25 of the result.  Accumulators are fresh for every short K (one
// plane sample, one layer, one tile of Gaussians) and partial results are
// added in fp32 on the CUDA cores.  kind::f16 takes K = 16 per instruction,
// so this issues as many MMAs as a 3xTF32 split; unlike kind::tf32, which
// returned zero products for MN-major (transposed) operand tiles without
// swizzle here, it reads such tiles, which the weight gradients need.
//
// Persistent CTAs of 256 threads handle 128-Gaussian tiles, two threads per
// Gaussian (32 of its 64 hidden columns, or 16 of a sample's 32 channels,
// each).  The 576-wide first layer is streamed one plane sample (32
// channels) at a time through two shared-memory stages: while the tensor
// core multiplies sample k, the threads gather and split sample k+1 (16-byte
// loads of the channel-last rows) and stage the matching 64x32 slice of W1.
//
// Every operand tile is stored [row][col] in 8-row x 16-byte core matrices:
// element (r, c) of a tile with L columns sits at byte
// (r/8)*16L + (c/8)*128 + (r%8)*16 + (c%8)*2 of each of its three planes.
// Read with rows as M or N and columns as K this is the canonical K-major
// layout (LBO 128, SBO 16L); read with columns as M or N and rows as K it is
// the MN-major one (SBO 128 between 8-column blocks, LBO 16L between 8-row
// blocks).  A tile written once therefore serves a product and its
// transpose: the z stage is layer 1's A operand (rows = Gaussians) and the
// W1 gradient's B operand (K = Gaussians), the W1 stage is layer 1's B
// operand and dz's transposed B operand, and each activation or delta tile
// is the A operand of a data gradient and a transposed operand of a weight
// gradient.
// ---------------------------------------------------------------------------
namespace {

constexpr int kHexTile = 128;
constexpr int kHexThreads = 256;
constexpr uint32_t kHexWait = 1u << 24;

// Byte size of one bf16 plane of an R x L tile.
constexpr int plane_bytes(int R, int L) { return R * L * 2; }

// The forward's z tiles are K-major with the 8-row groups adjacent (128 B
// apart) and the four 8-column chunks kZChunk = 2080 bytes apart: the 32-byte
// skew sends a warp's stores of four rows x 32 columns to distinct banks.
// (The backward keeps the plain layout, chunks adjacent; both fit Z_PLANE.)
constexpr int kZChunk = (kHexTile / 8) * 128 + 32;
__device__ __forceinline__ uint32_t zpad_off(int r, int c) {
  return (uint32_t)((r >> 3) * 128 + (c >> 3) * kZChunk + (r & 7) * 16 + (c & 7) * 2);
}

struct HexTcLayout {
  static constexpr int Z_PLANE = (kHexC / 8) * kZChunk;             // 8320 B (>= 8 KB of the plain layout)
  static constexpr int Z_STAGE = 3 * Z_PLANE;
  static constexpr int A = 0;                                      // 2 z stages = 48.75 KB; later the H tile
  static constexpr int H_PLANE = plane_bytes(kHexTile, kHexH);     // 16 KB: the H tile fills region A
  static constexpr int W_PLANE = plane_bytes(kHexH, kHexC);        // 4 KB
  static constexpr int W_STAGE = 3 * W_PLANE;
  static constexpr int B1 = A + 2 * Z_STAGE;                       // 2 W1 stages = 24 KB
  static constexpr int S_PLANE = plane_bytes(kHexH, kHexH);        // 8 KB
  static constexpr int W2 = B1 + 2 * W_STAGE;                      // [64][64] x 3 planes
  static constexpr int W3 = W2 + 3 * S_PLANE;                      // [64][64] x 3 planes (58 rows used)
  static __device__ __forceinline__ int z(int b) { return A + b * Z_STAGE; }
  static __device__ __forceinline__ int w(int b) { return B1 + b * W_STAGE; }
};
static_assert(3 * HexTcLayout::H_PLANE <= 2 * HexTcLayout::Z_STAGE, "the H tile must fit over the z stages");
static_assert(HexTcLayout::B1 % 128 == 0, "tile alignment");

// Backward: the forward's z stages, W1 stages and W2 | W3 at the same
// offsets, the scatter staging over W2 | W3, a second activation tile T1,
// then the biases and the CTA's bias-gradient sums.  The first activation
// tile T0 is the forward's H tile (over the z stages).
struct HexBwdLayout {
  // Per plane sample of the dz pass, the 4 bilinear corners' 128-byte rows of
  // w_c * dz for every Gaussian of the tile, 16 bytes of padding per Gaussian
  // so that a warp's row stores hit distinct banks.  Overlays W2 | W3, which
  // are staged again at the start of every tile.
  static constexpr int SCAT_ROW = 4 * kHexC * 4 + 16;
  static constexpr int SCAT = HexTcLayout::W2;
  static constexpr int T1 = SCAT + kHexTile * SCAT_ROW;       // [128][64] x 3 planes
  static constexpr int BIAS = T1 + 3 * HexTcLayout::H_PLANE;  // b1 | b2 | b3
  static constexpr int BACC = BIAS + 3 * kHexH * 4;           // db1 | db2 | db3 over the CTA's tiles
  static constexpr int MISC = BACC + 3 * kHexH * 4;           // 2 mbarriers + TMEM address
  static constexpr int GSUM = MISC + 32;                      // [128]: the SH half of d loss / d w (window)
  static constexpr int BYTES = GSUM + kHexTile * 4;
};
static_assert(HexBwdLayout::BYTES <= 227 * 1024, "backward tiles exceed the shared memory of one CTA");

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Stores 8 consecutive values of row r (8-column chunk kc of a tile with L
// columns) as its three bf16 planes (plane = bytes between planes).
__device__ __forceinline__ void store_split8(uint8_t* sm, int off, int plane, int r, int kc, int L, const float v[8]) {
  uint32_t p0[4], p1[4], p2[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    const float2 f0 = __bfloat1622float2(h0);
    const float r0 = v[2 * j] - f0.x, r1 = v[2 * j + 1] - f0.y;
    const __nv_bfloat162 h1 = __floats2bfloat162_rn(r0, r1);
    const float2 f1 = __bfloat1622float2(h1);
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(r0 - f1.x, r1 - f1.y);
    p0[j] = bf2_bits(h0);
    p1[j] = bf2_bits(h1);
    p2[j] = bf2_bits(h2);
  }
  const uint32_t o = (uint32_t)off + tc::kmaj_off(r, kc, L);
  *reinterpret_cast<uint4*>(sm + o) = make_uint4(p0[0], p0[1], p0[2], p0[3]);
  *reinterpret_cast<uint4*>(sm + o + plane) = make_uint4(p1[0], p1[1], p1[2], p1[3]);
  *reinterpret_cast<uint4*>(sm + o + 2 * plane) = make_uint4(p2[0], p2[1], p2[2], p2[3]);
}

__device__ __forceinline__ void store_split8(uint8_t* sm, int off, int plane, int r, int kc, int L, float4 a, float4 b) {
  const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  store_split8(sm, off, plane, r, kc, L, v);
}

// Stores 4 consecutive values (columns c .. c + 3, c % 4 == 0) of row r of
// a z tile in the skewed layout (zpad_off) as their three bf16 planes.
__device__ __forceinline__ void store_split4(uint8_t* sm, int off, int plane, int r, int c, float4 v) {
  const float x[4] = {v.x, v.y, v.z, v.w};
  uint32_t p0[2], p1[2], p2[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
    const float2 f0 = __bfloat1622float2(h0);
    const float r0 = x[2 * j] - f0.x, r1 = x[2 * j + 1] - f0.y;
    const __nv_bfloat162 h1 = __floats2bfloat162_rn(r0, r1);
    const float2 f1 = __bfloat1622float2(h1);
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(r0 - f1.x, r1 - f1.y);
    p0[j] = bf2_bits(h0);
    p1[j] = bf2_bits(h1);
    p2[j] = bf2_bits(h2);
  }
  const uint32_t o = (uint32_t)off + zpad_off(r, c);
  *reinterpret_cast<uint2*>(sm + o) = make_uint2(p0[0], p0[1]);
  *reinterpret_cast<uint2*>(sm + o + plane) = make_uint2(p1[0], p1[1]);
  *reinterpret_cast<uint2*>(sm + o + 2 * plane) = make_uint2(p2[0], p2[1]);
}

// Stores this thread's 32 values (columns half*32 ..) of row r of a 64-column tile.
__device__ __forceinline__ void store_row32(uint8_t* sm, int off, int r, int half, const float v[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) store_split8(sm, off, HexTcLayout::H_PLANE, r, half * 4 + q, kHexH, v + 8 * q);
}

// One operand of a split product: shared-memory address of plane 0, bytes
// between planes, descriptor strides, and how far the start address moves
// per 16-deep K slice.
struct SplitOp {
  uint32_t base, plane, lbo, sbo, step;
};
// Tile with L columns read K-major (rows are M or N, columns are K).
__device__ __forceinline__ SplitOp kmajor(uint32_t base, int plane, int L) {
  return {base, (uint32_t)plane, 128u, 16u * (uint32_t)L, 256u};
}
// A forward z tile (128 rows, skewed layout).
__device__ __forceinline__ SplitOp kmajor_zpad(uint32_t base, int plane) {
  return {base, (uint32_t)plane, (uint32_t)kZChunk, 128u, 2u * kZChunk};
}
// Tile with L columns read MN-major (columns are M or N, rows are K).
__device__ __forceinline__ SplitOp mnmajor(uint32_t base, int plane, int L) {
  return {base, (uint32_t)plane, 16u * (uint32_t)L, 128u, 32u * (uint32_t)L};
}

// Split product over K into two fresh accumulators: d_main = A0.B0 and
// d_corr = A0.B1 + A1.B0 + A0.B2 + A2.B0 + A1.B1.
__device__ __forceinline__ void mma6(uint32_t d_main, uint32_t d_corr, const SplitOp& a, const SplitOp& b, int K,
                                     uint32_t idesc) {
  // Descriptors are built once; a K slice moves the start-address field
  // (address / 16, low bits) by step / 16.
  uint64_t ad[3], bd[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    ad[i] = tc::smem_desc(a.base + i * a.plane, a.lbo, a.sbo);
    bd[i] = tc::smem_desc(b.base + i * b.plane, b.lbo, b.sbo);
  }
  for (int s = 0; s < K / 16; ++s) {
    if (s > 0) {
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        ad[i] += a.step >> 4;
        bd[i] += b.step >> 4;
      }
    }
    const uint32_t acc = s > 0 ? 1u : 0u;
    tc::mma_f16(d_main, ad[0], bd[0], idesc, acc);
    tc::mma_f16(d_corr, ad[0], bd[1], idesc, acc);
    tc::mma_f16(d_corr, ad[1], bd[0], idesc, 1u);
    tc::mma_f16(d_corr, ad[0], bd[2], idesc, 1u);
    tc::mma_f16(d_corr, ad[2], bd[0], idesc, 1u);
    tc::mma_f16(d_corr, ad[1], bd[1], idesc, 1u);
  }
}

// acc[i] += main[col0 + i] + corr[col0 + i] for this thread's 32 columns.
__device__ __forceinline__ void add_partial(uint32_t d_main, uint32_t d_corr, float acc[32]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float a[16], b[16];
    tc::tmem_ld16(d_main + 16 * h, a);
    tc::tmem_ld16(d_corr + 16 * h, b);
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[16 * h + i] += a[i] + b[i];
  }
}

// Commit barriers of the two stages; every commit is waited for exactly once.
struct HexBars {
  uint32_t bar0, bar1, ph0, ph1;
  __device__ __forceinline__ uint32_t addr(int b) const { return b ? bar1 : bar0; }
  __device__ __forceinline__ bool wait(int b) {
    const bool ok = tc::mbar_wait_bounded(b ? bar1 : bar0, b ? ph1 : ph0, kHexWait);
    if (b)
      ph1 ^= 1u;
    else
      ph0 ^= 1u;
    return ok;
  }
};

// 32 bytes (one sector) of read-only global data in one 256-bit load; p must
// be 32-byte aligned.
__device__ __forceinline__ void ld_nc_v8(const float* p, float v[8]) {
  asm volatile("ld.global.nc.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
               : "l"(p));
}

// An L2 policy that evicts first: the latent streams through L2 (1.15 GB at
// 500k Gaussians) and should not push out the planes or their gradients.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void st_v4_stream(float* p, float4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1,%2,%3,%4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w), "l"(pol)
               : "memory");
}
// The planes are the one data set worth keeping in L2 across a launch: their
// rows are read with an evict-last policy, and the per-Gaussian inputs and
// outputs (hundreds of MB that each pass exactly once) with evict-first.
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ float4 ld_nc_v4_hint(const float4* p, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.f32 {%0,%1,%2,%3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ float ld_nc_hint(const float* p, uint64_t pol) {
  float v;
  asm volatile("ld.global.nc.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(v) : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ void st_hint(float* p, float v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

// Global data of one plane sample for one thread: its chunk of the W1 slice
// (row tid/4, 8 columns) and, for its Gaussian, either the 16 channels
// (half*16 ..) of the four corner rows with their bilinear weights, or the
// 16 values of a saved latent.
// One thread's share of a plane sample in flight: its W1 slice chunk, its
// half of the four corner rows, and the bilinear weights.
struct SampleRegs {
  float w[8];
  float c[4][16];
  float wt[4];
};

// Streams the plane samples of one tile through the two stages.  Stage
// b = k & 1 receives sample k: the 64x32 slice of W1 for the sample and the
// tile's 128x32 feature block z_k (split), sampled from the planes.
// issue(k, b) runs on thread 0 once the stage is written and its MMAs are
// committed to stage b's barrier; consume(k, b) runs on every thread once
// they are done, before the stage takes sample k + 2.  Each thread reads its
// half of its Gaussian's four corner rows as 32-byte sectors, one sample
// ahead.  The sample count is even (6 per scale).  Returns false if a wait
// ran out.
template <class Issue, class Consume>
__device__ __forceinline__ bool hex_stream(uint8_t* sm, const HexParams& hp, const float* __restrict__ planes,
                                           const float* __restrict__ W1, bool valid, const float xt[4],
                                           HexBars& bars, Issue issue, Consume consume) {
  using Lay = HexTcLayout;
  const int tid = threadIdx.x, row = tid & (kHexTile - 1), half = tid / kHexTile;
  const int IN = hp.in_dim, NS = hp.n_samples;
  SampleRegs r;
  auto prefetch = [&](int k) {
    ld_nc_v8(W1 + (size_t)(tid >> 2) * IN + k * kHexC + (tid & 3) * 8, r.w);
    if (!valid) return;
    const PlaneSample ps = plane_sample(xt, hp, k);
    r.wt[0] = ps.w00;
    r.wt[1] = ps.w01;
    r.wt[2] = ps.w10;
    r.wt[3] = ps.w11;
    const int64_t off[4] = {ps.o00, ps.o01, ps.o10, ps.o11};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      ld_nc_v8(planes + off[c] + half * 16, r.c[c]);
      ld_nc_v8(planes + off[c] + half * 16 + 8, r.c[c] + 8);
    }
  };
  auto step = [&](int k) -> bool {
    const int b = k & 1;
    bool ok = true;
    if (k >= 2) {   // sample k-2 used this stage: take its results, then refill
      // Every thread sees the commit itself, so no block barrier is needed
      // before reading the results or refilling the stage; a wait that ran
      // out is reported at the barrier below.
      ok = bars.wait(b);
      tc::fence_after_sync();
      if (ok) consume(k - 2, b);
    }
    store_split8(sm, Lay::w(b), Lay::W_PLANE, tid >> 2, tid & 3, kHexC, r.w);
    float z[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      z[i] = 0.f;
      if (valid) z[i] = r.wt[0] * r.c[0][i] + r.wt[1] * r.c[1][i] + r.wt[2] * r.c[2][i] + r.wt[3] * r.c[3][i];
    }
    store_split8(sm, Lay::z(b), Lay::Z_PLANE, row, half * 2, kHexC, z);
    store_split8(sm, Lay::z(b), Lay::Z_PLANE, row, half * 2 + 1, kHexC, z + 8);
    tc::fence_proxy_async();
    tc::fence_before_sync();
    if (__syncthreads_or(!ok)) return false;
    if (tid == 0) {
      tc::fence_after_sync();
      issue(k, b);
      tc::mma_commit(bars.addr(b));
    }
    if (k + 1 < NS) prefetch(k + 1);
    return true;
  };
  prefetch(0);
  for (int k = 0; k < NS; ++k)
    if (!step(k)) return false;
  for (int k = NS - 2; k < NS; ++k) {   // the last two samples
    const int b = k & 1;
    const bool ok = bars.wait(b);
    if (__syncthreads_or(!ok)) return false;
    tc::fence_after_sync();
    consume(k, b);
  }
  return true;
}

// grad[0..63] += the 256 bytes at shared address src, asynchronously (one
// bulk reduction); completion is tracked by this thread's bulk groups.
__device__ __forceinline__ void bulk_add_2rows(float* grad, uint32_t src) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], 256;" ::"l"(grad), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// This thread's bulk operations have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// This thread's bulk operations are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Makes every thread's shared-memory tile writes visible to the tensor core
// and lines the threads up before thread 0 issues the next MMAs.
__device__ __forceinline__ void tiles_ready() {
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
}

// Stages W2 and W3 (split, W3 padded with zero rows to 64).
__device__ __forceinline__ void stage_w23(uint8_t* sm, const float* __restrict__ W2g, const float* __restrict__ W3g) {
  using Lay = HexTcLayout;
  const int tid = threadIdx.x;
  for (int i = tid; i < kHexH * (kHexH / 8); i += kHexThreads) {
    const int r = i / (kHexH / 8), kc = i % (kHexH / 8);
    const float4* w2 = reinterpret_cast<const float4*>(W2g + r * kHexH) + 2 * kc;
    store_split8(sm, Lay::W2, Lay::S_PLANE, r, kc, kHexH, __ldg(w2), __ldg(w2 + 1));
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (r < kHexHead) {
      const float4* w3 = reinterpret_cast<const float4*>(W3g + r * kHexH) + 2 * kc;
      a = __ldg(w3);
      b = __ldg(w3 + 1);
    }
    store_split8(sm, Lay::W3, Lay::S_PLANE, r, kc, kHexH, a, b);
  }
}

// Stages W2 and W3 and the three bias vectors, once per CTA.
__device__ __forceinline__ void stage_small_layers(uint8_t* sm, int bias_off, const float* __restrict__ W2g,
                                                   const float* __restrict__ b1, const float* __restrict__ b2,
                                                   const float* __restrict__ W3g, const float* __restrict__ b3) {
  const int tid = threadIdx.x;
  stage_w23(sm, W2g, W3g);
  float* bias = reinterpret_cast<float*>(sm + bias_off);
  for (int o = tid; o < kHexH; o += kHexThreads) {
    bias[o] = __ldg(b1 + o);
    bias[kHexH + o] = __ldg(b2 + o);
    bias[2 * kHexH + o] = o < kHexHead ? __ldg(b3 + o) : 0.f;
  }
}

// ---------------------------------------------------------------------------
// Forward, warp-specialised: the tensor-core form of the layers (bf16x3
// split products, fresh accumulators per plane sample added in fp32), with
// the per-sample chain taken apart so that no step waits for the whole CTA:
//   * 8 producer warps gather the tile's corner rows and the sample's W1
//     slice into registers two plane samples ahead, interpolate, and write
//     the split z_k and W1 slice into a two-stage shared-memory ring; a ring
//     stage is full once all 8 have arrived;
//   * 4 consumer warps (one thread per Gaussian, TMEM lane = row): one lane
//     issues each sample's split MMAs into a three-stage TMEM ring and
//     commits them to the stage's "empty" and "ready" barriers; all 128 add
//     the sample's two accumulators to their fp32 row and free the TMEM
//     stage; after the last sample they run layers 2 and 3 (through the H
//     tile and TMEM columns 384..511) and write the outputs, while the
//     producers already gather the next tile.
// Every hand-off is an mbarrier with a bounded wait; the roles' own named
// barriers reduce a failure flag, so a timed-out wait ends both roles at their
// next barrier instead of leaving either waiting.
// ---------------------------------------------------------------------------
constexpr int kWsProducerWarps = 8;
constexpr int kWsProducers = 32 * kWsProducerWarps;
constexpr int kWsConsumers = kHexTile;
constexpr int kWsThreads = kWsProducers + kWsConsumers;
constexpr int kWsTStages = 3;
// Polls of one mbarrier before a wait gives up: every legitimate wait here is
// for work of microseconds (a sample's gather, its MMAs, a tile's epilogue)
constexpr uint32_t kWsWait = 1u << 20;
static_assert(2 * 4 * 32 * 184 + 4 * 32 * 136 == kWsThreads * 168, "the register split must equal the launch's total");

// A producer's corner rows of one plane sample: [Gaussian j][corner 00, 01, 10, 11]
struct CornerRegs {
  float4 c[4][4];
};

struct HexWsLayout {
  static constexpr int Z_STAGE = HexTcLayout::Z_STAGE;             // split z_k, skewed (24,960 B)
  static constexpr int W_STAGE = HexTcLayout::W_STAGE;             // split W1 slice (12,288 B)
  static constexpr int STAGE = Z_STAGE + W_STAGE;                  // one ring stage
  static constexpr int H = 2 * STAGE;                              // split H tile, 3 x 16 KB
  static constexpr int W2 = H + 3 * HexTcLayout::H_PLANE;          // split W2, 3 x 8 KB
  static constexpr int W3 = W2 + 3 * HexTcLayout::S_PLANE;         // split W3 (58 rows, padded), 3 x 8 KB
  static constexpr int BIAS = W3 + 3 * HexTcLayout::S_PLANE;       // b1 | b2 | b3
  static constexpr int BARS = BIAS + 3 * kHexH * 4;                // 12 mbarriers, then the TMEM address
  static constexpr int SMP = BARS + 128;                           // per sample and Gaussian {row, wa, wb, 0}
  static constexpr int BYTES = SMP + 24 * kHexTile * 16;
  static __device__ __forceinline__ int z(int s) { return s * STAGE; }
  static __device__ __forceinline__ int w(int s) { return s * STAGE + Z_STAGE; }
};
static_assert(HexWsLayout::STAGE % 128 == 0 && HexWsLayout::W2 % 128 == 0 && HexWsLayout::SMP % 16 == 0,
              "tile alignment");
static_assert(HexWsLayout::W2 - HexWsLayout::H == 3 * HexTcLayout::H_PLANE, "H tile size");
static_assert(HexWsLayout::BYTES <= 227 * 1024, "warp-specialised tiles exceed the shared memory of one CTA");

// mbarriers of the warp-specialised forward
enum : int { kBarFull = 0, kBarEmpty = 2, kBarReady = 4, kBarFree = 7, kBarLayer = 10, kBarFinal = 11, kNumWsBars = 12 };
static_assert(8 * kNumWsBars + 4 <= 128, "the mbarriers and the TMEM address fit their 128 bytes");

// bar.sync on a named barrier for `n` threads of one role
__device__ __forceinline__ void role_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// The same with an OR over the role's predicates: true if any thread's p was.
__device__ __forceinline__ bool role_sync_or(int id, int n, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Bounded wait by every lane of a warp, agreed across the warp.
__device__ __forceinline__ bool warp_wait(uint32_t mbar, uint32_t parity) {
  const bool ok = tc::mbar_wait_bounded(mbar, parity, kWsWait);
  return __all_sync(0xffffffffu, ok);
}

// acc[i] += main[i] + corr[i] for this thread's TMEM lane, 64 columns (four
// rounds with a main and a correction load in flight per wait).
__device__ __forceinline__ void add_partial64(uint32_t d_main, uint32_t d_corr, float acc[64]) {
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    float a[16], b[16];
    tc::tmem_ld16x2(d_main + 16 * h, d_corr + 16 * h, a, b);
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[16 * h + i] += a[i] + b[i];
  }
}

// The consumers' share of a ring stage: the W1 slice of plane sample k
// (64 rows x 32 columns), row c / 2, columns 16 (c % 2) .. + 15, loaded into
// registers a sample ahead and stored split.
__device__ __forceinline__ void load_w1_slice(const float* __restrict__ W1, int IN, int k, int c, float v[16]) {
  const float* src = W1 + (size_t)(c >> 1) * IN + k * kHexC + (c & 1) * 16;
  ld_nc_v8(src, v);
  ld_nc_v8(src + 8, v + 8);
}
__device__ __forceinline__ void store_w1_slice(uint8_t* sm, int off, int c, const float v[16]) {
  store_split8(sm, off, HexTcLayout::W_PLANE, c >> 1, (c & 1) * 2, kHexC, v);
  store_split8(sm, off, HexTcLayout::W_PLANE, c >> 1, (c & 1) * 2 + 1, kHexC, v + 8);
}
// One of 256 threads' share of a split W1 slice (64 rows x 32 columns): row
// c / 4, columns 8 (c % 4) .. + 7.
__device__ __forceinline__ void load_w1_slice8(const float* __restrict__ W1, int IN, int k, int c, float v[8]) {
  ld_nc_v8(W1 + (size_t)(c >> 2) * IN + k * kHexC + (c & 3) * 8, v);
}
__device__ __forceinline__ void store_w1_slice8(uint8_t* sm, int off, int c, const float v[8]) {
  store_split8(sm, off, HexTcLayout::W_PLANE, c >> 2, c & 3, kHexC, v);
}

__global__ void __launch_bounds__(kWsThreads, 1) hexplane_fwd_ws_kernel(
    HexParams hp, const float* __restrict__ mu, const int32_t* __restrict__ frame, int64_t N,
    const float* __restrict__ planes, const float* __restrict__ W, const float* __restrict__ q_can,
    const float* __restrict__ logs_can, const float* __restrict__ sh_can, HexOutPtrs out, float* __restrict__ latent,
    float* __restrict__ hidden) {
  using Lay = HexWsLayout;
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lid = tid & 31;
  const int IN = hp.in_dim, NS = hp.n_samples;
  const float* W1 = W;
  const float* b1 = W1 + kHexH * IN;
  const float* W2g = b1 + kHexH;
  const float* b2 = W2g + kHexH * kHexH;
  const float* W3g = b2 + kHexH;
  const float* b3 = W3g + kHexHead * kHexH;
  const uint32_t sbase = tc::smem_u32(sm);
  const uint32_t bar0 = sbase + Lay::BARS;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::BARS + 8 * kNumWsBars);
  float4* smp = reinterpret_cast<float4*>(sm + Lay::SMP);
  const float* bias = reinterpret_cast<const float*>(sm + Lay::BIAS);

  if (tid < kHexThreads) {
    // W2 | W3 split at the forward's offsets, relocated to this layout
    for (int i = tid; i < kHexH * (kHexH / 8); i += kHexThreads) {
      const int r = i / (kHexH / 8), kc = i % (kHexH / 8);
      const float4* w2 = reinterpret_cast<const float4*>(W2g + r * kHexH) + 2 * kc;
      store_split8(sm, Lay::W2, HexTcLayout::S_PLANE, r, kc, kHexH, __ldg(w2), __ldg(w2 + 1));
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (r < kHexHead) {
        const float4* w3 = reinterpret_cast<const float4*>(W3g + r * kHexH) + 2 * kc;
        a = __ldg(w3);
        b = __ldg(w3 + 1);
      }
      store_split8(sm, Lay::W3, HexTcLayout::S_PLANE, r, kc, kHexH, a, b);
    }
    float* bw = reinterpret_cast<float*>(sm + Lay::BIAS);
    for (int o = tid; o < kHexH; o += kHexThreads) {
      bw[o] = __ldg(b1 + o);
      bw[kHexH + o] = __ldg(b2 + o);
      bw[2 * kHexH + o] = o < kHexHead ? __ldg(b3 + o) : 0.f;
    }
  }
  if (warp == kWsProducerWarps) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(kBarFull + s), kWsProducerWarps);
      tc::mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int t = 0; t < kWsTStages; ++t) {
      tc::mbar_init(bar(kBarReady + t), 1);
      tc::mbar_init(bar(kBarFree + t), kWsConsumers / 32);
    }
    tc::mbar_init(bar(kBarLayer), 1);
    tc::mbar_init(bar(kBarFinal), 1);
    tc::mbar_fence_init();
  }
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if (warp < kWsProducerWarps) {
    // ------------------------------ producers ------------------------------
    // two warpgroups at 184 registers, the consumers' one at 136: together
    // exactly the 384 x 168 the block was launched with
    asm volatile("setmaxnreg.inc.sync.aligned.u32 184;" ::: "memory");
    const int row = tid & (kHexTile - 1), half = tid >> 7;
    const int sub = lid >> 3, c4 = lid & 7;
    uint32_t G = 0;   // samples this CTA has produced so far
    CornerRegs ra, rb;
    int64_t tile0 = 0;
    const uint64_t keep = l2_evict_last();
    // this thread's part of the W1 slice of the next sample to write, read one sample ahead
    float wnext[8];
    int wk = 0;
    load_w1_slice8(W1, IN, 0, tid, wnext);
    auto prefetch = [&](int k, CornerRegs& r) {
      const int64_t down = (int64_t)hp.res_a[k] * (kHexC / 4);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int g = 16 * warp + 4 * j + sub;
        if (tile0 + g < N) {
          const uint32_t crow = __float_as_uint(smp[k * kHexTile + g].x);
          const float4* p = reinterpret_cast<const float4*>(planes + (int64_t)crow * kHexC) + c4;
          r.c[j][0] = ld_nc_v4_hint(p, keep);
          r.c[j][1] = ld_nc_v4_hint(p + kHexC / 4, keep);
          r.c[j][2] = ld_nc_v4_hint(p + down, keep);
          r.c[j][3] = ld_nc_v4_hint(p + down + kHexC / 4, keep);
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) r.c[j][c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    };
    auto produce = [&](int k, CornerRegs& r) -> bool {
      const int s = G & 1;
      if (G >= 2 && !warp_wait(bar(kBarEmpty + s), ((G >> 1) + 1) & 1)) return false;
      store_w1_slice8(sm, Lay::w(s), tid, wnext);   // the slice of sample k
      wk = wk + 1 == NS ? 0 : wk + 1;
      load_w1_slice8(W1, IN, wk, tid, wnext);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int g = 16 * warp + 4 * j + sub;
        const float4 rec = smp[k * kHexTile + g];
        const float wa = rec.y, wb = rec.z;
        const float w00 = (1.0f - wa) * (1.0f - wb), w01 = wa * (1.0f - wb), w10 = (1.0f - wa) * wb, w11 = wa * wb;
        const float4 a = r.c[j][0], bb = r.c[j][1], c = r.c[j][2], d = r.c[j][3];
        float4 z;
        z.x = w00 * a.x + w01 * bb.x + w10 * c.x + w11 * d.x;
        z.y = w00 * a.y + w01 * bb.y + w10 * c.y + w11 * d.y;
        z.z = w00 * a.z + w01 * bb.z + w10 * c.z + w11 * d.z;
        z.w = w00 * a.w + w01 * bb.w + w10 * c.w + w11 * d.w;
        if (latent && tile0 + g < N) st_v4_stream(latent + (tile0 + g) * IN + k * kHexC + 4 * c4, z, l2_evict_first());
        store_split4(sm, Lay::z(s), HexTcLayout::Z_PLANE, g, 4 * c4, z);
      }
      tc::fence_proxy_async();
      __syncwarp();
      if (lid == 0) tc::mbar_arrive(bar(kBarFull + s));
      ++G;
      return true;
    };
    for (int64_t tile = blockIdx.x; tile * kHexTile < N; tile += gridDim.x) {
      // the previous tile's sample table is no longer read; a failure anywhere ends every producer here
      if (role_sync_or(1, kWsProducers, failed)) {
        failed = true;
        break;
      }
      tile0 = tile * kHexTile;
      {
        float xt[4] = {0.f, 0.f, 0.f, 0.f};
        const int64_t n = tile0 + row;
        const bool valid = n < N;
        if (valid) hex_normalise(mu, frame, n, hp, xt);
        for (int k = half; k < NS; k += 2) {
          float wa = 0.f, wb = 0.f;
          uint32_t crow = 0;
          if (valid) crow = (uint32_t)(plane_corner(xt, hp, k, wa, wb) / kHexC);
          smp[k * kHexTile + row] = make_float4(__uint_as_float(crow), wa, wb, 0.f);
        }
      }
      role_sync(1, kWsProducers);
      prefetch(0, ra);
      prefetch(1, rb);
      for (int k = 0; k < NS && !failed; k += 2) {
        if (!produce(k, ra)) {
          failed = true;
          break;
        }
        if (k + 2 < NS) prefetch(k + 2, ra);
        if (!produce(k + 1, rb)) {
          failed = true;
          break;
        }
        if (k + 3 < NS) prefetch(k + 3, rb);
      }
    }
  } else {
    // ------------------------------ consumers ------------------------------
    asm volatile("setmaxnreg.dec.sync.aligned.u32 136;" ::: "memory");
    const int c = tid - kWsProducers;                  // the tile row (Gaussian) and TMEM lane
    const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t L = tmem + 128 * kWsTStages;        // layers 2 and 3: main | correction
    const SplitOp Hk = kmajor(sbase + Lay::H, HexTcLayout::H_PLANE, kHexH);
    uint32_t G = 0, lph = 0;
    for (int64_t tile = blockIdx.x; tile * kHexTile < N; tile += gridDim.x) {
      const int64_t n = tile * kHexTile + c;
      const bool valid = n < N;
      float acc[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = 0.f;
      // ---- layer 1: issue sample k, then consume sample k - 1 ----
      for (int k = 0; k <= NS && !failed; ++k) {
        if (k < NS && c == 0) {
          const uint32_t g = G + k, s = g & 1, t = g % kWsTStages;
          bool ok = tc::mbar_wait_bounded(bar(kBarFull + s), (g >> 1) & 1, kWsWait);
          if (ok && g >= (uint32_t)kWsTStages)
            ok = tc::mbar_wait_bounded(bar(kBarFree + t), ((g / kWsTStages) - 1) & 1, kWsWait);
          if (ok) {
            tc::fence_after_sync();
            mma6(tmem + 128 * t, tmem + 128 * t + 64, kmajor_zpad(sbase + Lay::z(s), HexTcLayout::Z_PLANE),
                 kmajor(sbase + Lay::w(s), HexTcLayout::W_PLANE, kHexC), kHexC,
                 tc::idesc_bf16_f32(kHexTile, kHexH, false, false));
            tc::mma_commit(bar(kBarEmpty + s));
            tc::mma_commit(bar(kBarReady + t));
          } else {
            failed = true;
          }
        }
        __syncwarp();
        failed = __any_sync(0xffffffffu, failed);   // the issuing lane's outcome, for its whole warp
        if (k >= 1 && !failed) {
          const uint32_t g = G + k - 1, t = g % kWsTStages;
          if (!warp_wait(bar(kBarReady + t), (g / kWsTStages) & 1)) {
            failed = true;
          } else {
            tc::fence_after_sync();
            add_partial64(tmem + 128 * t + lane, tmem + 128 * t + 64 + lane, acc);
            tc::fence_before_sync();
            __syncwarp();
            if (lid == 0) tc::mbar_arrive(bar(kBarFree + t));
          }
        }
      }
      G += NS;
      // ---- h1 = relu(acc + b1) -> H; layer 2 ----
      if (!failed) {
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = fmaxf(acc[i] + bias[i], 0.f);
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) store_split8(sm, Lay::H, HexTcLayout::H_PLANE, c, kc, kHexH, acc + 8 * kc);
        if (hidden && valid) {
          float4* dst = reinterpret_cast<float4*>(hidden + n * kHexH);
#pragma unroll
          for (int q = 0; q < 16; ++q) dst[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        }
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      if (role_sync_or(2, kWsConsumers, failed)) {
        failed = true;
        break;
      }
      if (c == 0) {
        tc::fence_after_sync();
        mma6(L, L + 64, Hk, kmajor(sbase + Lay::W2, HexTcLayout::S_PLANE, kHexH), kHexH,
             tc::idesc_bf16_f32(kHexTile, kHexH, false, false));
        tc::mma_commit(bar(kBarLayer));
      }
      __syncwarp();
      failed = !warp_wait(bar(kBarLayer), lph);
      lph ^= 1u;
      tc::fence_after_sync();
      if (!failed) {
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0.f;
        add_partial64(L + lane, L + 64 + lane, acc);
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = fmaxf(acc[i] + bias[kHexH + i], 0.f);
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) store_split8(sm, Lay::H, HexTcLayout::H_PLANE, c, kc, kHexH, acc + 8 * kc);
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      if (role_sync_or(2, kWsConsumers, failed)) {
        failed = true;
        break;
      }
      // ---- the head (58 rows padded to 64) ----
      if (c == 0) {
        tc::fence_after_sync();
        mma6(L, L + 64, Hk, kmajor(sbase + Lay::W3, HexTcLayout::S_PLANE, kHexH), kHexH,
             tc::idesc_bf16_f32(kHexTile, kHexH, false, false));
        tc::mma_commit(bar(kBarLayer));
      }
      __syncwarp();
      failed = !warp_wait(bar(kBarLayer), lph);
      lph ^= 1u;
      tc::fence_after_sync();
      if (failed) continue;   // the next role_sync_or ends every consumer
      float* y = acc;
#pragma unroll
      for (int i = 0; i < 64; ++i) y[i] = bias[2 * kHexH + i];
      add_partial64(L + lane, L + 64 + lane, y);
      tc::fence_before_sync();
      if (valid) {
        const uint64_t once = l2_evict_first();
        float gw, gh, gt;
        float2 gcr;
        hex_window(hp, frame, n, gw, gh, gt, gcr);
        float qh[4], q[4], s[3], cov[6];
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const float m0 = ld_nc_hint(mu + 3 * n + i, once);
          st_hint(out.mu + 3 * n + i, gh != 0.0f ? m0 + y[i] : m0, once);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) qh[i] = ld_nc_hint(q_can + 4 * n + i, once) + y[3 + i];
        normalise_quat(qh, q);
#pragma unroll
        for (int i = 0; i < 3; ++i) s[i] = expf(ld_nc_hint(logs_can + 3 * n + i, once) + gw * y[7 + i]);
        covariance(s, q, cov);
        st_v4_stream(out.rot + 4 * n, make_float4(q[0], q[1], q[2], q[3]), once);
#pragma unroll
        for (int i = 0; i < 3; ++i) st_hint(out.scale + 3 * n + i, s[i], once);
#pragma unroll
        for (int i = 0; i < 6; ++i) st_hint(out.cov + 6 * n + i, cov[i], once);
        // the 48 SH offsets as 16-byte vectors (sh_can and out.sh are 16-byte aligned)
        const float4* shc = reinterpret_cast<const float4*>(sh_can + 48 * n);
        float* sho = out.sh + 48 * n;
        static_assert(kHexHead - 10 == 48, "48 SH coefficients");
#pragma unroll
        for (int q = 0; q < 12; ++q) {
          float4 v = ld_nc_v4_hint(shc + q, once);
          v.x += gw * y[10 + 4 * q];
          v.y += gw * y[11 + 4 * q];
          v.z += gw * y[12 + 4 * q];
          v.w += gw * y[13 + 4 * q];
          st_v4_stream(sho + 4 * q, v, once);
        }
      }
    }
    // every MMA this CTA issued is complete before the tensor memory goes
    if (c == 0) {
      tc::mma_commit(bar(kBarFinal));
      tc::mbar_wait_bounded(bar(kBarFinal), 0, kWsWait);
    }
  }

  if (failed) atomicExch(&g_hex_device_error, 1);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kWsProducerWarps) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Backward without a saved latent (the planes sampled again), one
// 128-Gaussian tile per step of a persistent CTA:
//   1. forward again (layer 1 streamed through the two stages), keeping h1
//      and h2 in registers;
//   2. the head's rows 0..15 give q' and s', and with them the head adjoint
//      dy (58 values, zero padded to 64);
//   3. dh2 = (dy W3) * [h2 > 0] and dW3 += dy^T h2, then
//      dh1 = (dh2 W2) * [h1 > 0] and dW2 += dh2^T h1 (one MMA group each);
//   4. per plane sample k, dz_k = dh1 W1_k and dW1_k += dh1^T z_k; w_c dz_k
//      goes to the sample's four bilinear corner rows by bulk reductions.
// Weight gradients are partial sums over one tile (K = 128, fresh
// accumulators) added in fp32 to the CTA's workspace slot, and bias
// gradients are warp column sums gathered in shared memory, so they do not
// depend on scheduling.  TMEM: stages as in the forward, plus the 64-row
// weight-gradient accumulators at columns 256 (main) and 320 (correction).
template <bool GATED>
__global__ void __launch_bounds__(kHexThreads, 1) hexplane_bwd_tc_kernel(
    HexParams hp, const float* __restrict__ mu, const int32_t* __restrict__ frame, int64_t N,
    const float* __restrict__ planes, const float* __restrict__ W, const float* __restrict__ q_can,
    const float* __restrict__ logs_can, HexGradPtrs go, float* __restrict__ grad_planes, float* __restrict__ ws,
    int n_params) {
  using Lay = HexTcLayout;
  using BL = HexBwdLayout;
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lid = tid & 31;
  const int row = tid & (kHexTile - 1), half = tid / kHexTile;
  const int IN = hp.in_dim;
  const float* W1 = W;
  const float* b1 = W1 + kHexH * IN;
  const float* W2g = b1 + kHexH;
  const float* b2 = W2g + kHexH * kHexH;
  const float* W3g = b2 + kHexH;
  const float* b3 = W3g + kHexHead * kHexH;
  float* slot = ws + (size_t)blockIdx.x * slot_stride(n_params);
  float* sW1 = slot;
  float* sb1 = sW1 + kHexH * IN;
  float* sW2 = sb1 + kHexH;
  float* sb2 = sW2 + kHexH * kHexH;
  float* sW3 = sb2 + kHexH;
  float* sb3 = sW3 + kHexHead * kHexH;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + BL::MISC + 16);
  const uint32_t mbar0 = tc::smem_u32(sm + BL::MISC), mbar1 = mbar0 + 8;
  const float* bias = reinterpret_cast<const float*>(sm + BL::BIAS);
  float* bacc = reinterpret_cast<float*>(sm + BL::BACC);

  for (int p = tid; p < n_params; p += kHexThreads) slot[p] = 0.f;
  stage_small_layers(sm, BL::BIAS, W2g, b1, b2, W3g, b3);
  for (int o = tid; o < 3 * kHexH; o += kHexThreads) bacc[o] = 0.f;
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(mbar0, 1);
    tc::mbar_init(mbar1, 1);
    tc::mbar_fence_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t col = (uint32_t)(half * 32);
  const uint32_t sbase = tc::smem_u32(sm);
  const int T0 = Lay::A;
  const SplitOp T0k = kmajor(sbase + T0, Lay::H_PLANE, kHexH), T0t = mnmajor(sbase + T0, Lay::H_PLANE, kHexH);
  const SplitOp T1k = kmajor(sbase + BL::T1, Lay::H_PLANE, kHexH), T1t = mnmajor(sbase + BL::T1, Lay::H_PLANE, kHexH);
  const SplitOp W2k = kmajor(sbase + Lay::W2, Lay::S_PLANE, kHexH), W2t = mnmajor(sbase + Lay::W2, Lay::S_PLANE, kHexH);
  const SplitOp W3k = kmajor(sbase + Lay::W3, Lay::S_PLANE, kHexH), W3t = mnmajor(sbase + Lay::W3, Lay::S_PLANE, kHexH);
  const uint32_t RW = tmem + 256;
  // Row m of a 64-row accumulator sits in TMEM lane (m % 16) + 32 (m / 16):
  // warp w reads rows 16 (w % 4) + lane for lanes below 16.
  const int wrow = (warp & 3) * 16 + lid;
  const bool wrow_ok = lid < 16;
  HexBars bars{mbar0, mbar1, 0u, 0u};
  bool failed = false;

  for (int64_t tile = blockIdx.x; tile * kHexTile < N; tile += gridDim.x) {
    const int64_t n = tile * kHexTile + row;
    const bool valid = n < N;
    float xt[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) hex_normalise(mu, frame, n, hp, xt);
    if (tile != blockIdx.x) stage_w23(sm, W2g, W3g);   // the last tile's scatter staging sat over them
    // ---- 1. forward ----
    float h1[32], h2[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) h1[i] = 0.f;
    auto issue1 = [&](int, int b) {
      mma6(tmem + 128 * b, tmem + 128 * b + 64, kmajor(sbase + Lay::z(b), Lay::Z_PLANE, kHexC),
           kmajor(sbase + Lay::w(b), Lay::W_PLANE, kHexC), kHexC, tc::idesc_bf16_f32(kHexTile, kHexH, false, false));
    };
    auto consume1 = [&](int, int b) { add_partial(tmem + 128 * b + lane + col, tmem + 128 * b + 64 + lane + col, h1); };
    if (!hex_stream(sm, hp, planes, W1, valid, xt, bars, issue1, consume1)) {
      failed = true;
      break;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) h1[i] = fmaxf(h1[i] + bias[half * 32 + i], 0.f);
    store_row32(sm, T0, row, half, h1);
    tiles_ready();
    if (tid == 0) {
      tc::fence_after_sync();
      mma6(tmem, tmem + 64, T0k, W2k, kHexH, tc::idesc_bf16_f32(kHexTile, kHexH, false, false));
      tc::mma_commit(mbar0);
    }
    if (__syncthreads_or(!bars.wait(0))) { failed = true; break; }
    tc::fence_after_sync();
#pragma unroll
    for (int i = 0; i < 32; ++i) h2[i] = 0.f;
    add_partial(tmem + lane + col, tmem + 64 + lane + col, h2);
#pragma unroll
    for (int i = 0; i < 32; ++i) h2[i] = fmaxf(h2[i] + bias[kHexH + half * 32 + i], 0.f);
    store_row32(sm, BL::T1, row, half, h2);
    tiles_ready();
    // head rows 0..15 (d_mu, d_q, d_logs) into stage 1's columns; with the
    // energy-flow window all 64 (d loss / d w needs the SH offsets too)
    if (tid == 0) {
      tc::fence_after_sync();
      mma6(tmem + 128, tmem + 192, T1k, W3k, kHexH, tc::idesc_bf16_f32(kHexTile, GATED ? kHexH : 16, false, false));
      tc::mma_commit(mbar0);
    }
    if (__syncthreads_or(!bars.wait(0))) { failed = true; break; }
    tc::fence_after_sync();
    // ---- 2. head adjoint ----
    float dy[32];
    float gw = 1.0f, gh = 1.0f, gt = 0.0f;
    float2 gcr = make_float2(0.f, 0.f);
    if constexpr (GATED) {
      if (valid) hex_window(hp, frame, n, gw, gh, gt, gcr);
    }
    float dldw = 0.0f;   // d loss / d w: this thread's part of the w-scaled offsets (window only)
    if (half == 0) {
      constexpr int HC = GATED ? 32 : 16;   // head columns this half reads
      float a[HC], c[HC];
      if constexpr (GATED) {
        tc::tmem_ld32(tmem + 128 + lane, a);
        tc::tmem_ld32(tmem + 192 + lane, c);
      } else {
        tc::tmem_ld16(tmem + 128 + lane, a);
        tc::tmem_ld16(tmem + 192 + lane, c);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) dy[i] = 0.f;
      if (valid) {
        float qh[4], q[4], s[3], gc[6], ds[3], dq[4], dqh[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qh[i] = __ldg(q_can + 4 * n + i) + (a[3 + i] + c[3 + i] + bias[2 * kHexH + 3 + i]);
        const float nrm = normalise_quat(qh, q);
        float dlogs_off[3];
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          dlogs_off[i] = a[7 + i] + c[7 + i] + bias[2 * kHexH + 7 + i];
          s[i] = expf(__ldg(logs_can + 3 * n + i) + gw * dlogs_off[i]);
        }
#pragma unroll
        for (int i = 0; i < 6; ++i) gc[i] = g_or0(go.cov, 6 * n + i);
#pragma unroll
        for (int i = 0; i < 3; ++i) ds[i] = g_or0(go.scale, 3 * n + i);
#pragma unroll
        for (int i = 0; i < 4; ++i) dq[i] = g_or0(go.rot, 4 * n + i);
        covariance_backward(s, q, gc, ds, dq);
        normalise_quat_backward(q, nrm, dq, dqh);
#pragma unroll
        for (int i = 0; i < 3; ++i) dy[i] = gh != 0.0f ? g_or0(go.mu, 3 * n + i) : 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) dy[3 + i] = dqh[i];
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const float dl = ds[i] * s[i];   // d loss / d(log s + w d_logs)
          dy[7 + i] = gw * dl;
          if constexpr (GATED) dldw += dl * dlogs_off[i];
        }
#pragma unroll
        for (int i = 10; i < 32; ++i) {
          const float g = g_or0(go.sh, 48 * n + (i - 10));
          dy[i] = gw * g;
          if constexpr (GATED) dldw += g * (a[i] + c[i] + bias[2 * kHexH + i]);
        }
      }
    } else {
      if constexpr (GATED) {
        float a[32], c[32];
        tc::tmem_ld32(tmem + 128 + lane + 32, a);
        tc::tmem_ld32(tmem + 192 + lane + 32, c);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float g = (valid && i < kHexHead - 32) ? g_or0(go.sh, 48 * n + 22 + i) : 0.f;
          dy[i] = gw * g;
          if (i < kHexHead - 32) dldw += g * (a[i] + c[i] + bias[2 * kHexH + 32 + i]);
        }
        reinterpret_cast<float*>(sm + BL::GSUM)[row] = dldw;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) dy[i] = (valid && i < kHexHead - 32) ? g_or0(go.sh, 48 * n + 22 + i) : 0.f;
      }
    }
    tc::fence_before_sync();
    store_row32(sm, T0, row, half, dy);
    atomicAdd(bacc + 2 * kHexH + half * 32 + lid, warp_column_sum(dy));
    tiles_ready();
    if (GATED && half == 0 && valid && hp.gate_grad) {
      // H(w) is piecewise constant: c and r receive gradient through w alone
      float gcr_out[2];
      temporal_gate_backward(gt, gcr.x, gcr.y, hp.gate_tau, dldw + reinterpret_cast<const float*>(sm + BL::GSUM)[row],
                             gcr_out);
      float2* dst = reinterpret_cast<float2*>(hp.gate_grad) + n;
      const float2 prev = *dst;
      *dst = make_float2(prev.x + gcr_out[0], prev.y + gcr_out[1]);
    }
    // ---- 3. dh2 = dy W3 (masked), dW3 = dy^T h2 ----
    if (tid == 0) {
      tc::fence_after_sync();
      mma6(tmem, tmem + 64, T0k, W3t, kHexH, tc::idesc_bf16_f32(kHexTile, kHexH, false, true));
      mma6(RW, RW + 64, T0t, T1t, kHexTile, tc::idesc_bf16_f32(64, kHexH, true, true));
      tc::mma_commit(mbar0);
    }
    if (__syncthreads_or(!bars.wait(0))) { failed = true; break; }
    tc::fence_after_sync();
    float d[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) d[i] = 0.f;
    add_partial(tmem + lane + col, tmem + 64 + lane + col, d);
#pragma unroll
    for (int i = 0; i < 32; ++i) d[i] = h2[i] > 0.f ? d[i] : 0.f;
    {
      float a[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) a[i] = 0.f;
      add_partial(RW + lane + (warp >> 2) * 32, RW + 64 + lane + (warp >> 2) * 32, a);
      if (wrow_ok && wrow < kHexHead) slot_add32(sW3 + wrow * kHexH + (warp >> 2) * 32, a);
    }
    tc::fence_before_sync();
    store_row32(sm, T0, row, half, d);
    store_row32(sm, BL::T1, row, half, h1);
    {
      float t[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) t[i] = d[i];
      atomicAdd(bacc + kHexH + half * 32 + lid, warp_column_sum(t));
    }
    tiles_ready();
    // ---- dh1 = dh2 W2 (masked), dW2 = dh2^T h1 ----
    if (tid == 0) {
      tc::fence_after_sync();
      mma6(tmem, tmem + 64, T0k, W2t, kHexH, tc::idesc_bf16_f32(kHexTile, kHexH, false, true));
      mma6(RW, RW + 64, T0t, T1t, kHexTile, tc::idesc_bf16_f32(64, kHexH, true, true));
      tc::mma_commit(mbar0);
    }
    if (__syncthreads_or(!bars.wait(0))) { failed = true; break; }
    tc::fence_after_sync();
#pragma unroll
    for (int i = 0; i < 32; ++i) d[i] = 0.f;
    add_partial(tmem + lane + col, tmem + 64 + lane + col, d);
#pragma unroll
    for (int i = 0; i < 32; ++i) d[i] = h1[i] > 0.f ? d[i] : 0.f;
    {
      float a[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) a[i] = 0.f;
      add_partial(RW + lane + (warp >> 2) * 32, RW + 64 + lane + (warp >> 2) * 32, a);
      if (wrow_ok) slot_add32(sW2 + wrow * kHexH + (warp >> 2) * 32, a);
    }
    tc::fence_before_sync();
    store_row32(sm, BL::T1, row, half, d);
    atomicAdd(bacc + half * 32 + lid, warp_column_sum(d));
    // ---- 4. per plane sample: dz_k = dh1 W1_k, dW1_k = dh1^T z_k ----
    // Stage b's TMEM columns: dz main | dz correction | dW1 main | dW1 correction (32 each).
    auto issue2 = [&](int, int b) {
      const uint32_t S = tmem + 128 * b;
      mma6(S, S + 32, T1k, mnmajor(sbase + Lay::w(b), Lay::W_PLANE, kHexC), kHexH,
           tc::idesc_bf16_f32(kHexTile, kHexC, false, true));
      mma6(S + 64, S + 96, T1t, mnmajor(sbase + Lay::z(b), Lay::Z_PLANE, kHexC), kHexTile,
           tc::idesc_bf16_f32(64, kHexC, true, true));
    };
    auto consume2 = [&](int k, int b) {
      const uint32_t S = tmem + 128 * b;
      float dz[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {   // both threads of a Gaussian read its whole dz row
        float a[16], c[16];
        tc::tmem_ld16(S + lane + 16 * h, a);
        tc::tmem_ld16(S + 32 + lane + 16 * h, c);
#pragma unroll
        for (int i = 0; i < 16; ++i) dz[16 * h + i] = a[i] + c[i];
      }
      {
        float a[16], c[16];
        tc::tmem_ld16(S + 64 + lane + (warp >> 2) * 16, a);
        tc::tmem_ld16(S + 96 + lane + (warp >> 2) * 16, c);
        tc::fence_before_sync();
        if (wrow_ok) {   // this thread alone updates these slot elements: see slot_add32
          float4* dst = reinterpret_cast<float4*>(sW1 + (size_t)wrow * IN + k * kHexC + (warp >> 2) * 16);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            atomicAdd(dst + q, make_float4(a[4 * q] + c[4 * q], a[4 * q + 1] + c[4 * q + 1],
                                           a[4 * q + 2] + c[4 * q + 2], a[4 * q + 3] + c[4 * q + 3]));
        }
      }
      if (valid) {
        // corners 2*half and 2*half + 1 are neighbouring cells along the
        // plane's first axis, so their gradient rows are contiguous: w_c * dz
        // is staged as those two 128-byte rows and added with one bulk
        // reduction
        const PlaneSample ps = plane_sample(xt, hp, k);
        bulk_wait_read();   // this thread's rows of the previous sample have been read
        uint8_t* rows = sm + BL::SCAT + row * BL::SCAT_ROW;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const float w = half ? (cc ? ps.w11 : ps.w10) : (cc ? ps.w01 : ps.w00);
          float4* d = reinterpret_cast<float4*>(rows + (2 * half + cc) * (kHexC * 4));
#pragma unroll
          for (int q = 0; q < 8; ++q) d[q] = make_float4(w * dz[4 * q], w * dz[4 * q + 1], w * dz[4 * q + 2], w * dz[4 * q + 3]);
        }
        tc::fence_proxy_async();
        bulk_add_2rows(grad_planes + (half ? ps.o10 : ps.o00), tc::smem_u32(rows + 2 * half * (kHexC * 4)));
        bulk_commit();
      }
    };
    if (!hex_stream(sm, hp, planes, W1, valid, xt, bars, issue2, consume2)) {
      failed = true;
      break;
    }
    bulk_wait_read();   // the staging rows are W2 | W3 again in the next tile
    tc::fence_before_sync();
    __syncthreads();
  }
  bulk_wait_all();

  if (failed) {
    if (tid == 0) atomicExch(&g_hex_device_error, 1);
    bars.wait(0);
    bars.wait(1);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (!failed)
    for (int o = tid; o < kHexH; o += kHexThreads) {
      sb1[o] += bacc[o];
      sb2[o] += bacc[kHexH + o];
      if (o < kHexHead) sb3[o] += bacc[2 * kHexH + o];
    }
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Backward from a saved latent, warp-specialised, in two kernels per launch:
//   A. hexplane_bwd_head_ws_kernel: per 128-Gaussian tile, layer 1 again
//      from the latent, the head adjoint and the small layers' data and
//      weight gradients; it writes the tile's dh1 = d loss / d(W1 z + b1)
//      (N x 64 fp32) to the workspace;
//   B. hexplane_bwd_dz_ws_kernel: per tile and plane sample, dz_k = dh1 W1_k
//      and dW1_k = dh1^T z_k; dz_k's four bilinear corner rows go to the plane
//      gradients by bulk reductions, dW1_k to the CTA's workspace slot.
// In both, 4 producer warps read the tile's latent rows of each plane sample
// into registers two samples ahead and write them split into a ring of z
// stages, and 8 consumer warps (two threads per Gaussian, 32 columns each;
// TMEM lane = tile row) stage the split W1 slices into the ring, issue the
// MMAs from one lane into a ring of TMEM stages and take the results out.
// Two kernels rather than one: the dz pass issues 72 small split-product
// MMAs per sample, whose latency must be hidden two samples deep, and its
// scatter staging needs 66 KB; with the small layers' tiles and weights
// beside them the ring would have only two stages.  dh1 costs 256 bytes per
// Gaussian written and read again.  Every hand-off is an mbarrier with a
// bounded wait; the consumers' named barriers reduce a failure flag.
// ---------------------------------------------------------------------------
constexpr int kBwProducerWarps = 4;
constexpr int kBwProducers = 32 * kBwProducerWarps;
constexpr int kBwConsumers = 2 * kHexTile;
constexpr int kBwThreads = kBwProducers + kBwConsumers;
static_assert(kBwProducerWarps == 4 && 4 * 32 * 152 + 8 * 32 * 176 == kBwThreads * 168 &&
                  4 * 32 * 56 + 8 * 32 * 224 == kBwThreads * 168,
              "the register splits must equal the launch's total");

// Kernel A: z ring | W1 ring | T0 | T1 | W2 | W3 | biases and sums.
struct HexBwWsLayout {
  static constexpr int Z_STAGE = HexTcLayout::Z_STAGE;             // split z_k, skewed (24,960 B)
  static constexpr int W_STAGE = HexTcLayout::W_STAGE;             // split W1 slice (12,288 B)
  static constexpr int ZR = 0;                                     // 2 z stages
  static constexpr int WR = ZR + 2 * Z_STAGE;                      // 2 W1 stages
  static constexpr int T0 = WR + 2 * W_STAGE;                      // [128][64] x 3 planes
  static constexpr int T1 = T0 + 3 * HexTcLayout::H_PLANE;         // [128][64] x 3 planes
  static constexpr int W2 = T1 + 3 * HexTcLayout::H_PLANE;         // split W2
  static constexpr int W3 = W2 + 3 * HexTcLayout::S_PLANE;         // split W3 (58 rows, padded)
  static constexpr int BIAS = W3 + 3 * HexTcLayout::S_PLANE;       // b1 | b2 | b3
  static constexpr int BACC = BIAS + 3 * kHexH * 4;                // db1 | db2 | db3 over the CTA's tiles
  static constexpr int GSUM = BACC + 3 * kHexH * 4;                // [128]: the SH half of d loss / d w
  static constexpr int BARS = GSUM + kHexTile * 4;                 // 12 mbarriers, then the TMEM address
  static constexpr int BYTES = BARS + 128;
  static __device__ __forceinline__ int z(int s) { return ZR + s * Z_STAGE; }
  static __device__ __forceinline__ int w(int s) { return WR + s * W_STAGE; }
};
static_assert(HexBwWsLayout::T0 % 128 == 0 && HexBwWsLayout::W2 % 128 == 0, "tile alignment");
static_assert(HexBwWsLayout::BYTES <= 227 * 1024, "warp-specialised backward tiles exceed the shared memory of one CTA");

// A z tile in the skewed layout read MN-major (its columns are N, its rows
// K): the 8-row groups are adjacent, the 8-column chunks kZChunk apart.
__device__ __forceinline__ SplitOp mnmajor_zpad(uint32_t base, int plane) {
  return {base, (uint32_t)plane, 128u, (uint32_t)kZChunk, 256u};
}


// W2 and W3 split (W3 padded with zero rows to 64) by threads t of nt.
__device__ __forceinline__ void stage_w23_at(uint8_t* sm, int w2, int w3, const float* __restrict__ W2g,
                                             const float* __restrict__ W3g, int t, int nt) {
  for (int i = t; i < kHexH * (kHexH / 8); i += nt) {
    const int r = i / (kHexH / 8), kc = i % (kHexH / 8);
    const float4* a2 = reinterpret_cast<const float4*>(W2g + r * kHexH) + 2 * kc;
    store_split8(sm, w2, HexTcLayout::S_PLANE, r, kc, kHexH, __ldg(a2), __ldg(a2 + 1));
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (r < kHexHead) {
      const float4* a3 = reinterpret_cast<const float4*>(W3g + r * kHexH) + 2 * kc;
      a = __ldg(a3);
      b = __ldg(a3 + 1);
    }
    store_split8(sm, w3, HexTcLayout::S_PLANE, r, kc, kHexH, a, b);
  }
}


// Kernel B: 3 z stages | 3 W1 stages | T0 (dh1) | scatter staging | barriers.
constexpr int kDzIssuerWarp = kBwProducerWarps + kBwConsumers / 32;   // warps 12 (dz) and 13 (dW1)
constexpr int kDzThreads = 32 * (kDzIssuerWarp + 2);
struct HexDzWsLayout {
  static constexpr int STAGES = 3;
  static constexpr int TSTAGES = 4;
  static constexpr int ZR = 0;
  static constexpr int WR = ZR + STAGES * HexTcLayout::Z_STAGE;
  static constexpr int T0 = WR + STAGES * HexTcLayout::W_STAGE;
  static constexpr int SCAT = T0 + 3 * HexTcLayout::H_PLANE;       // per Gaussian its 4 corner rows, padded
  static constexpr int SCAT_ROW = HexBwdLayout::SCAT_ROW;
  static constexpr int BARS = SCAT + kHexTile * SCAT_ROW;           // 16 mbarriers, then the TMEM address
  static constexpr int BYTES = BARS + 144;
  static __device__ __forceinline__ int z(int s) { return ZR + s * HexTcLayout::Z_STAGE; }
  static __device__ __forceinline__ int w(int s) { return WR + s * HexTcLayout::W_STAGE; }
};
static_assert(HexDzWsLayout::T0 % 128 == 0 && HexDzWsLayout::SCAT % 16 == 0 && HexDzWsLayout::SCAT_ROW % 16 == 0,
              "tile alignment");
static_assert(HexDzWsLayout::BYTES <= 227 * 1024, "dz-pass tiles exceed the shared memory of one CTA");
static_assert(kWsTStages * 128 + 128 <= 512 && HexDzWsLayout::TSTAGES * 128 <= 512, "TMEM columns");
// mbarriers of kernel B
enum : int { kDzFull = 0, kDzEmpty = 3, kDzReady = 6, kDzFree = 10, kDzT0 = 14, kDzFinal = 15, kNumDzBars = 16 };
static_assert(8 * kNumDzBars + 4 <= 144, "the mbarriers and the TMEM address fit their 144 bytes");

// The producers of both backward kernels: the latent rows of every plane
// sample of this CTA's tiles, in tile order, into a ring of S split z stages
// at zring (with W_TOO, the sample's split W1 slice into the ring of W
// stages at wring as well); a stage is written once the MMAs of the sample S
// before it are done (its "empty" barrier) and then announced on its "full"
// barrier.  Global loads run two samples ahead in registers.  Returns false
// if a wait ran out.
template <int S, bool W_TOO>
__device__ __forceinline__ bool bw_stream_latent(uint8_t* sm, int zring, int wring, uint32_t full0, uint32_t empty0,
                                                 const float* __restrict__ latent, const float* __restrict__ W1,
                                                 int64_t N, int IN, int NS, uint32_t total) {
  const int warp = threadIdx.x >> 5, lid = threadIdx.x & 31;
  const int sub = lid >> 3, c4 = lid & 7;
  const uint64_t once = l2_evict_first();
  int64_t ptile = blockIdx.x;
  int pk = 0;   // the next sample to read: tile ptile, plane sample pk
  float4 ra[8], rb[8];
  float wa[W_TOO ? 16 : 1], wb[W_TOO ? 16 : 1];
  auto prefetch = [&](float4 (&r)[8], float (&w)[W_TOO ? 16 : 1]) {
    if constexpr (W_TOO) load_w1_slice(W1, IN, pk, threadIdx.x, w);
    const int64_t tile0 = ptile * kHexTile;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t n = tile0 + 32 * warp + 4 * j + sub;
      r[j] = n < N ? ld_nc_v4_hint(reinterpret_cast<const float4*>(latent + n * IN + pk * kHexC) + c4, once)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (++pk == NS) {
      pk = 0;
      ptile += gridDim.x;
    }
  };
  uint32_t G = 0;   // samples written so far
  auto produce = [&](const float4 (&r)[8], const float (&w)[W_TOO ? 16 : 1]) -> bool {
    const uint32_t s = G % S;
    if (G >= (uint32_t)S && !warp_wait(empty0 + 8u * s, ((G / S) - 1) & 1)) return false;
    if constexpr (W_TOO) store_w1_slice(sm, wring + (int)s * HexTcLayout::W_STAGE, threadIdx.x, w);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      store_split4(sm, zring + (int)s * HexTcLayout::Z_STAGE, HexTcLayout::Z_PLANE, 32 * warp + 4 * j + sub, 4 * c4,
                   r[j]);
    tc::fence_proxy_async();
    __syncwarp();
    if (lid == 0) tc::mbar_arrive(full0 + 8u * s);
    ++G;
    return true;
  };
  prefetch(ra, wa);
  prefetch(rb, wb);
  for (uint32_t g = 0; g < total; g += 2) {
    if (!produce(ra, wa)) return false;
    prefetch(ra, wa);
    if (g + 1 < total) {
      if (!produce(rb, wb)) return false;
      prefetch(rb, wb);
    }
  }
  return true;
}

// Kernel A, the head of the backward from a saved latent: per tile, layer 1
// again (z from the latent through the two-stage ring), h1 and h2, the head
// adjoint dy, dh2 = (dy W3) * [h2 > 0] with dW3 = dy^T h2, and
// dh1 = (dh2 W2) * [h1 > 0] with dW2 = dh2^T h1; it writes dh1 to dh1_out
// (N x 64) and adds the weight and bias gradients of W2, W3 and the biases to
// the CTA's workspace slot, which it zeroes first.
template <bool GATED, bool HIDDEN>
__global__ void __launch_bounds__(kBwThreads, 1) hexplane_bwd_head_ws_kernel(
    HexParams hp, const float* __restrict__ mu, const int32_t* __restrict__ frame, int64_t N,
    const float* __restrict__ W, const float* __restrict__ q_can, const float* __restrict__ logs_can,
    const float* __restrict__ latent, const float* __restrict__ hidden, HexGradPtrs go, float* __restrict__ dh1_out,
    float* __restrict__ ws, int n_params) {
  using Lay = HexBwWsLayout;
  using TL = HexTcLayout;
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lid = tid & 31;
  const int IN = hp.in_dim, NS = hp.n_samples;
  const float* W1 = W;
  const float* b1 = W1 + kHexH * IN;
  const float* W2g = b1 + kHexH;
  const float* b2 = W2g + kHexH * kHexH;
  const float* W3g = b2 + kHexH;
  const float* b3 = W3g + kHexHead * kHexH;
  float* slot = ws + (size_t)blockIdx.x * slot_stride(n_params);
  const uint32_t sbase = tc::smem_u32(sm);
  const uint32_t bar0 = sbase + Lay::BARS;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::BARS + 8 * kNumWsBars);
  const float* bias = reinterpret_cast<const float*>(sm + Lay::BIAS);
  float* bacc = reinterpret_cast<float*>(sm + Lay::BACC);
  // tiles of this CTA and the samples they pass through the ring
  const int64_t ntiles = (N + kHexTile - 1) / kHexTile;
  const int64_t my_tiles = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
  const uint32_t total = (uint32_t)(my_tiles * NS);

  for (int p = tid; p < n_params; p += kBwThreads) slot[p] = 0.f;
  stage_w23_at(sm, Lay::W2, Lay::W3, W2g, W3g, tid, kBwThreads);
  {
    float* bw = reinterpret_cast<float*>(sm + Lay::BIAS);
    for (int o = tid; o < kHexH; o += kBwThreads) {
      bw[o] = __ldg(b1 + o);
      bw[kHexH + o] = __ldg(b2 + o);
      bw[2 * kHexH + o] = o < kHexHead ? __ldg(b3 + o) : 0.f;
    }
    for (int o = tid; o < 3 * kHexH; o += kBwThreads) bacc[o] = 0.f;
  }
  if (warp == kBwProducerWarps) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(kBarFull + s), kBwProducerWarps + kBwConsumers / 32);
      tc::mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int t = 0; t < kWsTStages; ++t) {
      tc::mbar_init(bar(kBarReady + t), 1);
      tc::mbar_init(bar(kBarFree + t), kBwConsumers / 32);
    }
    tc::mbar_init(bar(kBarLayer), 1);
    tc::mbar_init(bar(kBarFinal), 1);
    tc::mbar_fence_init();
  }
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if (warp < kBwProducerWarps) {
    // ------------------------------ producers ------------------------------
    // with the saved h1 the producers have nothing to do: their registers go
    // to the consumers (4 x 32 x 56 + 8 x 32 x 224 = 384 x 168)
    if constexpr (HIDDEN)
      asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    else
      asm volatile("setmaxnreg.dec.sync.aligned.u32 152;" ::: "memory");
    if constexpr (!HIDDEN)
      failed = !bw_stream_latent<2, false>(sm, Lay::ZR, 0, bar(kBarFull), bar(kBarEmpty), latent, nullptr, N, IN, NS,
                                           total);
  } else {
    // ------------------------------ consumers ------------------------------
    if constexpr (HIDDEN)
      asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    else
      asm volatile("setmaxnreg.inc.sync.aligned.u32 176;" ::: "memory");
    const int ct = tid - kBwProducers;                 // 0 .. 255
    const int row = ct & (kHexTile - 1), half = ct >> 7;
    const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t col = (uint32_t)(half * 32);
    const uint32_t L = tmem + 128 * kWsTStages;        // small layers: main | correction
    const uint32_t RW = tmem;                          // their weight gradients (64-row layout): the ring is idle then
    // Row m of a 64-row accumulator sits in TMEM lane (m % 16) + 32 (m / 16):
    // lanes below 16 of warp w hold rows 16 (w % 4) + lane.
    const int wrow = (warp & 3) * 16 + lid;
    const bool wrow_ok = lid < 16;
    const bool issuer = ct == 0;
    float* sW1 = slot;
    float* sW2 = sW1 + kHexH * IN + kHexH;
    float* sW3 = sW2 + kHexH * kHexH + kHexH;
    const SplitOp T0k = kmajor(sbase + Lay::T0, TL::H_PLANE, kHexH), T0t = mnmajor(sbase + Lay::T0, TL::H_PLANE, kHexH);
    const SplitOp T1k = kmajor(sbase + Lay::T1, TL::H_PLANE, kHexH), T1t = mnmajor(sbase + Lay::T1, TL::H_PLANE, kHexH);
    const SplitOp W2k = kmajor(sbase + Lay::W2, TL::S_PLANE, kHexH), W2t = mnmajor(sbase + Lay::W2, TL::S_PLANE, kHexH);
    const SplitOp W3k = kmajor(sbase + Lay::W3, TL::S_PLANE, kHexH), W3t = mnmajor(sbase + Lay::W3, TL::S_PLANE, kHexH);
    uint32_t G = 0, lph = 0;
    // W1 slices of the first two ring samples; wreg then holds the next (sample 2)
    float wreg[8];
    if constexpr (!HIDDEN) {
      for (int s = 0; s < 2; ++s) {
        load_w1_slice8(W1, IN, s, ct, wreg);
        store_w1_slice8(sm, Lay::w(s), ct, wreg);
        tc::fence_proxy_async();
        __syncwarp();
        if (lid == 0) tc::mbar_arrive(bar(kBarFull + s));
      }
      load_w1_slice8(W1, IN, 2, ct, wreg);
    }
    // with the saved h1: this thread's half row of the next tile's
    float hn[HIDDEN ? 32 : 1];
    auto load_h1 = [&](int64_t tile) {
      if constexpr (HIDDEN) {
        const int64_t m = tile * kHexTile + row;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = m < N ? __ldg(reinterpret_cast<const float4*>(hidden + m * kHexH + half * 32) + q)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
          hn[4 * q] = v.x;
          hn[4 * q + 1] = v.y;
          hn[4 * q + 2] = v.z;
          hn[4 * q + 3] = v.w;
        }
      }
    };
    load_h1(blockIdx.x);

    // Ring sample g: its MMAs by the issuing lane once its stage is full and its TMEM stage free.
    auto issue = [&](uint32_t g, auto&& mmas) {
      const uint32_t s = g & 1, t = g % kWsTStages;
      bool ok = tc::mbar_wait_bounded(bar(kBarFull + s), (g >> 1) & 1, kWsWait);
      if (ok && g >= (uint32_t)kWsTStages)
        ok = tc::mbar_wait_bounded(bar(kBarFree + t), ((g / kWsTStages) - 1) & 1, kWsWait);
      if (ok) {
        tc::fence_after_sync();
        mmas(s, tmem + 128 * t);
        tc::mma_commit(bar(kBarEmpty + s));
        tc::mma_commit(bar(kBarReady + t));
      }
      return ok;
    };
    // After sample g's TMEM stage is read: free it, and put the W1 slice of
    // sample g + 2 into g's ring stage (g's MMAs are done with it).
    auto release = [&](uint32_t g) {
      tc::fence_before_sync();
      __syncwarp();
      if (lid == 0) tc::mbar_arrive(bar(kBarFree + g % kWsTStages));
      if (g + 2 < total) {
        store_w1_slice8(sm, Lay::w(g & 1), ct, wreg);
        tc::fence_proxy_async();
        __syncwarp();
        if (lid == 0) tc::mbar_arrive(bar(kBarFull + (g & 1)));
        load_w1_slice8(W1, IN, (int)((g + 3) % (uint32_t)NS), ct, wreg);
      }
    };

    for (int64_t tile = blockIdx.x; tile * kHexTile < N; tile += gridDim.x) {
      const int64_t n = tile * kHexTile + row;
      const bool valid = n < N;
      float xt[4] = {0.f, 0.f, 0.f, 0.f};
      if (valid) hex_normalise(mu, frame, n, hp, xt);
      // ---- 1. layer 1 again (or the saved h1): issue sample k, then add sample k - 1 ----
      float h1[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) h1[i] = 0.f;
      if constexpr (HIDDEN) {
#pragma unroll
        for (int i = 0; i < 32; ++i) h1[i] = hn[i];
        if ((tile + gridDim.x) * kHexTile < N) load_h1(tile + gridDim.x);
      }
      for (int k = 0; !HIDDEN && k <= NS && !failed; ++k) {
        if (k < NS && issuer)
          failed = !issue(G + k, [&](uint32_t s, uint32_t S) {
            mma6(S, S + 64, kmajor_zpad(sbase + Lay::z(s), TL::Z_PLANE), kmajor(sbase + Lay::w(s), TL::W_PLANE, kHexC),
                 kHexC, tc::idesc_bf16_f32(kHexTile, kHexH, false, false));
          });
        __syncwarp();
        failed = __any_sync(0xffffffffu, failed);
        if (k >= 1 && !failed) {
          const uint32_t g = G + k - 1, t = g % kWsTStages;
          if (!warp_wait(bar(kBarReady + t), (g / kWsTStages) & 1)) {
            failed = true;
          } else {
            tc::fence_after_sync();
            add_partial(tmem + 128 * t + lane + col, tmem + 128 * t + 64 + lane + col, h1);
            release(g);
          }
        }
      }
      G += NS;
      // ---- 2. h1, h2 and the head ----
      if constexpr (!HIDDEN) {
#pragma unroll
        for (int i = 0; i < 32; ++i) h1[i] = fmaxf(h1[i] + bias[half * 32 + i], 0.f);
      }
      store_row32(sm, Lay::T0, row, half, h1);
      tc::fence_proxy_async();
      tc::fence_before_sync();
      if (role_sync_or(2, kBwConsumers, failed)) {
        failed = true;
        break;
      }
      if (issuer) {
        tc::fence_after_sync();
        mma6(L, L + 64, T0k, W2k, kHexH, tc::idesc_bf16_f32(kHexTile, kHexH, false, false));
        tc::mma_commit(bar(kBarLayer));
      }
      __syncwarp();
      failed = !warp_wait(bar(kBarLayer), lph);
      lph ^= 1u;
      tc::fence_after_sync();
      uint32_t m2 = 0;   // bit i: h2 column half * 32 + i is positive
      {
        float h2[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) h2[i] = 0.f;
        if (!failed) add_partial(L + lane + col, L + 64 + lane + col, h2);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          h2[i] = fmaxf(h2[i] + bias[kHexH + half * 32 + i], 0.f);
          m2 |= (h2[i] > 0.f ? 1u : 0u) << i;
        }
        store_row32(sm, Lay::T1, row, half, h2);
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      if (role_sync_or(2, kBwConsumers, failed)) {
        failed = true;
        break;
      }
      // head rows 0..15 (d_mu, d_q, d_logs); with the energy-flow window all
      // 64 (d loss / d w needs the SH offsets too)
      if (issuer) {
        tc::fence_after_sync();
        mma6(L, L + 64, T1k, W3k, kHexH, tc::idesc_bf16_f32(kHexTile, GATED ? kHexH : 16, false, false));
        tc::mma_commit(bar(kBarLayer));
      }
      __syncwarp();
      failed = !warp_wait(bar(kBarLayer), lph);
      lph ^= 1u;
      tc::fence_after_sync();
      // ---- 3. head adjoint ----
      float dy[32];
      float gw = 1.0f, gh = 1.0f, gt = 0.0f;
      float2 gcr = make_float2(0.f, 0.f);
      if constexpr (GATED) {
        if (valid) hex_window(hp, frame, n, gw, gh, gt, gcr);
      }
      float dldw = 0.0f;   // d loss / d w: this thread's part of the w-scaled offsets (window only)
#pragma unroll
      for (int i = 0; i < 32; ++i) dy[i] = 0.f;
      // this thread's head outputs: columns half * 32 .. (the first 16 of half 0 without the window)
      constexpr int HC = GATED ? 32 : 16;
      float y[HC];
      if (GATED || half == 0) {
#pragma unroll
        for (int h = 0; h < HC / 16; ++h) {
          float a[16], c[16];
          tc::tmem_ld16x2(L + lane + col + 16 * h, L + 64 + lane + col + 16 * h, a, c);
#pragma unroll
          for (int i = 0; i < 16; ++i) y[16 * h + i] = a[i] + c[i] + bias[2 * kHexH + half * 32 + 16 * h + i];
        }
      }
      if (half == 0) {
        if (valid && !failed) {
          float qh[4], q[4], s[3], gc[6], ds[3], dq[4], dqh[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) qh[i] = __ldg(q_can + 4 * n + i) + y[3 + i];
          const float nrm = normalise_quat(qh, q);
#pragma unroll
          for (int i = 0; i < 3; ++i) s[i] = expf(__ldg(logs_can + 3 * n + i) + gw * y[7 + i]);
#pragma unroll
          for (int i = 0; i < 6; ++i) gc[i] = g_or0(go.cov, 6 * n + i);
#pragma unroll
          for (int i = 0; i < 3; ++i) ds[i] = g_or0(go.scale, 3 * n + i);
#pragma unroll
          for (int i = 0; i < 4; ++i) dq[i] = g_or0(go.rot, 4 * n + i);
          covariance_backward(s, q, gc, ds, dq);
          normalise_quat_backward(q, nrm, dq, dqh);
#pragma unroll
          for (int i = 0; i < 3; ++i) dy[i] = gh != 0.0f ? g_or0(go.mu, 3 * n + i) : 0.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i) dy[3 + i] = dqh[i];
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            const float dl = ds[i] * s[i];   // d loss / d(log s + w d_logs)
            dy[7 + i] = gw * dl;
            if constexpr (GATED) dldw += dl * y[7 + i];
          }
#pragma unroll
          for (int i = 10; i < 32; ++i) {
            const float g = g_or0(go.sh, 48 * n + (i - 10));
            dy[i] = gw * g;
            if constexpr (GATED) dldw += g * y[i];
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float g = (valid && i < kHexHead - 32) ? g_or0(go.sh, 48 * n + 22 + i) : 0.f;
          dy[i] = gw * g;
          if constexpr (GATED) {
            if (i < kHexHead - 32) dldw += g * y[i];
          }
        }
        if constexpr (GATED) reinterpret_cast<float*>(sm + Lay::GSUM)[row] = dldw;
      }
      tc::fence_before_sync();
      store_row32(sm, Lay::T0, row, half, dy);
      atomicAdd(bacc + 2 * kHexH + half * 32 + lid, warp_column_sum(dy));
      tc::fence_proxy_async();
      tc::fence_before_sync();
      if (role_sync_or(2, kBwConsumers, failed)) {
        failed = true;
        break;
      }
      if (GATED && half == 0 && valid && hp.gate_grad) {
        // H(w) is piecewise constant: c and r receive gradient through w alone
        float gcr_out[2];
        temporal_gate_backward(gt, gcr.x, gcr.y, hp.gate_tau, dldw + reinterpret_cast<const float*>(sm + Lay::GSUM)[row],
                               gcr_out);
        float2* dst = reinterpret_cast<float2*>(hp.gate_grad) + n;
        const float2 prev = *dst;
        *dst = make_float2(prev.x + gcr_out[0], prev.y + gcr_out[1]);
      }
      // ---- 4. dh2 = (dy W3) * [h2 > 0], dW3 = dy^T h2 ----
      if (issuer) {
        tc::fence_after_sync();
        mma6(L, L + 64, T0k, W3t, kHexH, tc::idesc_bf16_f32(kHexTile, kHexH, false, true));
        mma6(RW, RW + 64, T0t, T1t, kHexTile, tc::idesc_bf16_f32(64, kHexH, true, true));
        tc::mma_commit(bar(kBarLayer));
      }
      __syncwarp();
      failed = !warp_wait(bar(kBarLayer), lph);
      lph ^= 1u;
      tc::fence_after_sync();
      {
        float d[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) d[i] = 0.f;
        if (!failed) add_partial(L + lane + col, L + 64 + lane + col, d);
#pragma unroll
        for (int i = 0; i < 32; ++i) d[i] = (m2 >> i) & 1u ? d[i] : 0.f;
        {
          float a[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = 0.f;
          if (!failed) add_partial(RW + lane + col, RW + 64 + lane + col, a);
          if (!failed && wrow_ok && wrow < kHexHead) slot_add32(sW3 + wrow * kHexH + half * 32, a);
        }
        tc::fence_before_sync();
        store_row32(sm, Lay::T0, row, half, d);
        store_row32(sm, Lay::T1, row, half, h1);
        atomicAdd(bacc + kHexH + half * 32 + lid, warp_column_sum(d));
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      if (role_sync_or(2, kBwConsumers, failed)) {
        failed = true;
        break;
      }
      // ---- 5. dh1 = (dh2 W2) * [h1 > 0], dW2 = dh2^T h1 ----
      if (issuer) {
        tc::fence_after_sync();
        mma6(L, L + 64, T0k, W2t, kHexH, tc::idesc_bf16_f32(kHexTile, kHexH, false, true));
        mma6(RW, RW + 64, T0t, T1t, kHexTile, tc::idesc_bf16_f32(64, kHexH, true, true));
        tc::mma_commit(bar(kBarLayer));
      }
      __syncwarp();
      failed = !warp_wait(bar(kBarLayer), lph);
      lph ^= 1u;
      tc::fence_after_sync();
      {
        float d[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) d[i] = 0.f;
        if (!failed) add_partial(L + lane + col, L + 64 + lane + col, d);
#pragma unroll
        for (int i = 0; i < 32; ++i) d[i] = h1[i] > 0.f ? d[i] : 0.f;
        {
          float a[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = 0.f;
          if (!failed) add_partial(RW + lane + col, RW + 64 + lane + col, a);
          if (!failed && wrow_ok) slot_add32(sW2 + wrow * kHexH + half * 32, a);
        }
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(dh1_out + n * kHexH + half * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[q] = make_float4(d[4 * q], d[4 * q + 1], d[4 * q + 2], d[4 * q + 3]);
        }
        atomicAdd(bacc + half * 32 + lid, warp_column_sum(d));
      }
      // the weight-gradient columns (ring stage 0) are read before the next tile's MMAs
      tc::fence_before_sync();
      if (role_sync_or(2, kBwConsumers, failed)) {
        failed = true;
        break;
      }
    }
    // every MMA this CTA issued is complete before the tensor memory goes
    if (issuer) {
      tc::mma_commit(bar(kBarFinal));
      tc::mbar_wait_bounded(bar(kBarFinal), 0, kWsWait);
    }
  }

  if (failed) atomicExch(&g_hex_device_error, 1);
  tc::fence_before_sync();
  __syncthreads();
  if (!failed) {
    float* sb1 = slot + kHexH * IN;
    float* sb2 = sb1 + kHexH + kHexH * kHexH;
    float* sb3 = sb2 + kHexH + kHexHead * kHexH;
    for (int o = tid; o < kHexH; o += kBwThreads) {
      sb1[o] += bacc[o];
      sb2[o] += bacc[kHexH + o];
      if (o < kHexHead) sb3[o] += bacc[2 * kHexH + o];
    }
  }
  if (warp == kBwProducerWarps) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Kernel B, the W1 pass of the backward from a saved latent: per tile, T0 =
// dh1 (from kernel A), then per plane sample k the split MMAs
//   dz_k [128 x 32]  = dh1 W1_k        (TMEM stage columns 0..63)
//   dW1_k [64 x 32]  = dh1^T z_k       (columns 64..127, 64-row layout)
// Roles: 4 producer warps write z_k and the W1 slice into the three-stage
// ring; two issuer warps (the dz products and the dW1 products, so that the
// single-thread issue of 72 small MMAs per sample is shared) issue each
// sample's MMAs as soon as its ring stage is full and its TMEM stage (of
// four) free, so the tensor core runs up to four samples ahead; 8 consumer
// warps take dz_k and dW1_k out of TMEM, scatter w_c dz_k to the plane
// gradients by bulk reductions and add dW1_k to the CTA's workspace slot
// (zeroed by kernel A, which ran first on the same grid).  The consumers write T0 for the next tile once they have taken out
// every sample of the last one, and announce it on the T0 barrier.
__global__ void __launch_bounds__(kDzThreads, 1) hexplane_bwd_dz_ws_kernel(
    HexParams hp, const float* __restrict__ mu, const int32_t* __restrict__ frame, int64_t N,
    const float* __restrict__ W1, const float* __restrict__ latent, const float* __restrict__ dh1,
    float* __restrict__ grad_planes, float* __restrict__ ws, int n_params) {
  using Lay = HexDzWsLayout;
  using TL = HexTcLayout;
  constexpr int S = Lay::STAGES, TS = Lay::TSTAGES;
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lid = tid & 31;
  const int IN = hp.in_dim, NS = hp.n_samples;
  float* sW1 = ws + (size_t)blockIdx.x * slot_stride(n_params);
  const uint32_t sbase = tc::smem_u32(sm);
  const uint32_t bar0 = sbase + Lay::BARS;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::BARS + 8 * kNumDzBars);
  const int64_t ntiles = (N + kHexTile - 1) / kHexTile;
  const int64_t my_tiles = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
  const uint32_t total = (uint32_t)(my_tiles * NS);

  if (warp == kDzIssuerWarp) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(bar(kDzFull + s), kBwProducerWarps);
      tc::mbar_init(bar(kDzEmpty + s), 2);   // both issuers commit
    }
    for (int t = 0; t < TS; ++t) {
      tc::mbar_init(bar(kDzReady + t), 2);
      tc::mbar_init(bar(kDzFree + t), kBwConsumers / 32);
    }
    tc::mbar_init(bar(kDzT0), kBwConsumers / 32);
    tc::mbar_init(bar(kDzFinal), 2);
    tc::mbar_fence_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if (warp < kBwProducerWarps) {
    // ------------------------------ producers ------------------------------
    failed = !bw_stream_latent<S, true>(sm, Lay::ZR, Lay::WR, bar(kDzFull), bar(kDzEmpty), latent, W1, N, IN, NS,
                                        total);
  } else if (warp >= kDzIssuerWarp) {
    // ------------------------------- issuers -------------------------------
    // One lane of each issuer warp: warp 12 issues the dz products, warp 13
    // the dW1 products, and each commits its own to the stage's barriers (a
    // commit tracks the MMAs its thread issued).
    if (lid == 0) {
      const SplitOp T0k = kmajor(sbase + Lay::T0, TL::H_PLANE, kHexH);
      const SplitOp T0t = mnmajor(sbase + Lay::T0, TL::H_PLANE, kHexH);
      uint32_t g = 0;
      for (int64_t i = 0; i < my_tiles && !failed; ++i) {
        if (!tc::mbar_wait_bounded(bar(kDzT0), (uint32_t)i & 1u, kWsWait)) {
          failed = true;
          break;
        }
        for (int k = 0; k < NS; ++k, ++g) {
          const uint32_t s = g % S, t = g % TS;
          bool ok = tc::mbar_wait_bounded(bar(kDzFull + s), (g / S) & 1, kWsWait);
          if (ok && g >= (uint32_t)TS) ok = tc::mbar_wait_bounded(bar(kDzFree + t), ((g / TS) - 1) & 1, kWsWait);
          if (!ok) {
            failed = true;
            break;
          }
          tc::fence_after_sync();
          const uint32_t D = tmem + 128 * t;
          if (warp == kDzIssuerWarp)
            mma6(D, D + 32, T0k, mnmajor(sbase + Lay::w(s), TL::W_PLANE, kHexC), kHexH,
                 tc::idesc_bf16_f32(kHexTile, kHexC, false, true));
          else
            mma6(D + 64, D + 96, T0t, mnmajor_zpad(sbase + Lay::z(s), TL::Z_PLANE), kHexTile,
                 tc::idesc_bf16_f32(64, kHexC, true, true));
          tc::mma_commit(bar(kDzEmpty + s));
          tc::mma_commit(bar(kDzReady + t));
        }
      }
      // every MMA this CTA issued is complete before the tensor memory goes
      tc::mma_commit(bar(kDzFinal));
      tc::mbar_wait_bounded(bar(kDzFinal), 0, kWsWait);
    }
    __syncwarp();
  } else {
    // ------------------------------ consumers ------------------------------
    const int ct = tid - kBwProducers;                 // 0 .. 255
    const int row = ct & (kHexTile - 1), half = ct >> 7;
    const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
    // Row m of a 64-row accumulator sits in TMEM lane (m % 16) + 32 (m / 16):
    // lanes below 16 of warp w hold rows 16 (w % 4) + lane.
    const int wrow = (warp & 3) * 16 + lid;
    const bool wrow_ok = lid < 16;
    uint8_t* rows = sm + Lay::SCAT + row * Lay::SCAT_ROW;
    // this thread's half row of the next tile's dh1
    float dn[32];
    auto load_dh1 = [&](int64_t tile) {
      const int64_t n = tile * kHexTile + row;
      const bool ok = n < N;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v = ok ? __ldg(reinterpret_cast<const float4*>(dh1 + n * kHexH + half * 32) + q)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        dn[4 * q] = v.x;
        dn[4 * q + 1] = v.y;
        dn[4 * q + 2] = v.z;
        dn[4 * q + 3] = v.w;
      }
    };
    uint32_t g = 0;
    load_dh1(blockIdx.x);
    for (int64_t tile = blockIdx.x; tile * kHexTile < N && !failed; tile += gridDim.x) {
      const int64_t n = tile * kHexTile + row;
      const bool valid = n < N;
      float xt[4] = {0.f, 0.f, 0.f, 0.f};
      if (valid) hex_normalise(mu, frame, n, hp, xt);
      // T0 = dh1 of this tile: this warp has taken out every sample of the
      // last tile, so their MMAs, the last readers of T0, are done
      store_row32(sm, Lay::T0, row, half, dn);
      if ((tile + gridDim.x) * kHexTile < N) load_dh1(tile + gridDim.x);
      tc::fence_proxy_async();
      __syncwarp();
      if (lid == 0) tc::mbar_arrive(bar(kDzT0));
      for (int k = 0; k < NS; ++k, ++g) {
        const uint32_t t = g % TS;
        const uint32_t D = tmem + 128 * t;
        if (!warp_wait(bar(kDzReady + t), (g / TS) & 1)) {
          failed = true;
          break;
        }
        tc::fence_after_sync();
        float dz[32], wa[16], wc[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {   // both threads of a Gaussian read its whole dz row
          float a[16], c[16];
          tc::tmem_ld16x2(D + lane + 16 * h, D + 32 + lane + 16 * h, a, c);
#pragma unroll
          for (int i = 0; i < 16; ++i) dz[16 * h + i] = a[i] + c[i];
        }
        tc::tmem_ld16x2(D + 64 + lane + half * 16, D + 96 + lane + half * 16, wa, wc);
        tc::fence_before_sync();
        __syncwarp();
        if (lid == 0) tc::mbar_arrive(bar(kDzFree + t));
        if (wrow_ok) {   // this thread alone updates these slot elements: see slot_add32
          float4* dst = reinterpret_cast<float4*>(sW1 + (size_t)wrow * IN + k * kHexC + half * 16);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            atomicAdd(dst + q, make_float4(wa[4 * q] + wc[4 * q], wa[4 * q + 1] + wc[4 * q + 1],
                                           wa[4 * q + 2] + wc[4 * q + 2], wa[4 * q + 3] + wc[4 * q + 3]));
        }
        if (valid) {
          // corners 2 half and 2 half + 1 are neighbouring cells along the
          // plane's first axis, so their gradient rows are contiguous: w_c dz
          // is staged as those two 128-byte rows and added with one bulk
          // reduction
          const PlaneSample ps = plane_sample(xt, hp, k);
          bulk_wait_read();   // this thread's rows of the previous sample have been read
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const float w = half ? (cc ? ps.w11 : ps.w10) : (cc ? ps.w01 : ps.w00);
            float4* d = reinterpret_cast<float4*>(rows + (2 * half + cc) * (kHexC * 4));
#pragma unroll
            for (int q = 0; q < 8; ++q)
              d[q] = make_float4(w * dz[4 * q], w * dz[4 * q + 1], w * dz[4 * q + 2], w * dz[4 * q + 3]);
          }
          tc::fence_proxy_async();
          bulk_add_2rows(grad_planes + (half ? ps.o10 : ps.o00), tc::smem_u32(rows + 2 * half * (kHexC * 4)));
          bulk_commit();
        }
      }
    }
    bulk_wait_all();
  }

  if (failed) atomicExch(&g_hex_device_error, 1);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kDzIssuerWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

static const int kAxes[6][2] = {{0, 1}, {0, 2}, {1, 2}, {0, 3}, {1, 3}, {2, 3}};   // XY XZ YZ XT YT ZT

static HexParams make_hex_params(const spin4d_hexplane_desc* h) {
  HexParams p;
  memset(&p, 0, sizeof(p));
  p.n_samples = h->n_scales * 6;
  p.in_dim = p.n_samples * h->channels;
  p.frames_m1 = (float)(h->n_frames - 1);
  int64_t off = 0;
  for (int s = 0; s < h->n_scales; ++s)
    for (int q = 0; q < 6; ++q) {
      const int k = s * 6 + q;
      p.axis_a[k] = kAxes[q][0];
      p.axis_b[k] = kAxes[q][1];
      p.res_a[k] = h->scales[s];
      p.res_b[k] = kAxes[q][1] == 3 ? h->time_res : h->scales[s];
      p.scale_a[k] = (float)(p.res_a[k] - 1);
      p.scale_b[k] = (float)(p.res_b[k] - 1);
      p.off[k] = off;
      off += (int64_t)p.res_a[k] * p.res_b[k] * h->channels;
    }
  return p;
}

static int hex_supported(const spin4d_hexplane_desc* h) {
  return (h->channels == kHexC && h->hidden == kHexH && h->n_hidden == 2) ? SPIN4D_OK : SPIN4D_ERR_UNSUPPORTED;
}

static int hex_bwd_blocks(int64_t N) { return persistent_blocks((N + kHexBwdBlock - 1) / kHexBwdBlock, 2); }

static int hex_check(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame, int64_t N,
                     const float* planes, const float* weights, const float* q_can, const float* logs_can) {
  SPIN4D_CHECK(validate_hex(h));
  if (N < 0) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  if (!mu || !frame || !planes || !weights || !q_can || !logs_can) return SPIN4D_ERR_INVALID;
  if (!aligned(planes, 32) || !aligned(weights, 32) || !aligned(mu, 4) || !aligned(frame, 4) ||
      !aligned(q_can, 4) || !aligned(logs_can, 4))
    return SPIN4D_ERR_INVALID;
  return hex_supported(h);
}

}  // namespace spin4d

using namespace spin4d;

extern "C" int64_t spin4d_hexplane_plane_count(const spin4d_hexplane_desc* h) {
  if (validate_hex(h) != SPIN4D_OK) return -1;
  int64_t n = 0;
  for (int s = 0; s < h->n_scales; ++s) {
    int64_t m = h->scales[s];
    n += 3 * m * m + 3 * m * (int64_t)h->time_res;
  }
  return n * h->channels;
}

extern "C" int64_t spin4d_hexplane_param_count(const spin4d_hexplane_desc* h) {
  if (validate_hex(h) != SPIN4D_OK) return -1;
  int64_t n = 0, d = (int64_t)h->n_scales * 6 * h->channels;
  for (int j = 0; j < h->n_hidden; ++j) {
    n += (int64_t)h->hidden * d + h->hidden;
    d = h->hidden;
  }
  return n + (int64_t)kHexHead * d + kHexHead;
}

namespace spin4d {
// The window's arguments: cr N x 2 (8-byte aligned), tau > 0 and finite;
// grad_cr (backward only) N x 2, 8-byte aligned, or NULL.
static int hex_gate_check(const spin4d_hex_gate* gate, bool backward) {
  if (!gate || !gate->cr || !aligned(gate->cr, 8)) return SPIN4D_ERR_INVALID;
  if (!(gate->tau > 0.0f) || !std::isfinite(gate->tau)) return SPIN4D_ERR_INVALID;
  if (gate->grad_cr && (!backward || !aligned(gate->grad_cr, 8))) return SPIN4D_ERR_INVALID;
  return SPIN4D_OK;
}

static void hex_set_gate(HexParams& p, const spin4d_hex_gate* gate) {
  if (!gate) return;
  p.gate_cr = gate->cr;
  p.gate_grad = gate->grad_cr;
  p.gate_tau = gate->tau;
}
}  // namespace spin4d

static int hexplane_fwd_impl(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame, int64_t N,
                             const float* planes, const float* weights, const float* q_can, const float* logs_can,
                             const float* sh_can, const spin4d_hex_gate* gate, spin4d_hex_outputs out,
                             spin4d_stream_t stream, const char* name) {
  SPIN4D_CHECK(hex_check(h, mu, frame, N, planes, weights, q_can, logs_can));
  if (N == 0) return SPIN4D_OK;
  if (!sh_can || !out.mu || !out.rot || !out.scale || !out.sh || !out.cov || !aligned(out.rot, 16) ||
      !aligned(sh_can, 16) || !aligned(out.sh, 16))
    return SPIN4D_ERR_INVALID;
  if (out.latent && !aligned(out.latent, 32)) return SPIN4D_ERR_INVALID;
  if (out.hidden && !aligned(out.hidden, 16)) return SPIN4D_ERR_INVALID;
  if (gate) SPIN4D_CHECK(hex_gate_check(gate, false));
  if (fault_injected(name)) return SPIN4D_ERR_INJECTED;
  HexParams p = make_hex_params(h);
  hex_set_gate(p, gate);
  HexOutPtrs o{out.mu, out.rot, out.scale, out.sh, out.cov};
  if (h->n_scales * 6 <= 24) {
    // tensor cores, bf16x3 split, warp-specialised
    static bool ws_configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    const int smem = HexWsLayout::BYTES;
    if (!ws_configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(hexplane_fwd_ws_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return cuda_status(e);
      int occ = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, hexplane_fwd_ws_kernel, kWsThreads, smem);
      if (e != cudaSuccess) return cuda_status(e);
      if (occ != 1) return SPIN4D_ERR_UNSUPPORTED;   // one CTA holds all 512 TMEM columns
      ws_configured[dev] = true;
    }
    const int blocks = persistent_blocks((N + kHexTile - 1) / kHexTile, 1);
    hexplane_fwd_ws_kernel<<<blocks, kWsThreads, smem, (cudaStream_t)stream>>>(p, mu, frame, N, planes, weights, q_can,
                                                                             logs_can, sh_can, o, out.latent,
                                                                             out.hidden);
    return launch_status();
  }
  if (gate) return SPIN4D_ERR_UNSUPPORTED;   // the window is built into the tensor-core kernels only
  int blocks = persistent_blocks((N + 127) / 128, 4);
  hexplane_fwd_kernel<<<blocks, 128, 0, (cudaStream_t)stream>>>(p, mu, frame, N, planes, weights, q_can, logs_can,
                                                                sh_can, o);
  return launch_status();
}

extern "C" int spin4d_hexplane_fwd(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame, int64_t N,
                                   const float* planes, const float* weights, const float* q_can,
                                   const float* logs_can, const float* sh_can, spin4d_hex_outputs out,
                                   spin4d_stream_t stream) {
  return hexplane_fwd_impl(h, mu, frame, N, planes, weights, q_can, logs_can, sh_can, nullptr, out, stream,
                           "spin4d_hexplane_fwd");
}

extern "C" int spin4d_hexplane_fwd_gated(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame,
                                         int64_t N, const float* planes, const float* weights, const float* q_can,
                                         const float* logs_can, const float* sh_can, const spin4d_hex_gate* gate,
                                         spin4d_hex_outputs out, spin4d_stream_t stream) {
  if (!gate) return SPIN4D_ERR_INVALID;
  return hexplane_fwd_impl(h, mu, frame, N, planes, weights, q_can, logs_can, sh_can, gate, out, stream,
                           "spin4d_hexplane_fwd_gated");
}

namespace spin4d {
// Workspace: the per-block weight-gradient slots, then (from a 256-byte
// boundary) N x 64 fp32 for dh1 between the two kernels of the backward from
// a saved latent.
static size_t hex_slots_bytes(const spin4d_hexplane_desc* h, int64_t N) {
  const size_t b = (size_t)hex_bwd_blocks(N) * slot_stride((int)spin4d_hexplane_param_count(h)) * sizeof(float);
  return (b + 255) & ~(size_t)255;
}
static float* hex_dh1_buffer(void* workspace, int64_t N, const spin4d_hexplane_desc* h) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + hex_slots_bytes(h, N));
}
}  // namespace spin4d

extern "C" size_t spin4d_hexplane_bwd_workspace(const spin4d_hexplane_desc* h, int64_t N) {
  if (validate_hex(h) != SPIN4D_OK || N <= 0) return 0;
  return hex_slots_bytes(h, N) + (size_t)N * kHexH * sizeof(float);
}

static int hexplane_bwd_impl(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame, int64_t N,
                             const float* planes, const float* weights, const float* q_can, const float* logs_can,
                             const float* latent, const float* hidden, const spin4d_hex_gate* gate,
                             const spin4d_hex_output_grads* grad_out, float* grad_planes, float* grad_weights,
                             void* workspace, size_t ws_bytes, spin4d_stream_t stream, const char* name) {
  SPIN4D_CHECK(hex_check(h, mu, frame, N, planes, weights, q_can, logs_can));
  if (N == 0) return SPIN4D_OK;
  if (!grad_out || !grad_planes || !grad_weights || !workspace) return SPIN4D_ERR_INVALID;
  if (!aligned(grad_planes, 16) || !aligned(grad_weights, 4) || !aligned(workspace, 256)) return SPIN4D_ERR_INVALID;
  if (latent && !aligned(latent, 32)) return SPIN4D_ERR_INVALID;
  if (hidden && (!latent || !aligned(hidden, 16))) return SPIN4D_ERR_INVALID;
  if (ws_bytes < spin4d_hexplane_bwd_workspace(h, N)) return SPIN4D_ERR_INVALID;
  if (gate) SPIN4D_CHECK(hex_gate_check(gate, true));
  if (fault_injected(name)) return SPIN4D_ERR_INJECTED;
  HexParams p = make_hex_params(h);
  hex_set_gate(p, gate);
  HexGradPtrs go{grad_out->mu, grad_out->rot, grad_out->scale, grad_out->sh, grad_out->cov};
  const int n_params = (int)spin4d_hexplane_param_count(h);
  cudaStream_t s = (cudaStream_t)stream;
  int blocks = 0;
  {
    // tensor cores, bf16x3 split: one CTA per SM (it holds 512 TMEM columns)
    static bool configured[64] = {false};
    static bool usable[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    const int smem = HexBwdLayout::BYTES;
    if (!configured[dev]) {
      bool ok = true;
      for (auto* kern : {hexplane_bwd_tc_kernel<false>, hexplane_bwd_tc_kernel<true>}) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e);
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kHexThreads, smem);
        if (e != cudaSuccess) return cuda_status(e);
        ok = ok && occ == 1;
      }
      for (auto* kern : {hexplane_bwd_head_ws_kernel<false, false>, hexplane_bwd_head_ws_kernel<true, false>,
                         hexplane_bwd_head_ws_kernel<false, true>, hexplane_bwd_head_ws_kernel<true, true>}) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, HexBwWsLayout::BYTES);
        if (e != cudaSuccess) return cuda_status(e);
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kBwThreads, HexBwWsLayout::BYTES);
        if (e != cudaSuccess) return cuda_status(e);
        ok = ok && occ == 1;
      }
      {
        cudaError_t e = cudaFuncSetAttribute(hexplane_bwd_dz_ws_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             HexDzWsLayout::BYTES);
        if (e != cudaSuccess) return cuda_status(e);
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, hexplane_bwd_dz_ws_kernel, kDzThreads,
                                                          HexDzWsLayout::BYTES);
        if (e != cudaSuccess) return cuda_status(e);
        ok = ok && occ == 1;
      }
      usable[dev] = ok;
      configured[dev] = true;
    }
    if (usable[dev]) {
      blocks = persistent_blocks((N + kHexTile - 1) / kHexTile, 1);
      if (latent) {
        // from the saved latent: warp-specialised, the head then the W1 pass
        float* dh1 = hex_dh1_buffer(workspace, N, h);
        auto* kern = gate ? (hidden ? hexplane_bwd_head_ws_kernel<true, true> : hexplane_bwd_head_ws_kernel<true, false>)
                          : (hidden ? hexplane_bwd_head_ws_kernel<false, true> : hexplane_bwd_head_ws_kernel<false, false>);
        kern<<<blocks, kBwThreads, HexBwWsLayout::BYTES, s>>>(p, mu, frame, N, weights, q_can, logs_can, latent, hidden,
                                                               go, dh1, static_cast<float*>(workspace), n_params);
        SPIN4D_CHECK(launch_status());
        hexplane_bwd_dz_ws_kernel<<<blocks, kDzThreads, HexDzWsLayout::BYTES, s>>>(
            p, mu, frame, N, weights, latent, dh1, grad_planes, static_cast<float*>(workspace), n_params);
      } else {
        auto* kern = gate ? hexplane_bwd_tc_kernel<true> : hexplane_bwd_tc_kernel<false>;
        kern<<<blocks, kHexThreads, smem, s>>>(p, mu, frame, N, planes, weights, q_can, logs_can, go, grad_planes,
                                               static_cast<float*>(workspace), n_params);
      }
      SPIN4D_CHECK(launch_status());
    }
  }
  if (blocks == 0) {
    if (gate) return SPIN4D_ERR_UNSUPPORTED;   // the window is built into the tensor-core kernels only
    // fp32 SIMT fallback (the saved latent is not used)
    blocks = hex_bwd_blocks(N);
    const int smem = (4 * kHexH + kHexHead + kHexC) * kHexBwdBlock * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(hexplane_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_status(e);
    hexplane_bwd_kernel<<<blocks, kHexBwdBlock, smem, s>>>(p, mu, frame, N, planes, weights, q_can, logs_can, go,
                                                        grad_planes, static_cast<float*>(workspace), n_params);
    SPIN4D_CHECK(launch_status());
  }
  hex_reduce_slots<<<(n_params + 255) / 256, 256, 0, s>>>(static_cast<float*>(workspace), blocks, n_params,
                                                          grad_weights);
  return launch_status();
}

extern "C" int spin4d_hexplane_bwd(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame, int64_t N,
                                   const float* planes, const float* weights, const float* q_can,
                                   const float* logs_can, const float* sh_can, const float* latent,
                                   const spin4d_hex_output_grads* grad_out, float* grad_planes,
                                   float* grad_weights, void* workspace, size_t ws_bytes, spin4d_stream_t stream) {
  (void)sh_can;   // sh' = sh_can + d_sh: the upstream sh gradient flows through unchanged
  return hexplane_bwd_impl(h, mu, frame, N, planes, weights, q_can, logs_can, latent, nullptr, nullptr, grad_out,
                           grad_planes, grad_weights, workspace, ws_bytes, stream, "spin4d_hexplane_bwd");
}

extern "C" int spin4d_hexplane_bwd_gated(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame,
                                         int64_t N, const float* planes, const float* weights, const float* q_can,
                                         const float* logs_can, const float* sh_can, const float* latent,
                                         const spin4d_hex_gate* gate, const spin4d_hex_output_grads* grad_out,
                                         float* grad_planes, float* grad_weights, void* workspace, size_t ws_bytes,
                                         spin4d_stream_t stream) {
  (void)sh_can;
  if (!gate) return SPIN4D_ERR_INVALID;
  return hexplane_bwd_impl(h, mu, frame, N, planes, weights, q_can, logs_can, latent, nullptr, gate, grad_out,
                           grad_planes, grad_weights, workspace, ws_bytes, stream, "spin4d_hexplane_bwd_gated");
}

extern "C" int spin4d_hexplane_bwd_saved(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame,
                                         int64_t N, const float* planes, const float* weights, const float* q_can,
                                         const float* logs_can, const spin4d_hex_saved* saved,
                                         const spin4d_hex_gate* gate, const spin4d_hex_output_grads* grad_out,
                                         float* grad_planes, float* grad_weights, void* workspace, size_t ws_bytes,
                                         spin4d_stream_t stream) {
  if (!saved || !saved->latent) return SPIN4D_ERR_INVALID;
  return hexplane_bwd_impl(h, mu, frame, N, planes, weights, q_can, logs_can, saved->latent, saved->hidden, gate,
                           grad_out, grad_planes, grad_weights, workspace, ws_bytes, stream,
                           "spin4d_hexplane_bwd_saved");
}
