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
#include <string.h>

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
};

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
  s.o01 = s.o00 + kHexC;
  s.o10 = s.o00 + row;
  s.o11 = s.o10 + kHexC;
  s.w00 = (1.0f - wa) * (1.0f - wb);
  s.w01 = wa * (1.0f - wb);
  s.w10 = (1.0f - wa) * wb;
  s.w11 = wa * wb;
  return s;
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
// Forward on the tensor cores, fp32-accurate: 3xTF32 (kind::tf32).
//
// Every operand x is split into hi = tf32(x) and lo = x - hi, and each
// product is hi.hi + hi.lo + lo.hi (the dropped lo.lo term is below 2^-21 of
// the result), which keeps the 1e-5 fp32 parity that plain tf32 misses.
// Persistent CTAs of 256 threads handle 128-Gaussian tiles.  The 576-wide
// first layer is streamed one plane sample (32 channels) at a time through
// two shared-memory stages: while the tensor core multiplies sample k, the
// threads gather and split sample k+1 (two threads per Gaussian, 16 channels
// each, 16-byte loads of the channel-last rows) and stage the matching 64x32
// slice of W1.  Trunk layer 2 and the 58-row head follow from one 128x64
// activation tile; the epilogue writes mu', q', s', sh' and Sigma.
// ---------------------------------------------------------------------------
namespace {

constexpr int kHexTile = 128;
constexpr int kHexThreads = 256;
constexpr uint32_t kHexWait = 1u << 24;

struct HexTcLayout {
  static constexpr int A = 0;                      // 2 stages x (hi, lo) [128][32] fp32 = 64 KB; later the H tile
  static constexpr int A_STAGE = 2 * kHexTile * kHexC * 4;
  static constexpr int H_LO = kHexTile * kHexH * 4;   // H tile: hi at A, lo at A + H_LO
  static constexpr int B1 = A + 2 * A_STAGE;       // 2 stages x (hi, lo) [64][32]
  static constexpr int B1_STAGE = 2 * kHexH * kHexC * 4;
  static constexpr int W2 = B1 + 2 * B1_STAGE;     // hi, lo [64][64]
  static constexpr int W3 = W2 + 2 * kHexH * kHexH * 4;   // hi, lo [64][64] (58 rows used)
  static constexpr int BIAS = W3 + 2 * kHexH * kHexH * 4; // b1 | b2 | b3 (64 each)
  static constexpr int MISC = BIAS + 3 * kHexH * 4;  // 2 mbarriers + TMEM address
  static constexpr int BYTES = MISC + 32;
};

// Stores 4 consecutive values of a row (K-major 32-bit tile with K columns,
// 4-value chunk kc) as tf32 hi and lo parts.
__device__ __forceinline__ void store_split4(uint8_t* sm, int hi_off, int lo_off, int r, int kc, int K, float4 v) {
  float h0, h1, h2, h3, l0, l1, l2, l3;
  tc::split_tf32(v.x, h0, l0);
  tc::split_tf32(v.y, h1, l1);
  tc::split_tf32(v.z, h2, l2);
  tc::split_tf32(v.w, h3, l3);
  *reinterpret_cast<float4*>(sm + hi_off + tc::kmaj_off32(r, kc, K)) = make_float4(h0, h1, h2, h3);
  *reinterpret_cast<float4*>(sm + lo_off + tc::kmaj_off32(r, kc, K)) = make_float4(l0, l1, l2, l3);
}

// 3xTF32 product over K columns into two fresh accumulators: d_main = A_hi.B_hi
// and d_corr = A_hi.B_lo + A_lo.B_hi (the dropped lo.lo term is below 2^-21).
// The tensor core aligns addends to the running sum and truncates, so the
// small correction terms get an accumulator of their own, and callers keep K
// short and add the partial results in fp32 on the CUDA cores.
__device__ __forceinline__ void mma_3xtf32(uint32_t d_main, uint32_t d_corr, uint32_t a_hi, uint32_t a_lo, uint32_t b_hi,
                                           uint32_t b_lo, int K, int N) {
  const uint32_t sbo = (uint32_t)K * 32u;
  const uint32_t idesc = tc::idesc_tf32_f32(kHexTile, N);
  for (int s = 0; s < K / 8; ++s) {
    const uint32_t o = (uint32_t)s * 256u;
    tc::mma_tf32(d_main, tc::smem_desc(a_hi + o, 128, sbo), tc::smem_desc(b_hi + o, 128, sbo), idesc, s > 0 ? 1u : 0u);
    tc::mma_tf32(d_corr, tc::smem_desc(a_hi + o, 128, sbo), tc::smem_desc(b_lo + o, 128, sbo), idesc, s > 0 ? 1u : 0u);
    tc::mma_tf32(d_corr, tc::smem_desc(a_lo + o, 128, sbo), tc::smem_desc(b_hi + o, 128, sbo), idesc, 1u);
  }
}

// acc[i] += main[col0 + i] + corr[col0 + i] for this thread's 32 columns.
__device__ __forceinline__ void add_partial(uint32_t d_main, uint32_t d_corr, float acc[32]) {
  float a[32], b[32];
  tc::tmem_ld32(d_main, a);
  tc::tmem_ld32(d_corr, b);
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] += a[i] + b[i];
}

__global__ void __launch_bounds__(kHexThreads, 1) hexplane_fwd_tc_kernel(
    HexParams hp, const float* __restrict__ mu, const int32_t* __restrict__ frame, int64_t N,
    const float* __restrict__ planes, const float* __restrict__ W, const float* __restrict__ q_can,
    const float* __restrict__ logs_can, const float* __restrict__ sh_can, HexOutPtrs out, float* __restrict__ latent) {
  using Lay = HexTcLayout;
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (kHexTile - 1), half = tid / kHexTile;
  const int IN = hp.in_dim, NS = hp.n_samples;
  const float* W1 = W;
  const float* b1 = W1 + kHexH * IN;
  const float* W2g = b1 + kHexH;
  const float* b2 = W2g + kHexH * kHexH;
  const float* W3g = b2 + kHexH;
  const float* b3 = W3g + kHexHead * kHexH;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::MISC + 16);
  const uint32_t mbar0 = tc::smem_u32(sm + Lay::MISC), mbar1 = mbar0 + 8;
  float* bias = reinterpret_cast<float*>(sm + Lay::BIAS);

  // ---- W2, W3 (split) and biases, once per CTA ----
  for (int i = tid; i < kHexH * (kHexH / 4); i += kHexThreads) {
    const int r = i / (kHexH / 4), kc = i % (kHexH / 4);
    store_split4(sm, Lay::W2, Lay::W2 + kHexH * kHexH * 4, r, kc, kHexH,
                 __ldg(reinterpret_cast<const float4*>(W2g + r * kHexH) + kc));
    const float4 w3 = r < kHexHead ? __ldg(reinterpret_cast<const float4*>(W3g + r * kHexH) + kc)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    store_split4(sm, Lay::W3, Lay::W3 + kHexH * kHexH * 4, r, kc, kHexH, w3);
  }
  for (int o = tid; o < kHexH; o += kHexThreads) {
    bias[o] = __ldg(b1 + o);
    bias[kHexH + o] = __ldg(b2 + o);
    bias[2 * kHexH + o] = o < kHexHead ? __ldg(b3 + o) : 0.f;
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 256);
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
  // TMEM regions of 64 columns: R0..R3.  Plane sample k accumulates into
  // (R0, R1) when k is even and (R2, R3) when odd; layer 2 uses (R0, R1) and
  // the head (R2, R3).
  const uint32_t R[4] = {tmem, tmem + 64, tmem + 128, tmem + 192};
  uint32_t ph0 = 0, ph1 = 0;
  bool failed = false;
  auto wait_bar = [&](int b) -> bool {
    const uint32_t bar = b ? mbar1 : mbar0;
    uint32_t& ph = b ? ph1 : ph0;
    const bool ok = tc::mbar_wait_bounded(bar, ph, kHexWait);
    ph ^= 1u;
    return ok;
  };
  const uint32_t sA = tc::smem_u32(sm + Lay::A), sB1 = tc::smem_u32(sm + Lay::B1);
  const uint32_t col = (uint32_t)(half * 32);

  for (int64_t tile = blockIdx.x; tile * kHexTile < N; tile += gridDim.x) {
    const int64_t n = tile * kHexTile + row;
    const bool valid = n < N;
    float xt[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) hex_normalise(mu, frame, n, hp, xt);
    float acc1[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc1[i] = 0.f;
    // ---- layer 1, streamed over the plane samples ----
    // Registers hold sample k+1's global data (its W1 slice and its four
    // corner rows) while sample k is multiplied, so load latency overlaps
    // the MMAs and the barriers.
    float4 wpre[2], cpre[4][4];
    float cw[4];
    auto prefetch = [&](int k) {
      const int r = tid >> 2, c2 = (tid & 3) * 2;
#pragma unroll
      for (int q = 0; q < 2; ++q) wpre[q] = __ldg(reinterpret_cast<const float4*>(W1 + (size_t)r * IN + k * kHexC) + c2 + q);
      if (valid) {
        const PlaneSample ps = plane_sample(xt, hp, k);
        cw[0] = ps.w00; cw[1] = ps.w01; cw[2] = ps.w10; cw[3] = ps.w11;
        const int64_t off[4] = {ps.o00, ps.o01, ps.o10, ps.o11};
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int q = 0; q < 4; ++q) cpre[c][q] = __ldg(reinterpret_cast<const float4*>(planes + off[c]) + half * 4 + q);
      }
    };
    prefetch(0);
    for (int k = 0; k < NS; ++k) {
      const int b = k & 1;
      if (k >= 2) {   // sample k-2 used this stage: fold its partial sums in, then reuse
        const bool ok = wait_bar(b);
        if (__syncthreads_or(!ok)) { failed = true; break; }
        tc::fence_after_sync();
        add_partial(R[2 * b] + lane + col, R[2 * b + 1] + lane + col, acc1);
      }
      const int a_hi = Lay::A + b * Lay::A_STAGE, a_lo = a_hi + kHexTile * kHexC * 4;
      const int w_hi = Lay::B1 + b * Lay::B1_STAGE, w_lo = w_hi + kHexH * kHexC * 4;
      {
        const int r = tid >> 2, c2 = (tid & 3) * 2;
#pragma unroll
        for (int q = 0; q < 2; ++q) store_split4(sm, w_hi, w_lo, r, c2 + q, kHexC, wpre[q]);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c4 = half * 4 + q;
        float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) {
          z4.x = cw[0] * cpre[0][q].x + cw[1] * cpre[1][q].x + cw[2] * cpre[2][q].x + cw[3] * cpre[3][q].x;
          z4.y = cw[0] * cpre[0][q].y + cw[1] * cpre[1][q].y + cw[2] * cpre[2][q].y + cw[3] * cpre[3][q].y;
          z4.z = cw[0] * cpre[0][q].z + cw[1] * cpre[1][q].z + cw[2] * cpre[2][q].z + cw[3] * cpre[3][q].z;
          z4.w = cw[0] * cpre[0][q].w + cw[1] * cpre[1][q].w + cw[2] * cpre[2][q].w + cw[3] * cpre[3][q].w;
          if (latent) reinterpret_cast<float4*>(latent + n * IN + k * kHexC)[c4] = z4;
        }
        store_split4(sm, a_hi, a_lo, row, c4, kHexC, z4);
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      __syncthreads();
      if (tid == 0) {
        tc::fence_after_sync();
        mma_3xtf32(R[2 * b], R[2 * b + 1], sA + a_hi, sA + a_lo, sB1 + (w_hi - Lay::B1), sB1 + (w_lo - Lay::B1), kHexC,
                   kHexH);
        tc::mma_commit(b ? mbar1 : mbar0);
      }
      if (k + 1 < NS) prefetch(k + 1);
    }
    if (failed) break;
    // the last two samples (in the order their barriers completed)
    for (int k = (NS >= 2 ? NS - 2 : 0); k < NS; ++k) {
      const int b = k & 1;
      const bool ok = wait_bar(b);
      if (__syncthreads_or(!ok)) { failed = true; break; }
      tc::fence_after_sync();
      add_partial(R[2 * b] + lane + col, R[2 * b + 1] + lane + col, acc1);
    }
    if (failed) break;
    // ---- h1 = relu(sum + b1) -> split H tile (over the A stages) ----
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 h;
      h.x = fmaxf(acc1[4 * q] + bias[half * 32 + 4 * q], 0.f);
      h.y = fmaxf(acc1[4 * q + 1] + bias[half * 32 + 4 * q + 1], 0.f);
      h.z = fmaxf(acc1[4 * q + 2] + bias[half * 32 + 4 * q + 2], 0.f);
      h.w = fmaxf(acc1[4 * q + 3] + bias[half * 32 + 4 * q + 3], 0.f);
      store_split4(sm, Lay::A, Lay::A + Lay::H_LO, row, half * 8 + q, kHexH, h);
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    // ---- layer 2 into (R0, R1) ----
    if (tid == 0) {
      tc::fence_after_sync();
      mma_3xtf32(R[0], R[1], sA, sA + Lay::H_LO, tc::smem_u32(sm + Lay::W2), tc::smem_u32(sm + Lay::W2) + kHexH * kHexH * 4,
                 kHexH, kHexH);
      tc::mma_commit(mbar0);
    }
    if (__syncthreads_or(!wait_bar(0))) { failed = true; break; }
    tc::fence_after_sync();
    {
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
      add_partial(R[0] + lane + col, R[1] + lane + col, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 h;
        h.x = fmaxf(v[4 * q] + bias[kHexH + half * 32 + 4 * q], 0.f);
        h.y = fmaxf(v[4 * q + 1] + bias[kHexH + half * 32 + 4 * q + 1], 0.f);
        h.z = fmaxf(v[4 * q + 2] + bias[kHexH + half * 32 + 4 * q + 2], 0.f);
        h.w = fmaxf(v[4 * q + 3] + bias[kHexH + half * 32 + 4 * q + 3], 0.f);
        store_split4(sm, Lay::A, Lay::A + Lay::H_LO, row, half * 8 + q, kHexH, h);
      }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    // ---- head (58 rows, padded to 64) into (R2, R3) ----
    if (tid == 0) {
      tc::fence_after_sync();
      mma_3xtf32(R[2], R[3], sA, sA + Lay::H_LO, tc::smem_u32(sm + Lay::W3), tc::smem_u32(sm + Lay::W3) + kHexH * kHexH * 4,
                 kHexH, kHexH);
      tc::mma_commit(mbar0);
    }
    if (__syncthreads_or(!wait_bar(0))) { failed = true; break; }
    tc::fence_after_sync();
    {
      float y[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] = bias[2 * kHexH + half * 32 + i];
      add_partial(R[2] + lane + col, R[3] + lane + col, y);
      tc::fence_before_sync();
      if (valid) {
        if (half == 0) {
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
#pragma unroll
          for (int i = 10; i < 32; ++i) out.sh[48 * n + (i - 10)] = __ldg(sh_can + 48 * n + (i - 10)) + y[i];
        } else {
#pragma unroll
          for (int i = 0; i < kHexHead - 32; ++i) out.sh[48 * n + 22 + i] = __ldg(sh_can + 48 * n + 22 + i) + y[i];
        }
      }
    }
    __syncthreads();
  }

  if (failed) {
    if (tid == 0) atomicExch(&g_hex_device_error, 1);
    wait_bar(0);
    wait_bar(1);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
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
  if (!aligned(planes, 16) || !aligned(weights, 16) || !aligned(mu, 4) || !aligned(frame, 4) ||
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

extern "C" int spin4d_hexplane_fwd(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame, int64_t N,
                                   const float* planes, const float* weights, const float* q_can,
                                   const float* logs_can, const float* sh_can, spin4d_hex_outputs out,
                                   spin4d_stream_t stream) {
  SPIN4D_CHECK(hex_check(h, mu, frame, N, planes, weights, q_can, logs_can));
  if (N == 0) return SPIN4D_OK;
  if (!sh_can || !out.mu || !out.rot || !out.scale || !out.sh || !out.cov || !aligned(out.rot, 16))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_hexplane_fwd")) return SPIN4D_ERR_INJECTED;
  HexParams p = make_hex_params(h);
  HexOutPtrs o{out.mu, out.rot, out.scale, out.sh, out.cov};
  if (h->n_scales * 6 <= 24) {
    // tensor cores, 3xTF32
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    const int smem = HexTcLayout::BYTES;
    if (!configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(hexplane_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return cuda_status(e);
      int occ = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, hexplane_fwd_tc_kernel, kHexThreads, smem);
      if (e != cudaSuccess) return cuda_status(e);
      if (occ < 1 || occ * 256 > 512) return SPIN4D_ERR_UNSUPPORTED;
      configured[dev] = true;
    }
    const int blocks = persistent_blocks((N + kHexTile - 1) / kHexTile, 1);
    hexplane_fwd_tc_kernel<<<blocks, kHexThreads, smem, (cudaStream_t)stream>>>(p, mu, frame, N, planes, weights, q_can,
                                                                               logs_can, sh_can, o, out.latent);
    return launch_status();
  }
  int blocks = persistent_blocks((N + 127) / 128, 4);
  hexplane_fwd_kernel<<<blocks, 128, 0, (cudaStream_t)stream>>>(p, mu, frame, N, planes, weights, q_can, logs_can,
                                                                sh_can, o);
  return launch_status();
}

extern "C" size_t spin4d_hexplane_bwd_workspace(const spin4d_hexplane_desc* h, int64_t N) {
  if (validate_hex(h) != SPIN4D_OK || N <= 0) return 0;
  return (size_t)hex_bwd_blocks(N) * slot_stride((int)spin4d_hexplane_param_count(h)) * sizeof(float);
}

extern "C" int spin4d_hexplane_bwd(const spin4d_hexplane_desc* h, const float* mu, const int32_t* frame, int64_t N,
                                   const float* planes, const float* weights, const float* q_can,
                                   const float* logs_can, const float* sh_can,
                                   const spin4d_hex_output_grads* grad_out, float* grad_planes,
                                   float* grad_weights, void* workspace, size_t ws_bytes, spin4d_stream_t stream) {
  (void)sh_can;   // sh' = sh_can + d_sh: the upstream sh gradient flows through unchanged
  SPIN4D_CHECK(hex_check(h, mu, frame, N, planes, weights, q_can, logs_can));
  if (N == 0) return SPIN4D_OK;
  if (!grad_out || !grad_planes || !grad_weights || !workspace) return SPIN4D_ERR_INVALID;
  if (!aligned(grad_planes, 16) || !aligned(grad_weights, 4) || !aligned(workspace, 256)) return SPIN4D_ERR_INVALID;
  if (ws_bytes < spin4d_hexplane_bwd_workspace(h, N)) return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_hexplane_bwd")) return SPIN4D_ERR_INJECTED;
  HexParams p = make_hex_params(h);
  HexGradPtrs go{grad_out->mu, grad_out->rot, grad_out->scale, grad_out->sh, grad_out->cov};
  const int n_params = (int)spin4d_hexplane_param_count(h);
  const int blocks = hex_bwd_blocks(N);
  cudaStream_t s = (cudaStream_t)stream;
  const int smem = (4 * kHexH + kHexHead + kHexC) * kHexBwdBlock * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(hexplane_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_status(e);
  hexplane_bwd_kernel<<<blocks, kHexBwdBlock, smem, s>>>(p, mu, frame, N, planes, weights, q_can, logs_can, go,
                                                      grad_planes, static_cast<float*>(workspace), n_params);
  SPIN4D_CHECK(launch_status());
  hex_reduce_slots<<<(n_params + 255) / 256, 256, 0, s>>>(static_cast<float*>(workspace), blocks, n_params,
                                                          grad_weights);
  return launch_status();
}
