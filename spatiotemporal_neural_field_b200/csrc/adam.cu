// Fused Adam (Kingma & Ba, with bias correction) over fp32 master parameters,
// optionally writing the fp16 working copy the decoder reads and clearing the
// gradient.  One pass over memory: HBM-bound.
#include "host.h"

namespace spin4d {

struct AdamParams {
  float lr, b1, b2, eps, omb1, omb2, inv_bc1, inv_bc2;
  int zero_grad;
};

__device__ __forceinline__ float adam_one(float p, float g, float& m, float& v, const AdamParams& a) {
  m = a.b1 * m + a.omb1 * g;
  v = a.b2 * v + a.omb2 * (g * g);
  float mh = m * a.inv_bc1;
  float vh = v * a.inv_bc2;
  return p - a.lr * mh / (sqrtf(vh) + a.eps);
}

__global__ void __launch_bounds__(256) adam_kernel(float* __restrict__ p, __half* __restrict__ work,
                                                   float* __restrict__ g, float* __restrict__ m,
                                                   float* __restrict__ v, int64_t n, AdamParams a,
                                                   int32_t* __restrict__ flag) {
  const int64_t n4 = n / 4;
  bool bad = false;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 P = reinterpret_cast<float4*>(p)[i];
    float4 G = reinterpret_cast<float4*>(g)[i];
    float4 M = reinterpret_cast<float4*>(m)[i];
    float4 V = reinterpret_cast<float4*>(v)[i];
    P.x = adam_one(P.x, G.x, M.x, V.x, a);
    P.y = adam_one(P.y, G.y, M.y, V.y, a);
    P.z = adam_one(P.z, G.z, M.z, V.z, a);
    P.w = adam_one(P.w, G.w, M.w, V.w, a);
    reinterpret_cast<float4*>(p)[i] = P;
    reinterpret_cast<float4*>(m)[i] = M;
    reinterpret_cast<float4*>(v)[i] = V;
    if (a.zero_grad) reinterpret_cast<float4*>(g)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (work) {
      __half2 lo = __floats2half2_rn(P.x, P.y), hi = __floats2half2_rn(P.z, P.w);
      uint2 u;
      u.x = *reinterpret_cast<unsigned int*>(&lo);
      u.y = *reinterpret_cast<unsigned int*>(&hi);
      reinterpret_cast<uint2*>(work)[i] = u;
    }
    bad |= !(isfinite(P.x) && isfinite(P.y) && isfinite(P.z) && isfinite(P.w));
  }
  for (int64_t i = n4 * 4 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += stride) {
    float mm = m[i], vv = v[i];
    float q = adam_one(p[i], g[i], mm, vv, a);
    p[i] = q;
    m[i] = mm;
    v[i] = vv;
    if (a.zero_grad) g[i] = 0.0f;
    if (work) work[i] = __float2half_rn(q);
    bad |= !isfinite(q);
  }
  if (flag && __syncthreads_or(bad) && threadIdx.x == 0) atomicExch(flag, 1);
}

// Per-group learning rates: element i takes the rate of the first group
// whose end exceeds i.  Scalar elements (a group boundary may split a float4).
struct AdamGroups {
  int n;
  int64_t end[SPIN4D_MAX_ADAM_GROUPS];
  float lr[SPIN4D_MAX_ADAM_GROUPS];
};

__global__ void __launch_bounds__(256) adam_groups_kernel(float* __restrict__ p, __half* __restrict__ work,
                                                          float* __restrict__ g, float* __restrict__ m,
                                                          float* __restrict__ v, int64_t n, AdamParams a,
                                                          AdamGroups gr, int32_t* __restrict__ flag) {
  bool bad = false;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int grp = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += stride) {
    while (grp + 1 < gr.n && i >= gr.end[grp]) ++grp;   // i only grows along this thread's loop
    AdamParams ai = a;
    ai.lr = gr.lr[grp];
    float mm = m[i], vv = v[i];
    const float q = adam_one(p[i], g[i], mm, vv, ai);
    p[i] = q;
    m[i] = mm;
    v[i] = vv;
    if (a.zero_grad) g[i] = 0.0f;
    if (work) work[i] = __float2half_rn(q);
    bad |= !isfinite(q);
  }
  if (flag && __syncthreads_or(bad) && threadIdx.x == 0) atomicExch(flag, 1);
}

}  // namespace spin4d

using namespace spin4d;

extern "C" double spin4d_lr_warmup_cosine(int64_t step, double lr_max, double lr_min, int64_t warmup, int64_t total) {
  if (warmup > 0 && step <= warmup) return lr_max * (double)step / (double)warmup;
  if (step >= total) return lr_min;
  const double span = (double)(total - warmup > 0 ? total - warmup : 1);
  const double u = (double)(step - warmup) / span;
  return lr_min + 0.5 * (lr_max - lr_min) * (1.0 + cos(3.14159265358979323846 * u));
}

extern "C" int spin4d_adam_step_groups(float* params, void* params_work, float* grad, float* m, float* v, int64_t n,
                                       const spin4d_adam_group* groups, int n_groups, int step, float b1, float b2,
                                       float eps, int zero_grad, int32_t* nonfinite_flag, spin4d_stream_t stream) {
  if (n < 0 || step < 1 || !groups || n_groups < 1 || n_groups > SPIN4D_MAX_ADAM_GROUPS) return SPIN4D_ERR_INVALID;
  if (!(b1 >= 0.f && b1 < 1.f && b2 >= 0.f && b2 < 1.f && eps >= 0.f)) return SPIN4D_ERR_INVALID;
  AdamGroups gr;
  gr.n = n_groups;
  int64_t prev = 0;
  for (int k = 0; k < n_groups; ++k) {
    if (groups[k].end < prev || !isfinite(groups[k].lr)) return SPIN4D_ERR_INVALID;
    gr.end[k] = groups[k].end;
    gr.lr[k] = groups[k].lr;
    prev = groups[k].end;
  }
  if (prev != n) return SPIN4D_ERR_INVALID;
  if (n == 0) return SPIN4D_OK;
  if (!params || !grad || !m || !v) return SPIN4D_ERR_INVALID;
  if (!aligned(params, 4) || !aligned(grad, 4) || !aligned(m, 4) || !aligned(v, 4) ||
      (params_work && !aligned(params_work, 2)) || (nonfinite_flag && !aligned(nonfinite_flag, 4)))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_adam_step_groups")) return SPIN4D_ERR_INJECTED;
  AdamParams a;
  a.lr = 0.0f;
  a.b1 = b1;
  a.b2 = b2;
  a.eps = eps;
  a.omb1 = 1.0f - b1;
  a.omb2 = 1.0f - b2;
  a.inv_bc1 = (float)(1.0 / (1.0 - pow((double)b1, (double)step)));
  a.inv_bc2 = (float)(1.0 / (1.0 - pow((double)b2, (double)step)));
  a.zero_grad = zero_grad ? 1 : 0;
  int blocks = persistent_blocks((n + 255) / 256, 8);
  adam_groups_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(params, static_cast<__half*>(params_work), grad, m, v,
                                                               n, a, gr, nonfinite_flag);
  return launch_status();
}

extern "C" int spin4d_adam_step(float* params, void* params_work, float* grad, float* m, float* v, int64_t n,
                                int step, float lr, float b1, float b2, float eps, int zero_grad,
                                int32_t* nonfinite_flag, spin4d_stream_t stream) {
  if (n < 0 || step < 1) return SPIN4D_ERR_INVALID;
  if (!(b1 >= 0.f && b1 < 1.f && b2 >= 0.f && b2 < 1.f && eps >= 0.f && isfinite(lr))) return SPIN4D_ERR_INVALID;
  if (n == 0) return SPIN4D_OK;
  if (!params || !grad || !m || !v) return SPIN4D_ERR_INVALID;
  if (!aligned(params, 16) || !aligned(grad, 16) || !aligned(m, 16) || !aligned(v, 16) ||
      (params_work && !aligned(params_work, 8)) || (nonfinite_flag && !aligned(nonfinite_flag, 4)))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_adam_step")) return SPIN4D_ERR_INJECTED;
  AdamParams a;
  a.lr = lr;
  a.b1 = b1;
  a.b2 = b2;
  a.eps = eps;
  a.omb1 = 1.0f - b1;
  a.omb2 = 1.0f - b2;
  a.inv_bc1 = (float)(1.0 / (1.0 - pow((double)b1, (double)step)));
  a.inv_bc2 = (float)(1.0 / (1.0 - pow((double)b2, (double)step)));
  a.zero_grad = zero_grad ? 1 : 0;
  int blocks = persistent_blocks((n / 4 + 255) / 256 + 1, 8);
  adam_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(params, static_cast<__half*>(params_work), grad, m, v, n,
                                                        a, nonfinite_flag);
  return launch_status();
}
