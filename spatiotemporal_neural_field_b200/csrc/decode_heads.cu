// The paper's attribute-aware decoder: four heads (scale, rotation, SH
// colour, opacity), each a three-layer MLP in -> hidden -> hidden -> rows
// with GELU after the first two layers, on the shared latent z of the 4D
// hash encoder (SPIN-4DGS section 3.3, Eqs. 9-11; Sigma by Eq. 2).
//
// Two implementations.  With fp16 tables and weights, F = 4, in_dim =
// hidden = 64 and the degree-3 SH head of 48 rows (the paper's
// configuration) the layers run on the tensor cores: the forward as a
// full-occupancy gather of z into a workspace followed by heads_fwd_tc_kernel
// (or that kernel alone, gathering itself, without a workspace), and the
// backward, given the forward's z and raw outputs, as heads_bwd_tc_kernel.
// Operands are fp16 (z, activations, deltas), accumulation fp32.  Every other
// case runs the fp32 SIMT kernels below.
//
// SIMT kernels: 32 positions and 128 threads per block.  The hash gather
// takes one (position, level group) per thread.  The layers run out of
// shared memory: activations [position][feature], one layer's weights staged
// as fp32 rows, every product register-blocked 4 x 4 over 16-byte loads.
//
// Forward: gather z, then per head two GELU layers and the output layer,
// then Eq. 11 and Eq. 2.
// Backward: forward again keeping the raw outputs of the scale, rotation
// and opacity heads (they couple through Sigma), the activations' adjoint,
// then per head the forward again with its pre-activations, the data
// gradient through the three layers into dz (kept in registers across the
// heads) and the weight gradient summed over the block's positions into the
// block's workspace slot (a second kernel adds the slots in a fixed order);
// dz is scattered into the tables with fp32 atomics.
#include <type_traits>

#include "host.h"
#include "pdl.cuh"
#include "tc.cuh"

namespace spin4d {

// Set when a bounded wait of the tensor-core forward runs out.
__device__ int g_heads_device_error = 0;

int heads_device_error(int clear) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_heads_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_status(e);
  if (clear && v) {
    int zero = 0;
    e = cudaMemcpyToSymbol(g_heads_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_status(e);
  }
  return v ? SPIN4D_ERR_TIMEOUT : SPIN4D_OK;
}

namespace {

constexpr int kHeadsBwdBlock = 32;   // positions per block (forward and backward)
constexpr int kMaxDim = 64;          // in_dim, hidden and sh_dim limit of the shared-memory layout

struct HeadsParams {
  int in_dim, hidden, sh_dim;
  int rows[4];        // 3, 4, sh_dim, 1
  int off[4];         // parameter offset of each head
};

struct HeadsOut {
  float *scale, *rot, *sh, *opacity, *cov, *latent, *raw;
  uint4* z16;   // workspace of the split tensor-core forward (N rows of 64 fp16), or null
};
struct HeadsGrads {
  const float *scale, *rot, *sh, *opacity, *cov;
};

// Exact GELU, x Phi(x), and its derivative Phi(x) + x phi(x).
__device__ __forceinline__ float gelu(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad(float x) {
  return 0.5f * (1.0f + erff(x * 0.70710678118654752f)) + x * 0.39894228040143268f * expf(-0.5f * x * x);
}

// GELU for the tensor-core forward, whose hidden activations are rounded to
// fp16 right after it.  erf from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.28: for u >= 0,
// erf(u) = 1 - (1 + a1 u + ... + a6 u^6)^-16 with |error| <= 3e-7, three
// orders below the fp16 rounding; one reciprocal and no exponential.  With
// e = 1 - erf(|x| / sqrt 2): gelu(x) = x - x e / 2 for x >= 0, x e / 2 below.
__device__ __forceinline__ float gelu_fast(float x) {
  const float u = fabsf(x) * 0.70710678118654752f;
  float p = fmaf(u, 0.0000430638f, 0.0002765672f);
  p = fmaf(p, u, 0.0001520143f);
  p = fmaf(p, u, 0.0092705272f);
  p = fmaf(p, u, 0.0422820123f);
  p = fmaf(p, u, 0.0705230784f);
  p = fmaf(p, u, 1.0f);
  p *= p;   // ^2
  p *= p;   // ^4
  p *= p;   // ^8
  p *= p;   // ^16 (inf for large u, and then e = 0)
  const float he = 0.5f * x * __fdividef(1.0f, p);
  return x >= 0.0f ? x - he : he;
}

// kParts threads share the hash gather of each position (levels part,
// part + kParts, ...).
constexpr int kParts = 4;

// raw[0..2] scale^, raw[3..6] rot^, raw[7] opacity^ -> Eq. 11 and Eq. 2.
__device__ __forceinline__ void store_heads(const HeadsOut& out, int64_t n, const float raw[8]) {
  float s[3], r[4], cov[6];
#pragma unroll
  for (int i = 0; i < 3; ++i) s[i] = expf(fminf(raw[i], 20.0f));
  normalise_quat(raw + 3, r);
  covariance(s, r, cov);
#pragma unroll
  for (int i = 0; i < 3; ++i) out.scale[3 * n + i] = s[i];
  reinterpret_cast<float4*>(out.rot)[n] = make_float4(r[0], r[1], r[2], r[3]);
  out.opacity[n] = sigmoidf_(raw[7]);
#pragma unroll
  for (int i = 0; i < 6; ++i) out.cov[6 * n + i] = cov[i];
}

__device__ __forceinline__ float g0(const float* p, int64_t i) { return p ? __ldg(p + i) : 0.0f; }

// ---------------------------------------------------------------------------
// Backward.  Activations live in shared memory [position][feature] with a
// pitch of kQ = 68 floats (16-byte rows; 68 = 4 mod 32, so the eight
// positions p, p + 8, ... of a thread group fall in different banks).  One
// layer's weights at a time are staged as fp32 rows of the same pitch (rows
// padded with zeros to a multiple of 4).  Every inner loop is register
// blocked 4 x 4: one 16-byte shared load feeds four FMAs, so the loops are
// bound by the FMA pipe rather than by loads.  Threads: 128 = 16 feature
// groups x 8 position groups; position group g owns positions g, g + 8,
// g + 16, g + 24 of the block's 32.
// ---------------------------------------------------------------------------
constexpr int kQ = 68;
constexpr int kBwdThreads = 128;

template <typename W>
__device__ __forceinline__ void stage_layer(const W* __restrict__ src, int n_out, int n_in, float* __restrict__ Ws,
                                            float* __restrict__ bs) {
  const int n_out4 = (n_out + 3) & ~3;
  for (int i = threadIdx.x; i < n_out4 * n_in; i += kBwdThreads) {
    const int o = i / n_in, k = i - o * n_in;
    Ws[o * kQ + k] = o < n_out ? to_f32<W>(__ldg(src + i)) : 0.0f;
  }
  for (int o = threadIdx.x; o < n_out4; o += kBwdThreads) bs[o] = o < n_out ? to_f32<W>(__ldg(src + n_out * n_in + o)) : 0.0f;
}

// out[t][o] = b[o] + sum_k W[o][k] in[t][k] for o < n_out; pre[t][o] keeps
// the value when given, out receives gelu of it when `act`.  Thread (rg, pg)
// computes rows rg, rg + 16, rg + 32, rg + 48 for its four positions.
__device__ __forceinline__ void layer_q(const float* __restrict__ Ws, const float* __restrict__ bs, int n_out,
                                        int n_in, const float* in, float* out, float* pre, bool act) {
  const int pg = threadIdx.x & 7, rg = threadIdx.x >> 3;
  if (rg >= n_out) return;
  float acc[4][4];
  int row[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    row[j] = min(rg + 16 * j, kMaxDim - 1);   // rows past n_out compute on a staged row and are not stored
    const float bj = rg + 16 * j < n_out ? bs[rg + 16 * j] : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = bj;
  }
  for (int k = 0; k < n_in; k += 4) {
    float4 x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const float4*>(in + (pg + 8 * i) * kQ + k);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 w = *reinterpret_cast<const float4*>(Ws + row[j] * kQ + k);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        acc[j][i] = fmaf(w.x, x[i].x, fmaf(w.y, x[i].y, fmaf(w.z, x[i].z, fmaf(w.w, x[i].w, acc[j][i]))));
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int o = rg + 16 * j;
    if (o >= n_out) break;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = pg + 8 * i;
      if (pre) pre[t * kQ + o] = acc[j][i];
      out[t * kQ + o] = act ? gelu(acc[j][i]) : acc[j][i];
    }
  }
}

// acc[kk][i] = sum_o W[o][4 kg + kk] d[t_i][o] over o < n_out4 (d's columns
// and W's rows past n_out are zero).  Thread (kg, pg), kg < n_in / 4.
__device__ __forceinline__ void dgrad_q(const float* __restrict__ Ws, int n_out4, const float* d, int kg,
                                        float (&acc)[4][4]) {
  const int pg = threadIdx.x & 7;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[kk][i] = 0.0f;
  for (int o = 0; o < n_out4; o += 4) {
    float4 dv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) dv[i] = *reinterpret_cast<const float4*>(d + (pg + 8 * i) * kQ + o);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const float4 w = *reinterpret_cast<const float4*>(Ws + (o + jj) * kQ + 4 * kg);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float dd = jj == 0 ? dv[i].x : (jj == 1 ? dv[i].y : (jj == 2 ? dv[i].z : dv[i].w));
        acc[0][i] = fmaf(w.x, dd, acc[0][i]);
        acc[1][i] = fmaf(w.y, dd, acc[1][i]);
        acc[2][i] = fmaf(w.z, dd, acc[2][i]);
        acc[3][i] = fmaf(w.w, dd, acc[3][i]);
      }
    }
  }
}

// dx[t][k] = (sum_o W[o][k] d[t][o]) * gelu'(pre[t][k]), in place over pre.
__device__ __forceinline__ void dgrad_gelu_q(const float* __restrict__ Ws, int n_out4, int n_in, const float* d,
                                             float* pre_dx) {
  const int pg = threadIdx.x & 7, kg = threadIdx.x >> 3;
  if (4 * kg >= n_in) return;
  float acc[4][4];
  dgrad_q(Ws, n_out4, d, kg, acc);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float* q = pre_dx + (pg + 8 * i) * kQ + 4 * kg + kk;
      *q = acc[kk][i] * gelu_grad(*q);
    }
}

// slot += the block's gradient of one layer: W[o][k] += sum_t d[t][o] x[t][k],
// b[o] += sum_t d[t][o], as fp32 reductions (no load to wait for).  Each slot
// element belongs to one task of one thread, so its adds come in program
// order and the sum does not depend on scheduling.
__device__ __forceinline__ void wgrad_q(const float* d, const float* x, int n_out, int n_in, float* slot, int npos) {
  const int ogs = (n_out + 3) >> 2, kgs = n_in >> 2;
  for (int task = threadIdx.x; task < ogs * kgs; task += kBwdThreads) {
    const int kg = task % kgs, og = task / kgs;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.0f;
    for (int t = 0; t < npos; ++t) {
      const float4 dv = *reinterpret_cast<const float4*>(d + t * kQ + 4 * og);
      const float4 xv = *reinterpret_cast<const float4*>(x + t * kQ + 4 * kg);
      const float dd[4] = {dv.x, dv.y, dv.z, dv.w}, xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(dd[a], xx[c], acc[a][c]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int o = 4 * og + a;
      if (o >= n_out) break;
#pragma unroll
      for (int c = 0; c < 4; ++c) atomicAdd(slot + o * n_in + 4 * kg + c, acc[a][c]);
    }
  }
  for (int o = threadIdx.x; o < n_out; o += kBwdThreads) {
    float sb = 0.0f;
    for (int t = 0; t < npos; ++t) sb += d[t * kQ + o];
    atomicAdd(slot + n_out * n_in + o, sb);
  }
}

template <typename T, int F, typename W>
__global__ void __launch_bounds__(kBwdThreads) heads_bwd_kernel(
    GridParams g, HeadsParams hp, const float4* __restrict__ pos, int64_t N, const T* __restrict__ tables,
    const W* __restrict__ weights, const float* __restrict__ latent, const float* __restrict__ raw_in, HeadsGrads go,
    float* __restrict__ grad_tables, float* __restrict__ ws, int n_params) {
  constexpr int B = kHeadsBwdBlock;     // 32 positions
  extern __shared__ float sm[];
  float* z = sm;                        // [B][kQ]; after the last head, dz
  float* p1 = z + B * kQ;               // pre-activations of layer 1, later d(pre 1)
  float* h1 = p1 + B * kQ;
  float* p2 = h1 + B * kQ;              // pre-activations of layer 2, later d(pre 2)
  float* h2 = p2 + B * kQ;
  float* dy = h2 + B * kQ;              // one head's output (first pass) or output adjoint
  float* Ws = dy + B * kQ;              // one staged layer: kMaxDim rows of kQ
  float* bs = Ws + kMaxDim * kQ;        // its biases
  float* dattr = bs + kMaxDim;          // [B][8]: adjoint of raw scale^, rot^, opacity^
  const int IN = hp.in_dim, H = hp.hidden;
  const int pg = threadIdx.x & 7, fg = threadIdx.x >> 3;
  float* slot = ws + (size_t)blockIdx.x * slot_stride(n_params);
  for (int p = threadIdx.x; p < n_params; p += kBwdThreads) slot[p] = 0.0f;

  for (int64_t n0 = (int64_t)blockIdx.x * B; n0 < N; n0 += (int64_t)gridDim.x * B) {
    // z: thread (fg, pg) fills features of its positions; levels for the gather
    for (int e = threadIdx.x; e < B * IN; e += kBwdThreads) {
      const int t = e / IN, k = e - t * IN;
      const int64_t n = n0 + t;
      z[t * kQ + k] = (n < N && latent) ? __ldg(latent + n * IN + k) : 0.0f;
    }
    if (!latent) {
      // one thread per (position, level group): the gather writes its levels of z
      for (int e = threadIdx.x; e < B * kParts; e += kBwdThreads) {
        const int t = e % B, part = e / B;
        const int64_t n = n0 + t;
        if (n >= N) continue;
        float xt[4];
        normalise_position(pos[n], g, xt);
        for (int l = part; l < g.L; l += kParts) {
          float acc[F];
          if constexpr (std::is_same<T, __half>::value && (F == 2 || F == 4))
            encode_level_f16_paired<F>(xt, g, l, tables, acc);
          else
            encode_level<T, F>(xt, g, l, tables, acc);
#pragma unroll
          for (int f = 0; f < F; ++f) z[t * kQ + l * F + f] = acc[f];
        }
      }
    }
    __syncthreads();
    // ---- first pass: raw outputs of the scale, rotation and opacity heads
    // (read from the forward's copy when given) ----
    float raw[8];
    if (raw_in && threadIdx.x < B && n0 + threadIdx.x < N) {
#pragma unroll
      for (int i = 0; i < 8; ++i) raw[i] = __ldg(raw_in + (n0 + threadIdx.x) * 8 + i);
    }
    for (int h = 0; h < 4 && !raw_in; ++h) {
      if (h == 2) continue;
      const W* w = weights + hp.off[h];
      stage_layer<W>(w, H, IN, Ws, bs);
      __syncthreads();
      layer_q(Ws, bs, H, IN, z, h1, nullptr, true);
      __syncthreads();
      w += H * IN + H;
      stage_layer<W>(w, H, H, Ws, bs);
      __syncthreads();
      layer_q(Ws, bs, H, H, h1, h2, nullptr, true);
      __syncthreads();
      w += H * H + H;
      stage_layer<W>(w, hp.rows[h], H, Ws, bs);
      __syncthreads();
      layer_q(Ws, bs, hp.rows[h], H, h2, dy, nullptr, false);
      __syncthreads();
      if (threadIdx.x < B) {
        const int base = h == 0 ? 0 : (h == 1 ? 3 : 7);
        for (int i = 0; i < hp.rows[h]; ++i) raw[base + i] = dy[threadIdx.x * kQ + i];
      }
      __syncthreads();
    }
    // ---- the adjoint of Eq. 11 and Eq. 2, one thread per position ----
    if (threadIdx.x < B) {
      const int64_t n = n0 + threadIdx.x;
      float d[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (n < N) {
        float s[3], r[4], cov_g[6], gs[3], gr[4];
#pragma unroll
        for (int i = 0; i < 3; ++i) s[i] = expf(fminf(raw[i], 20.0f));
        const float nrm = normalise_quat(raw + 3, r);
#pragma unroll
        for (int i = 0; i < 6; ++i) cov_g[i] = g0(go.cov, 6 * n + i);
#pragma unroll
        for (int i = 0; i < 3; ++i) gs[i] = g0(go.scale, 3 * n + i);
#pragma unroll
        for (int i = 0; i < 4; ++i) gr[i] = g0(go.rot, 4 * n + i);
        covariance_backward(s, r, cov_g, gs, gr);
#pragma unroll
        for (int i = 0; i < 3; ++i) d[i] = raw[i] <= 20.0f ? gs[i] * s[i] : 0.0f;
        normalise_quat_backward(r, nrm, gr, d + 3);
        const float o = sigmoidf_(raw[7]);
        d[7] = g0(go.opacity, n) * o * (1.0f - o);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) dattr[threadIdx.x * 8 + i] = d[i];
    }
    __syncthreads();
    // ---- per head: forward keeping pre-activations, then the three layers' gradients ----
    float dz[4][4];   // this thread's (feature group, position group) block of dz, summed over the heads
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int i = 0; i < 4; ++i) dz[kk][i] = 0.0f;
    for (int h = 0; h < 4; ++h) {
      const int rows = hp.rows[h], rows4 = (rows + 3) & ~3;
      const W* w1 = weights + hp.off[h];
      const W* w2 = w1 + H * IN + H;
      const W* w3 = w2 + H * H + H;
      float* s1 = slot + hp.off[h];
      float* s2 = s1 + H * IN + H;
      float* s3 = s2 + H * H + H;
      stage_layer<W>(w1, H, IN, Ws, bs);
      __syncthreads();
      layer_q(Ws, bs, H, IN, z, h1, p1, true);
      __syncthreads();
      stage_layer<W>(w2, H, H, Ws, bs);
      __syncthreads();
      layer_q(Ws, bs, H, H, h1, h2, p2, true);
      // the head's output adjoint, zero past its rows
      for (int e = threadIdx.x; e < B * rows4; e += kBwdThreads) {
        const int t = e / rows4, i = e - t * rows4;
        const int64_t n = n0 + t;
        float v = 0.0f;
        if (i < rows && n < N) {
          if (h == 2)
            v = g0(go.sh, (int64_t)hp.sh_dim * n + i);
          else
            v = dattr[t * 8 + (h == 0 ? 0 : (h == 1 ? 3 : 7)) + i];
        }
        dy[t * kQ + i] = v;
      }
      __syncthreads();
      stage_layer<W>(w3, rows, H, Ws, bs);
      wgrad_q(dy, h2, rows, H, s3, B);
      __syncthreads();
      dgrad_gelu_q(Ws, rows4, H, dy, p2);          // p2 <- d(pre 2)
      __syncthreads();
      stage_layer<W>(w2, H, H, Ws, bs);
      wgrad_q(p2, h1, H, H, s2, B);
      __syncthreads();
      dgrad_gelu_q(Ws, H, H, p2, p1);              // p1 <- d(pre 1)
      __syncthreads();
      stage_layer<W>(w1, H, IN, Ws, bs);
      wgrad_q(p1, z, H, IN, s1, B);
      __syncthreads();
      if (4 * fg < IN) {                           // dz += W1^T d(pre 1)
        float acc[4][4];
        dgrad_q(Ws, H, p1, fg, acc);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
          for (int i = 0; i < 4; ++i) dz[kk][i] += acc[kk][i];
      }
      __syncthreads();   // the next head restages the weights and rewrites the activations
    }
    // dz over z (free now), then the scatter into the tables
    if (4 * fg < IN) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int i = 0; i < 4; ++i) z[(pg + 8 * i) * kQ + 4 * fg + kk] = dz[kk][i];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < B * kParts; e += kBwdThreads) {
      const int t = e % B, part = e / B;
      const int64_t n = n0 + t;
      if (n >= N) continue;
      float xt[4];
      normalise_position(pos[n], g, xt);
      for (int l = part; l < g.L; l += kParts) {
        float d[F];
#pragma unroll
        for (int f = 0; f < F; ++f) d[f] = z[t * kQ + l * F + f];
        scatter_level<F>(xt, g, l, grad_tables, d);
      }
    }
    __syncthreads();
  }
}

// Forward with the backward's register-blocked layers: 32 positions per
// block, 128 threads; the gather takes one (position, level group) per
// thread, the layers run 4 x 4 blocks out of shared memory.
template <typename T, int F, typename W>
__global__ void __launch_bounds__(kBwdThreads) heads_fwd_q_kernel(GridParams g, HeadsParams hp,
                                                                  const float4* __restrict__ pos, int64_t N,
                                                                  const T* __restrict__ tables,
                                                                  const W* __restrict__ weights, HeadsOut out) {
  constexpr int B = kHeadsBwdBlock;
  extern __shared__ float sm[];
  float* z = sm;                        // [B][kQ]
  float* h1 = z + B * kQ;
  float* h2 = h1 + B * kQ;
  float* y = h1;                        // one head's raw outputs (layer 3 no longer needs h1)
  float* Ws = h2 + B * kQ;
  float* bs = Ws + kMaxDim * kQ;
  const int IN = hp.in_dim, H = hp.hidden;
  for (int64_t n0 = (int64_t)blockIdx.x * B; n0 < N; n0 += (int64_t)gridDim.x * B) {
    for (int e = threadIdx.x; e < B * kParts; e += kBwdThreads) {
      const int t = e % B, part = e / B;
      const int64_t n = n0 + t;
      if (n >= N) {
        for (int l = part; l < g.L; l += kParts)
          for (int f = 0; f < F; ++f) z[t * kQ + l * F + f] = 0.0f;
        continue;
      }
      float xt[4];
      normalise_position(pos[n], g, xt);
      for (int l = part; l < g.L; l += kParts) {
        float acc[F];
        if constexpr (std::is_same<T, __half>::value && (F == 2 || F == 4))
          encode_level_f16_paired<F>(xt, g, l, tables, acc);
        else
          encode_level<T, F>(xt, g, l, tables, acc);
#pragma unroll
        for (int f = 0; f < F; ++f) {
          z[t * kQ + l * F + f] = acc[f];
          if (out.latent) out.latent[n * IN + l * F + f] = acc[f];
        }
      }
    }
    float raw[8];
    for (int h = 0; h < 4; ++h) {
      const W* w = weights + hp.off[h];
      const int rows = hp.rows[h];
      __syncthreads();   // z written / the previous head's outputs read
      stage_layer<W>(w, H, IN, Ws, bs);
      __syncthreads();
      layer_q(Ws, bs, H, IN, z, h1, nullptr, true);
      __syncthreads();
      stage_layer<W>(w + H * IN + H, H, H, Ws, bs);
      __syncthreads();
      layer_q(Ws, bs, H, H, h1, h2, nullptr, true);
      __syncthreads();
      stage_layer<W>(w + H * IN + H + H * H + H, rows, H, Ws, bs);
      __syncthreads();
      layer_q(Ws, bs, rows, H, h2, y, nullptr, false);
      __syncthreads();
      if (h == 2) {
        for (int e = threadIdx.x; e < B * rows; e += kBwdThreads) {
          const int t = e / rows, i = e - t * rows;
          const int64_t n = n0 + t;
          if (n < N) out.sh[(int64_t)hp.sh_dim * n + i] = y[t * kQ + i];
        }
      } else if (threadIdx.x < B) {
        const int base = h == 0 ? 0 : (h == 1 ? 3 : 7);
        for (int i = 0; i < rows; ++i) raw[base + i] = y[threadIdx.x * kQ + i];
      }
    }
    if (threadIdx.x < B && n0 + threadIdx.x < N) {
      store_heads(out, n0 + threadIdx.x, raw);
      if (out.raw) {
#pragma unroll
        for (int i = 0; i < 8; ++i) out.raw[(n0 + threadIdx.x) * 8 + i] = raw[i];
      }
    }
  }
}

constexpr size_t kFwdQSmem = ((size_t)3 * kHeadsBwdBlock * kQ + (size_t)kMaxDim * kQ + kMaxDim) * sizeof(float);

// ---------------------------------------------------------------------------
// Forward on the tensor cores, for fp16 tables and weights with in_dim =
// hidden = 64 (the paper's configuration) and an SH head of 48 rows (the
// code takes 16 or 32 as well; only 48, the tested size, is dispatched).
// Persistent CTAs of 256 threads take tiles of 128 positions, two
// threads per position (each gathers half of the levels and handles half of
// every layer's columns).  z is rounded to fp16 into a K-major operand tile;
// then, head by head, three tcgen05.mma chains (M = 128, K = 64; N = 64,
// 64 and the head's rows padded to 16) run with the fp32 accumulators in
// tensor memory: columns 0-63 for the two hidden layers, 64 onwards for the
// output layer.  Each hidden epilogue reads a thread's 32 columns, adds the
// bias, applies the exact GELU and writes the next fp16 operand tile.  All
// weights are staged once per CTA (112 KB of shared memory with the tiles,
// so two CTAs share an SM and one gathers while the other multiplies).
// Every mbarrier wait is bounded; one that runs out sets a device error word
// and the CTA releases its tensor memory and exits.
// ---------------------------------------------------------------------------
constexpr int kHT = 128;
constexpr int kHTThreads = 256;
constexpr int kHTMaxSh = 48;
constexpr uint32_t kHTWait = 1u << 24;
constexpr uint32_t kHTCols = 128;

struct HeadsTcLayout {
  static constexpr int W1 = 0;                                   // 4 x [64][64] fp16, K-major
  static constexpr int W2 = W1 + 4 * 64 * 64 * 2;                // 4 x [64][64]
  static constexpr int W3 = W2 + 4 * 64 * 64 * 2;                // [16 | 16 | sh | 16 rows][64]
  static constexpr int kW3Rows = 48 + kHTMaxSh;
  static constexpr int BIAS = W3 + kW3Rows * 64 * 2;             // fp32: b1 4x64, b2 4x64, b3 kW3Rows
  static constexpr int ZT = BIAS + (512 + kW3Rows) * 4;          // [128][64] fp16
  static constexpr int HT = ZT + kHT * 64 * 2;                   // [128][64] fp16
  static constexpr int MISC = HT + kHT * 64 * 2;                 // mbarrier, TMEM address
  static constexpr int BYTES = MISC + 16;
};
static_assert(HeadsTcLayout::ZT % 128 == 0 && HeadsTcLayout::W3 % 128 == 0, "operand tiles 128-byte aligned");

// W[rows][K] (fp16, row-major in global memory, any 2-byte alignment) -> a
// K-major tile of `rows_pad` rows, the rows past `rows` zero.
__device__ __forceinline__ void stage_kmajor(uint8_t* sm, int soff, const __half* __restrict__ w, int rows,
                                             int rows_pad, int K) {
  for (int i = threadIdx.x; i < rows_pad * K; i += kHTThreads) {
    const int r = i / K, c = i - r * K;
    const __half v = r < rows ? w[(size_t)r * K + c] : __float2half(0.0f);
    *reinterpret_cast<__half*>(sm + soff + tc::kmaj_off(r, c >> 3, K) + (c & 7) * 2) = v;
  }
}

// Output rows of head h padded to 16, and their first row in the W3 tile.
__device__ __forceinline__ int tc_pad(int h, int sh_pad) { return h == 2 ? sh_pad : 16; }
__device__ __forceinline__ int tc_row3(int h, int sh_pad) { return h < 3 ? 16 * h : 32 + sh_pad; }

// Gather of the split forward: one thread per position, two levels (one
// 16-byte chunk of 8 fp16 features, rounded as the fused kernel rounds them)
// at a time, into z16 rows of 64 halves and into the fp32 latent when given.
// At 64 warps per SM the corner loads keep far more requests in flight than
// the fused kernel's 16 warps per SM.
template <int F>
__global__ void __launch_bounds__(128) heads_gather_kernel(GridParams g, const float4* __restrict__ pos, int64_t N,
                                                          const __half* __restrict__ tables, uint4* __restrict__ z16,
                                                          float* __restrict__ latent) {
  static_assert(F == 4, "the split forward takes L = 16, F = 4");
  pdl_release();
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N; n += (int64_t)gridDim.x * blockDim.x) {
    float xt[4];
    normalise_position(pos[n], g, xt);
#pragma unroll 1
    for (int kc = 0; kc < 8; ++kc) {
      float a[4], b[4];
      encode_level_f16_paired<4>(xt, g, 2 * kc, tables, a);
      encode_level_f16_paired<4>(xt, g, 2 * kc + 1, tables, b);
      z16[n * 8 + kc] = make_uint4(tc::pack_half2(a[0], a[1]), tc::pack_half2(a[2], a[3]), tc::pack_half2(b[0], b[1]),
                                   tc::pack_half2(b[2], b[3]));
      if (latent) {
        float4* zl = reinterpret_cast<float4*>(latent + n * 64 + kc * 8);
        zl[0] = make_float4(a[0], a[1], a[2], a[3]);
        zl[1] = make_float4(b[0], b[1], b[2], b[3]);
      }
    }
  }
}

// FROM_Z: the layers of the split forward, z read from the gather's z16
// rows (launched programmatically dependent on the gather: weights and
// tensor memory are set up before waiting for it); otherwise the fused
// forward that gathers z itself.
template <int F, bool FROM_Z>
__global__ void __launch_bounds__(kHTThreads, 2) heads_fwd_tc_kernel(GridParams g, HeadsParams hp,
                                                                      const float4* __restrict__ pos, int64_t N,
                                                                      const __half* __restrict__ tables,
                                                                      const __half* __restrict__ weights,
                                                                      HeadsOut out) {
  using Lay = HeadsTcLayout;
  constexpr int IN = 64;
  extern __shared__ __align__(1024) uint8_t hsm[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (kHT - 1), half = tid >> 7;
  float* bias = reinterpret_cast<float*>(hsm + Lay::BIAS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(hsm + Lay::MISC + 8);
  const uint32_t mbar = tc::smem_u32(hsm + Lay::MISC);
  const int sh_rows = hp.sh_dim, sh_pad = (sh_rows + 15) & ~15;
  // ---- all weights and biases, once per CTA ----
#pragma unroll 1
  for (int h = 0; h < 4; ++h) {
    const __half* w1 = weights + hp.off[h];
    const __half* w2 = w1 + 64 * IN + 64;
    const __half* w3 = w2 + 64 * 64 + 64;
    const int rows = hp.rows[h], pad = tc_pad(h, sh_pad), r3 = tc_row3(h, sh_pad);
    stage_kmajor(hsm, Lay::W1 + h * 8192, w1, 64, 64, IN);
    stage_kmajor(hsm, Lay::W2 + h * 8192, w2, 64, 64, 64);
    stage_kmajor(hsm, Lay::W3 + r3 * 128, w3, rows, pad, 64);
    for (int o = tid; o < 64; o += kHTThreads) {
      bias[h * 64 + o] = __half2float(w1[64 * IN + o]);
      bias[256 + h * 64 + o] = __half2float(w2[64 * 64 + o]);
    }
    for (int o = tid; o < pad; o += kHTThreads) bias[512 + r3 + o] = o < rows ? __half2float(w3[rows * 64 + o]) : 0.0f;
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), kHTCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(mbar, 1);
    tc::mbar_fence_init();
  }
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t sbase = tc::smem_u32(hsm);
  uint32_t phase = 0;
  bool failed = false;
  if constexpr (FROM_Z) pdl_wait();   // the gather's z16 rows are complete and visible

  // one K = 64 chain into TMEM column dcol: A rows = positions, B rows = outputs
  auto mma_chain = [&](uint32_t a_tile, uint32_t b_tile, int n_out, uint32_t dcol) {
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc::mma_f16(tmem + dcol, tc::smem_desc(a_tile + k * 256, 128, 1024), tc::smem_desc(b_tile + k * 256, 128, 1024),
                    tc::idesc_f16_f32(kHT, n_out), k > 0 ? 1u : 0u);
      tc::mma_commit(mbar);
    }
    const bool ok = tc::mbar_wait_bounded(mbar, phase, kHTWait);
    phase ^= 1u;
    const bool bad = __syncthreads_or(!ok);
    tc::fence_after_sync();
    return !bad;
  };
  // hidden epilogue: this thread's 32 columns + bias, GELU, fp16 into HT
  auto hidden_epilogue = [&](const float* b) {
    float v[32];
    tc::tmem_ld32(tmem + lane + half * 32, v);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = tc::pack_half2(gelu_fast(v[2 * i] + b[half * 32 + 2 * i]),
                             gelu_fast(v[2 * i + 1] + b[half * 32 + 2 * i + 1]));
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *reinterpret_cast<uint4*>(hsm + Lay::HT + tc::kmaj_off(row, half * 4 + q, 64)) =
          make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
  };

  for (int64_t tile = blockIdx.x; tile * kHT < N; tile += gridDim.x) {
    const int64_t n = tile * kHT + row;
    const bool valid = n < N;
    if constexpr (FROM_Z) {
      // the tile's z rows: a warp copies 8 rows x 4 chunks (64 contiguous
      // bytes of each row), which land in distinct banks of the K-major tile
      for (int i = tid; i < kHT * 8; i += kHTThreads) {
        const int w = i >> 5, l = i & 31;
        const int r = 8 * (w >> 1) + (l & 7), kc = 4 * (w & 1) + (l >> 3);
        const int64_t nr = tile * kHT + r;
        const uint4 v = nr < N ? __ldg(out.z16 + nr * 8 + kc) : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(hsm + Lay::ZT + tc::kmaj_off(r, kc, IN)) = v;
      }
    }
    float xt[4] = {0.f, 0.f, 0.f, 0.f};
    if (!FROM_Z && valid) normalise_position(pos[n], g, xt);
    // ---- gather: chunks kc = 4 half .. 4 half + 3 (8 features, 8 / F levels each) ----
#pragma unroll 1
    for (int kc = half * 4; kc < (FROM_Z ? 0 : half * 4 + 4); ++kc) {
      float zv[8];
#pragma unroll
      for (int q = 0; q < 8 / F; ++q) {
        float acc[F];
        if (valid) {
          encode_level_f16_paired<F>(xt, g, kc * (8 / F) + q, tables, acc);
        } else {
#pragma unroll
          for (int f = 0; f < F; ++f) acc[f] = 0.f;
        }
#pragma unroll
        for (int f = 0; f < F; ++f) zv[q * F + f] = acc[f];
      }
      if (out.latent && valid) {
        float4* zl = reinterpret_cast<float4*>(out.latent + n * IN + kc * 8);
        zl[0] = make_float4(zv[0], zv[1], zv[2], zv[3]);
        zl[1] = make_float4(zv[4], zv[5], zv[6], zv[7]);
      }
      *reinterpret_cast<uint4*>(hsm + Lay::ZT + tc::kmaj_off(row, kc, IN)) =
          make_uint4(tc::pack_half2(zv[0], zv[1]), tc::pack_half2(zv[2], zv[3]), tc::pack_half2(zv[4], zv[5]),
                     tc::pack_half2(zv[6], zv[7]));
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();

    float raw[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int h = 0; h < 4; ++h) {
      const int pad = tc_pad(h, sh_pad), r3 = tc_row3(h, sh_pad);
      if (!mma_chain(sbase + Lay::ZT, sbase + Lay::W1 + h * 8192, 64, 0)) { failed = true; break; }
      hidden_epilogue(bias + h * 64);
      if (!mma_chain(sbase + Lay::HT, sbase + Lay::W2 + h * 8192, 64, 0)) { failed = true; break; }
      hidden_epilogue(bias + 256 + h * 64);
      if (!mma_chain(sbase + Lay::HT, sbase + Lay::W3 + r3 * 128, pad, 64)) { failed = true; break; }
      const float* b3 = bias + 512 + r3;
      if (h == 2) {
        // SH rows 0-31 on warps 0-3, rows 32-47 on warps 4-7; rows are 16-byte aligned (sh_dim % 16 == 0)
        float4* dst = reinterpret_cast<float4*>(out.sh + (int64_t)sh_rows * n);
        if (half == 0) {
          float v[32];
          if (pad >= 32) {
            tc::tmem_ld32(tmem + lane + 64, v);
          } else {
            tc::tmem_ld16(tmem + lane + 64, v);
#pragma unroll
            for (int i = 16; i < 32; ++i) v[i] = 0.0f;
          }
          if (valid) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (4 * q < sh_rows)
                dst[q] = make_float4(v[4 * q] + b3[4 * q], v[4 * q + 1] + b3[4 * q + 1], v[4 * q + 2] + b3[4 * q + 2],
                                     v[4 * q + 3] + b3[4 * q + 3]);
          }
        } else if (pad > 32) {
          float v[16];
          tc::tmem_ld16(tmem + lane + 96, v);
          if (valid) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[8 + q] = make_float4(v[4 * q] + b3[32 + 4 * q], v[4 * q + 1] + b3[33 + 4 * q],
                                       v[4 * q + 2] + b3[34 + 4 * q], v[4 * q + 3] + b3[35 + 4 * q]);
          }
        }
      } else if (half == 0) {
        float v[16];
        tc::tmem_ld16(tmem + lane + 64, v);
        if (h == 0) {
#pragma unroll
          for (int i = 0; i < 3; ++i) raw[i] = v[i] + b3[i];
        } else if (h == 1) {
#pragma unroll
          for (int i = 0; i < 4; ++i) raw[3 + i] = v[i] + b3[i];
        } else {
          raw[7] = v[0] + b3[0];
        }
      }
      tc::fence_before_sync();
      __syncthreads();   // TMEM columns and HT free for the next head
    }
    if (failed) break;
    if (half == 0 && valid) {
      store_heads(out, n, raw);
      if (out.raw) {
        float4* r = reinterpret_cast<float4*>(out.raw + n * 8);
        r[0] = make_float4(raw[0], raw[1], raw[2], raw[3]);
        r[1] = make_float4(raw[4], raw[5], raw[6], raw[7]);
      }
    }
  }

  // ---- teardown: nothing of ours may still be writing TMEM when it is freed ----
  if (failed) {
    if (tid == 0) atomicExch(&g_heads_device_error, 1);
    tc::mbar_wait_bounded(mbar, phase ^ 1u, kHTWait);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kHTCols);
  }
}

// ---------------------------------------------------------------------------
// Backward on the tensor cores, for the configuration of heads_fwd_tc_kernel
// when the forward's z (fp32 latent) and raw head outputs are given.  One
// persistent CTA of 256 threads per SM takes tiles of 128 positions; thread
// (row, half) owns position `row` and columns half*32 .. of every M = 128
// product.  Per head, with fp16 operand tiles and fp32 accumulators in TMEM
// (columns: P1 0-63, P2 64-127, D 128-191, dz 192-255):
//   P1 = z W1^T, h1 = gelu(P1 + b1);  P2 = h1 W2^T, h2 = gelu(P2 + b2);
//   dy = the head's output adjoint (Eq. 11 / Eq. 2 backward, or dL/dsh);
//   D = dy W3, d2 = D * gelu'(P2 + b2);  D = d2 W2, d1 = D * gelu'(P1 + b1);
//   dz += d1 W1 (accumulated over the heads);
//   dW3 = dy^T h2, dW2 = d2^T h1, dW1 = d1^T z as M = 64 products over the
//   tile's 128 positions (rows of dW3 padded to 64 with zero columns of dy),
//   added to the CTA's workspace slot by vector reductions whose every element
//   has one owning thread (so the sum does not depend on scheduling).
// The slot is padded per head: [W1 64x64][b1][W2 64x64][b2][W3 64x64][b3 64]
// so every row is 16-byte aligned; heads_reduce_slots_tc maps it back to the
// packed order.  dz is then scattered into the tables as the SIMT kernel does.
// GELU and its derivative use the rational erf of gelu_fast (the operands
// they feed are fp16).
// ---------------------------------------------------------------------------
constexpr int kHBHead = 3 * (64 * 64 + 64);   // floats of one head in the padded slot
constexpr int kHBSlot = 4 * kHBHead;
constexpr int kHBW2 = 64 * 64 + 64, kHBW3 = 2 * (64 * 64 + 64), kHBB3 = kHBW3 + 64 * 64;

__device__ __forceinline__ float gelu_grad_fast(float x) {
  const float u = fabsf(x) * 0.70710678118654752f;
  float p = fmaf(u, 0.0000430638f, 0.0002765672f);
  p = fmaf(p, u, 0.0001520143f);
  p = fmaf(p, u, 0.0092705272f);
  p = fmaf(p, u, 0.0422820123f);
  p = fmaf(p, u, 0.0705230784f);
  p = fmaf(p, u, 1.0f);
  p *= p;
  p *= p;
  p *= p;
  p *= p;
  const float he = 0.5f * __fdividef(1.0f, p);   // (1 - erf(|x| / sqrt 2)) / 2
  const float Phi = x >= 0.0f ? 1.0f - he : he;
  return Phi + x * 0.39894228040143268f * __expf(-0.5f * x * x);
}

struct HeadsBwdLayout {
  static constexpr int W1 = HeadsTcLayout::W1, W2 = HeadsTcLayout::W2, W3 = HeadsTcLayout::W3;
  static constexpr int BIAS = HeadsTcLayout::BIAS;
  static constexpr int ZT = 81920;                    // [128][64] fp16 tiles, K-major
  static constexpr int H1 = ZT + 16384;
  static constexpr int H2 = H1 + 16384;
  static constexpr int DY = H2 + 16384;               // dy, later d1
  static constexpr int D2 = DY + 16384;
  static constexpr int PART = D2 + 16384;             // [4][64] fp32 column partial sums
  static constexpr int BACC = PART + 1024;            // [4 heads][3][64] fp32 bias gradients
  static constexpr int MISC = BACC + 3072;
  static constexpr int SCL = MISC + 16;               // operand scales: [4][2] weight-bound exponents,
                                                      // [8 warps][4 heads] tile maxima of |dy|
  static constexpr int BYTES = SCL + 256;
};
static_assert(HeadsTcLayout::BIAS + (512 + HeadsTcLayout::kW3Rows) * 4 <= HeadsBwdLayout::ZT, "layout overlap");

// Power of two that brings a magnitude m below 2^10 (into [2^9, 2^10)): the
// fp16 gradient tiles of the tensor-core backward are stored scaled by such
// factors, so that small gradients keep fp16's 11-bit precision instead of
// going subnormal, and no scaled value comes near fp16's maximum (65504).
// Exact; 1 for m = 0 or a non-finite m.
__device__ __forceinline__ float heads_pow2_below(float m, int target) {
  if (!(m > 0.f) || !isfinite(m)) return 1.0f;
  int e;
  frexpf(m, &e);   // m = f 2^e, f in [0.5, 1)
  return ldexpf(1.0f, max(-100, min(100, target - e)));
}
static_assert(HeadsBwdLayout::BYTES <= 227 * 1024, "backward tiles exceed one CTA's shared memory");

template <int F>
__global__ void __launch_bounds__(kHTThreads, 1) heads_bwd_tc_kernel(
    GridParams g, HeadsParams hp, const float4* __restrict__ pos, int64_t N, const __half* __restrict__ weights,
    const float* __restrict__ latent, const float* __restrict__ raw_in, HeadsGrads go,
    float* __restrict__ grad_tables, float* __restrict__ ws) {
  using Lay = HeadsBwdLayout;
  constexpr int IN = 64;
  extern __shared__ __align__(1024) uint8_t bsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lid = tid & 31;
  const int row = tid & (kHT - 1), half = tid >> 7;
  float* bias = reinterpret_cast<float*>(bsm + Lay::BIAS);
  float* part = reinterpret_cast<float*>(bsm + Lay::PART);
  float* bacc = reinterpret_cast<float*>(bsm + Lay::BACC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bsm + Lay::MISC + 8);
  const uint32_t mbar = tc::smem_u32(bsm + Lay::MISC);
  const int sh_rows = hp.sh_dim, sh_pad = (sh_rows + 15) & ~15;
  float* slot = ws + (size_t)blockIdx.x * slot_stride(kHBSlot);
  for (int p = tid; p < kHBSlot; p += kHTThreads) slot[p] = 0.f;
  for (int p = tid; p < 4 * 3 * 64; p += kHTThreads) bacc[p] = 0.f;
#pragma unroll 1
  for (int h = 0; h < 4; ++h) {
    const __half* w1 = weights + hp.off[h];
    const __half* w2 = w1 + 64 * IN + 64;
    const __half* w3 = w2 + 64 * 64 + 64;
    const int rows = hp.rows[h], pad = tc_pad(h, sh_pad), r3 = tc_row3(h, sh_pad);
    stage_kmajor(bsm, Lay::W1 + h * 8192, w1, 64, 64, IN);
    stage_kmajor(bsm, Lay::W2 + h * 8192, w2, 64, 64, 64);
    stage_kmajor(bsm, Lay::W3 + r3 * 128, w3, rows, pad, 64);
    for (int o = tid; o < 64; o += kHTThreads) {
      bias[h * 64 + o] = __half2float(w1[64 * IN + o]);
      bias[256 + h * 64 + o] = __half2float(w2[64 * 64 + o]);
    }
  }
  // Weight bounds of the dgrad chain, per head: |d2| <= max|dy| * B3 * 1.2 and
  // |d1| <= max|d2| * B2 * 1.2, with B the largest absolute column sum of W3
  // (W2) and 1.2 above GELU's largest slope (1.129).  Their powers of two
  // rescale d2 and d1 so that both stay below 2^10 after dy is scaled there.
  int* wexp = reinterpret_cast<int*>(bsm + Lay::SCL);         // [h][0] for d2, [h][1] for d1
  float* dymax = reinterpret_cast<float*>(bsm + Lay::SCL + 32);
  float* dzinv = reinterpret_cast<float*>(bsm + Lay::SCL + 160);   // [4] unscaling of each head's dz
  if (tid < 8) wexp[tid] = 0;
  __syncthreads();
  {
    const int h = tid >> 6, j = tid & 63;
    const __half* w2 = weights + hp.off[h] + 64 * IN + 64;
    const __half* w3 = w2 + 64 * 64 + 64;
    float b3 = 0.f, b2 = 0.f;
    for (int i = 0; i < hp.rows[h]; ++i) b3 += fabsf(__half2float(w3[i * 64 + j]));
    for (int i = 0; i < 64; ++i) b2 += fabsf(__half2float(w2[i * 64 + j]));
    // non-negative floats order like their bit patterns
    atomicMax(wexp + 2 * h, __float_as_int(1.2f * b3));
    atomicMax(wexp + 2 * h + 1, __float_as_int(1.2f * b2));
  }
  __syncthreads();
  if (tid < 8) {
    const float b = __int_as_float(wexp[tid]);
    int e = 0;
    if (b > 0.f && isfinite(b)) frexpf(b, &e);   // b < 2^e
    wexp[tid] = max(-60, min(60, e));
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(mbar, 1);
    tc::mbar_fence_init();
  }
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t sbase = tc::smem_u32(bsm);
  // each head's dz has its own accumulator (its own operand scale): DZ + 64 h
  const uint32_t P1 = tmem, P2 = tmem + 64, DD = tmem + 128, DZ = tmem + 192;
  // Row m of a 64-row (M = 64) accumulator sits in TMEM lane (m % 16) + 32 (m / 16):
  // warp w holds rows 16 (w % 4) + lane for lanes below 16, columns (w / 4) * 32 ..
  const int wrow = (warp & 3) * 16 + lid;
  const bool wrow_ok = lid < 16;
  const int wcol = (warp >> 2) * 32;
  uint32_t phase = 0;
  bool failed = false;

  // K-major tile with L columns; MN-major read of the same tile
  auto kdesc = [&](uint32_t off, int L, int k) { return tc::smem_desc(sbase + off + k * 256, 128, 16 * L); };
  auto mdesc = [&](uint32_t off, int L, int k) { return tc::smem_desc(sbase + off + k * 32 * L, 16 * L, 128); };
  auto wait_mma = [&]() -> bool {
    if (tid == 0) tc::mma_commit(mbar);
    const bool ok = tc::mbar_wait_bounded(mbar, phase, kHTWait);
    phase ^= 1u;
    const bool bad = __syncthreads_or(!ok);
    tc::fence_after_sync();
    return !bad;
  };
  auto store_row = [&](int off, const float v[32], float sc) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) pk[i] = tc::pack_half2(v[2 * i] * sc, v[2 * i + 1] * sc);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *reinterpret_cast<uint4*>(bsm + off + tc::kmaj_off(row, half * 4 + q, 64)) =
          make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  };
  auto tiles_ready = [&]() {
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
  };
  // column sums of this thread's 32 values over the tile's 128 rows: warp sums
  // into part[warp % 4][col], then (after the next barrier) bias_add adds
  // them in a fixed order
  auto col_partial = [&](const float v[32], float inv) {
    float t[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) t[i] = v[i] * inv;
    part[(warp & 3) * 64 + half * 32 + lid] = warp_column_sum(t);
  };
  auto bias_add = [&](float* dst) {
    if (tid < 64) dst[tid] += part[tid] + part[64 + tid] + part[128 + tid] + part[192 + tid];
  };
  auto flush64 = [&](uint32_t acc, float* dst, int nrows, float inv) {   // dst: 64 x 64 rows of the slot
    float a[32];
    tc::tmem_ld32(acc + lane + wcol, a);
#pragma unroll
    for (int i = 0; i < 32; ++i) a[i] *= inv;
    if (wrow_ok && wrow < nrows) slot_add32(dst + wrow * 64 + wcol, a);
  };

  for (int64_t tile = blockIdx.x; tile * kHT < N && !failed; tile += gridDim.x) {
    const int64_t n = tile * kHT + row;
    const bool valid = n < N;
    // ---- z (fp32 latent) -> fp16 K-major tile: a warp copies 8 rows x 4 float4 ----
    for (int i = tid; i < kHT * 16; i += kHTThreads) {
      const int w = i >> 5, l = i & 31;
      const int r = 8 * (w >> 2) + (l & 7), c4 = 4 * (w & 3) + (l >> 3);
      const int64_t nr = tile * kHT + r;
      const float4 v = nr < N ? __ldg(reinterpret_cast<const float4*>(latent + nr * IN) + c4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<uint2*>(bsm + Lay::ZT + tc::kmaj_off(r, c4 >> 1, IN) + (c4 & 1) * 8) =
          make_uint2(tc::pack_half2(v.x, v.y), tc::pack_half2(v.z, v.w));
    }
    // ---- the adjoint of Eq. 11 and Eq. 2 from the saved raw outputs ----
    float da[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (half == 0 && valid) {
      float raw[8], s[3], r[4], cov_g[6], gs[3], gr[4];
#pragma unroll
      for (int i = 0; i < 8; ++i) raw[i] = __ldg(raw_in + n * 8 + i);
#pragma unroll
      for (int i = 0; i < 3; ++i) s[i] = expf(fminf(raw[i], 20.0f));
      const float nrm = normalise_quat(raw + 3, r);
#pragma unroll
      for (int i = 0; i < 6; ++i) cov_g[i] = g0(go.cov, 6 * n + i);
#pragma unroll
      for (int i = 0; i < 3; ++i) gs[i] = g0(go.scale, 3 * n + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) gr[i] = g0(go.rot, 4 * n + i);
      covariance_backward(s, r, cov_g, gs, gr);
#pragma unroll
      for (int i = 0; i < 3; ++i) da[i] = raw[i] <= 20.0f ? gs[i] * s[i] : 0.0f;
      normalise_quat_backward(r, nrm, gr, da + 3);
      const float o = sigmoidf_(raw[7]);
      da[7] = g0(go.opacity, n) * o * (1.0f - o);
    }
    {
      // this tile's largest |dy| per head (scale, rotation, SH, opacity)
      float m[4] = {fmaxf(fabsf(da[0]), fmaxf(fabsf(da[1]), fabsf(da[2]))),
                    fmaxf(fmaxf(fabsf(da[3]), fabsf(da[4])), fmaxf(fabsf(da[5]), fabsf(da[6]))), 0.f, fabsf(da[7])};
      if (valid && go.sh)
        for (int c = half * 32; c < min(sh_rows, half * 32 + 32); ++c)
          m[2] = fmaxf(m[2], fabsf(__ldg(go.sh + (int64_t)sh_rows * n + c)));
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float wm = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m[h])));
        if (lid == 0) dymax[warp * 4 + h] = wm;
      }
    }
    tiles_ready();

#pragma unroll 1
    for (int h = 0; h < 4; ++h) {
      const int rows = hp.rows[h], pad = tc_pad(h, sh_pad), r3 = tc_row3(h, sh_pad);
      const float* b1 = bias + h * 64;
      const float* b2 = bias + 256 + h * 64;
      float* sh_slot = slot + h * kHBHead;
      float* bh = bacc + h * 192;   // db1 | db2 | db3
      // operand scales of this head on this tile: dy below 2^10 by its tile
      // maximum, d2 and d1 further by the weight bounds (all powers of two)
      float mdy = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) mdy = fmaxf(mdy, dymax[w * 4 + h]);
      const float s_dy = heads_pow2_below(mdy, 10);
      const float s_d2 = s_dy * ldexpf(1.0f, -wexp[2 * h]);
      const float s_d1 = s_d2 * ldexpf(1.0f, -wexp[2 * h + 1]);
      const float i_dy = 1.0f / s_dy, i_d2 = 1.0f / s_d2, i_d1 = 1.0f / s_d1;
      // ---- P1 = z W1^T ----
      if (tid == 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_f16(P1, kdesc(Lay::ZT, 64, k), kdesc(Lay::W1 + h * 8192, 64, k), tc::idesc_f16_f32(kHT, 64), k > 0);
      }
      if (!wait_mma()) { failed = true; break; }
      {
        float v[32];
        tc::tmem_ld32(P1 + lane + half * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = gelu_fast(v[i] + b1[half * 32 + i]);
        store_row(Lay::H1, v, 1.0f);
      }
      tiles_ready();
      // ---- P2 = h1 W2^T ----
      if (tid == 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_f16(P2, kdesc(Lay::H1, 64, k), kdesc(Lay::W2 + h * 8192, 64, k), tc::idesc_f16_f32(kHT, 64), k > 0);
      }
      if (!wait_mma()) { failed = true; break; }
      {
        float v[32];
        tc::tmem_ld32(P2 + lane + half * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = gelu_fast(v[i] + b2[half * 32 + i]);
        store_row(Lay::H2, v, 1.0f);
        // the head's output adjoint, zero past its rows (64 columns: rows of dW3 pad to 64)
        float dy[32];
        if (h == 2) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = half * 32 + i;
            dy[i] = (valid && c < rows && go.sh) ? __ldg(go.sh + (int64_t)sh_rows * n + c) : 0.f;
          }
        } else {
          const int base = h == 0 ? 0 : (h == 1 ? 3 : 7);
#pragma unroll
          for (int i = 0; i < 32; ++i) dy[i] = 0.f;
          if (half == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) dy[i] = i < rows ? da[min(base + i, 7)] : 0.f;
          }
        }
        store_row(Lay::DY, dy, s_dy);
        col_partial(dy, 1.0f);
      }
      tiles_ready();
      bias_add(bh + 128);
      // ---- D = dy W3 ----
      if (tid == 0) {
        tc::fence_after_sync();
        for (int k = 0; k < pad / 16; ++k)
          tc::mma_f16(DD, kdesc(Lay::DY, 64, k), mdesc(Lay::W3 + r3 * 128, 64, k), tc::idesc_f16t_f32(kHT, 64, false, true),
                      k > 0);
      }
      if (!wait_mma()) { failed = true; break; }
      {
        float d[32], p[32];
        tc::tmem_ld32(DD + lane + half * 32, d);
        tc::tmem_ld32(P2 + lane + half * 32, p);
#pragma unroll
        for (int i = 0; i < 32; ++i) d[i] *= gelu_grad_fast(p[i] + b2[half * 32 + i]);
        // d holds d2 s_dy; stored as d2 s_d2
        store_row(Lay::D2, d, s_d2 * i_dy);
        col_partial(d, i_dy);
      }
      tiles_ready();
      bias_add(bh + 64);
      // ---- dW3 = dy^T h2 (into P2's columns, free now); D = d2 W2 ----
      if (tid == 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc::mma_f16(P2, mdesc(Lay::DY, 64, k), mdesc(Lay::H2, 64, k), tc::idesc_f16t_f32(64, 64, true, true), k > 0);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_f16(DD, kdesc(Lay::D2, 64, k), mdesc(Lay::W2 + h * 8192, 64, k), tc::idesc_f16t_f32(kHT, 64, false, true),
                      k > 0);
      }
      if (!wait_mma()) { failed = true; break; }
      flush64(P2, sh_slot + kHBW3, rows, i_dy);
      {
        float d[32], p[32];
        tc::tmem_ld32(DD + lane + half * 32, d);
        tc::tmem_ld32(P1 + lane + half * 32, p);
#pragma unroll
        for (int i = 0; i < 32; ++i) d[i] *= gelu_grad_fast(p[i] + b1[half * 32 + i]);
        // d holds d1 s_d2; stored as d1 s_d1 over dy (its products are done)
        store_row(Lay::DY, d, s_d1 * i_d2);
        col_partial(d, i_d2);
      }
      tiles_ready();
      bias_add(bh);
      // ---- dW2 = d2^T h1 (P2's columns), dW1 = d1^T z (P1's), dz += d1 W1 ----
      if (tid == 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc::mma_f16(P2, mdesc(Lay::D2, 64, k), mdesc(Lay::H1, 64, k), tc::idesc_f16t_f32(64, 64, true, true), k > 0);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc::mma_f16(P1, mdesc(Lay::DY, 64, k), mdesc(Lay::ZT, 64, k), tc::idesc_f16t_f32(64, 64, true, true), k > 0);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_f16(DZ + 64 * h, kdesc(Lay::DY, 64, k), mdesc(Lay::W1 + h * 8192, 64, k),
                      tc::idesc_f16t_f32(kHT, 64, false, true), k > 0 ? 1u : 0u);
      }
      if (!wait_mma()) { failed = true; break; }
      flush64(P2, sh_slot + kHBW2, 64, i_d2);
      flush64(P1, sh_slot, 64, i_d1);
      if (tid == 0) dzinv[h] = i_d1;   // read after the loop
      tc::fence_before_sync();
      __syncthreads();   // the next head rewrites P1, P2 and the tiles
    }
    if (failed) break;
    // ---- dz (the heads' accumulators, each unscaled) into the tables: this
    // thread's levels half*8 .. half*8 + 7 ----
    {
      float dz[32];
      tc::tmem_ld32(DZ + lane + half * 32, dz);
#pragma unroll
      for (int i = 0; i < 32; ++i) dz[i] *= dzinv[0];
#pragma unroll 1
      for (int h = 1; h < 4; ++h) {
        float t[32];
        tc::tmem_ld32(DZ + 64 * h + lane + half * 32, t);
        const float inv = dzinv[h];
#pragma unroll
        for (int i = 0; i < 32; ++i) dz[i] = fmaf(t[i], inv, dz[i]);
      }
      if (valid) {
        float xt[4];
        normalise_position(pos[n], g, xt);
#pragma unroll 1
        for (int q = 0; q < 8; ++q) scatter_level<F>(xt, g, half * 8 + q, grad_tables, dz + 4 * q);
      }
    }
    tc::fence_before_sync();
    __syncthreads();
  }

  if (failed) {
    if (tid == 0) atomicExch(&g_heads_device_error, 1);
    tc::mbar_wait_bounded(mbar, phase ^ 1u, kHTWait);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (!failed)
    for (int p = tid; p < 4 * 3 * 64; p += kHTThreads) {
      const int h = p / 192, k = p - h * 192, which = k >> 6, o = k & 63;
      float* dst = slot + h * kHBHead + (which == 0 ? 64 * 64 : which == 1 ? kHBW2 + 64 * 64 : kHBB3);
      dst[o] += bacc[p];
    }
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// grad_weights (packed) += the padded slots of heads_bwd_tc_kernel, summed
// over the slots in a fixed order.
__global__ void heads_reduce_slots_tc(const float* __restrict__ ws, int n_slots, HeadsParams hp, int n_params,
                                      float* __restrict__ out) {
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < n_params; p += gridDim.x * blockDim.x) {
    int h = 0;
    while (h < 3 && p >= hp.off[h + 1]) ++h;
    const int q = p - hp.off[h];
    const int w3_end = kHBW3 + hp.rows[h] * 64;
    const int src = h * kHBHead + (q < w3_end ? q : kHBB3 + (q - w3_end));
    float s = 0.0f;
    for (int c = 0; c < n_slots; ++c) s += ws[(size_t)c * slot_stride(kHBSlot) + src];
    out[p] += s;
  }
}

__global__ void heads_reduce_slots(const float* __restrict__ ws, int n_slots, int n_params, float* __restrict__ out) {
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < n_params; p += gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int c = 0; c < n_slots; ++c) s += ws[(size_t)c * slot_stride(n_params) + p];
    out[p] += s;
  }
}

constexpr size_t kBwdSmem = ((size_t)6 * kHeadsBwdBlock * kQ + (size_t)kMaxDim * kQ + kMaxDim +
                             (size_t)kHeadsBwdBlock * 8) * sizeof(float);

int validate_heads(const spin4d_grid_desc* g, const spin4d_heads_desc* h) {
  if (!h) return SPIN4D_ERR_INVALID;
  if (h->in_dim != g->L * g->F) return SPIN4D_ERR_INVALID;
  if (h->hidden < 1 || h->sh_dim < 1 || h->w_dtype < 0 || h->w_dtype > 1) return SPIN4D_ERR_INVALID;
  if (h->in_dim > kMaxDim || h->hidden > kMaxDim || h->sh_dim > kMaxDim) return SPIN4D_ERR_UNSUPPORTED;
  // the backward's register blocking takes features four at a time
  if (h->in_dim % 4 || h->hidden % 4) return SPIN4D_ERR_UNSUPPORTED;
  return SPIN4D_OK;
}

HeadsParams make_heads(const spin4d_heads_desc* h) {
  HeadsParams p;
  p.in_dim = h->in_dim;
  p.hidden = h->hidden;
  p.sh_dim = h->sh_dim;
  const int rows[4] = {3, 4, h->sh_dim, 1};
  int o = 0;
  for (int k = 0; k < 4; ++k) {
    p.rows[k] = rows[k];
    p.off[k] = o;
    o += h->hidden * h->in_dim + h->hidden + h->hidden * h->hidden + h->hidden + rows[k] * h->hidden + rows[k];
  }
  return p;
}

int64_t param_count(const spin4d_heads_desc* h) {
  int64_t n = 0;
  const int rows[4] = {3, 4, h->sh_dim, 1};
  for (int k = 0; k < 4; ++k)
    n += (int64_t)h->hidden * h->in_dim + h->hidden + (int64_t)h->hidden * h->hidden + h->hidden +
         (int64_t)rows[k] * h->hidden + rows[k];
  return n;
}

// three blocks fit an SM (shared memory): the grid is three per SM, so there is no second wave
int bwd_blocks(int64_t N) { return persistent_blocks((N + kHeadsBwdBlock - 1) / kHeadsBwdBlock, 3); }

template <typename T, int F, typename W>
struct HeadsLaunch {
  // the tensor-core forward (fp16 tables and weights, in_dim = hidden = 64)
  template <bool FROM_Z>
  static int configure_tc(int smem) {
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (configured[dev]) return SPIN4D_OK;
    auto k = heads_fwd_tc_kernel<F, FROM_Z>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_status(e);
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kHTThreads, smem);
    if (e != cudaSuccess) return cuda_status(e);
    if (occ < 1 || occ * kHTCols > 512) return SPIN4D_ERR_UNSUPPORTED;   // TMEM would be oversubscribed
    configured[dev] = true;
    return SPIN4D_OK;
  }
  static int fwd_tc(const GridParams& gp, const HeadsParams& hp, const float* pos, int64_t N, const void* tables,
                    const void* weights, const HeadsOut& o, cudaStream_t s) {
    const int smem = HeadsTcLayout::BYTES;
    const int blocks = persistent_blocks((N + kHT - 1) / kHT, 2);
    const float4* P = reinterpret_cast<const float4*>(pos);
    const __half* tab = static_cast<const __half*>(tables);
    const __half* wts = static_cast<const __half*>(weights);
    if (!o.z16) {
      SPIN4D_CHECK(configure_tc<false>(smem));
      heads_fwd_tc_kernel<F, false><<<blocks, kHTThreads, smem, s>>>(gp, hp, P, N, tab, wts, o);
      return launch_status();
    }
    SPIN4D_CHECK(configure_tc<true>(smem));
    heads_gather_kernel<F><<<persistent_blocks((N + 127) / 128, 16), 128, 0, s>>>(gp, P, N, tab, o.z16, o.latent);
    SPIN4D_CHECK(launch_status());
    return cuda_status(launch_pdl(heads_fwd_tc_kernel<F, true>, dim3(blocks), dim3(kHTThreads), (size_t)smem, s, gp,
                                  hp, P, N, tab, wts, o));
  }
  static int fwd(const GridParams& gp, const HeadsParams& hp, const float* pos, int64_t N, const void* tables,
                 const void* weights, const HeadsOut& o, cudaStream_t s) {
    if constexpr (std::is_same<T, __half>::value && std::is_same<W, __half>::value && F == 4) {
      // its vector stores want 16-byte rows of sh and raw
      const bool vec = ((uintptr_t)o.sh & 15) == 0 && ((uintptr_t)o.raw & 15) == 0;
      if (hp.in_dim == 64 && hp.hidden == 64 && hp.sh_dim == kHTMaxSh && vec) {
        const int st = fwd_tc(gp, hp, pos, N, tables, weights, o, s);
        if (st != SPIN4D_ERR_UNSUPPORTED) return st;   // else the SIMT forward below
      }
    }
    auto k = heads_fwd_q_kernel<T, F, W>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFwdQSmem);
    if (e != cudaSuccess) return cuda_status(e);
    const int blocks = persistent_blocks((N + kHeadsBwdBlock - 1) / kHeadsBwdBlock, 5);   // 5 fit an SM
    k<<<blocks, kBwdThreads, kFwdQSmem, s>>>(gp, hp, reinterpret_cast<const float4*>(pos), N,
                                             static_cast<const T*>(tables), static_cast<const W*>(weights), o);
    return launch_status();
  }
  // the tensor-core backward (the forward's configuration, given its saved z and raw outputs)
  static int bwd_tc(const GridParams& gp, const HeadsParams& hp, const float* pos, int64_t N, const void* weights,
                    const float* latent, const float* raw, const HeadsGrads& go, float* grad_tables,
                    float* grad_weights, float* ws, int n_params, cudaStream_t s) {
    auto k = heads_bwd_tc_kernel<F>;
    const int smem = HeadsBwdLayout::BYTES;
    static bool configured[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return cuda_status(e);
      int occ = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kHTThreads, smem);
      if (e != cudaSuccess) return cuda_status(e);
      if (occ != 1) return SPIN4D_ERR_UNSUPPORTED;   // one CTA holds all 512 TMEM columns
      configured[dev] = true;
    }
    const int blocks = persistent_blocks((N + kHT - 1) / kHT, 1);
    k<<<blocks, kHTThreads, smem, s>>>(gp, hp, reinterpret_cast<const float4*>(pos), N,
                                      static_cast<const __half*>(weights), latent, raw, go, grad_tables, ws);
    SPIN4D_CHECK(launch_status());
    heads_reduce_slots_tc<<<(n_params + 255) / 256, 256, 0, s>>>(ws, blocks, hp, n_params, grad_weights);
    return launch_status();
  }
  static int bwd(const GridParams& gp, const HeadsParams& hp, const float* pos, int64_t N, const void* tables,
                 const void* weights, const float* latent, const float* raw, const HeadsGrads& go, float* grad_tables,
                 float* grad_weights, float* ws, int n_params, cudaStream_t s) {
    if constexpr (std::is_same<T, __half>::value && std::is_same<W, __half>::value && F == 4) {
      if (hp.in_dim == 64 && hp.hidden == 64 && hp.sh_dim == kHTMaxSh && latent && raw &&
          ((uintptr_t)latent & 15) == 0) {
        const int st = bwd_tc(gp, hp, pos, N, weights, latent, raw, go, grad_tables, grad_weights, ws, n_params, s);
        if (st != SPIN4D_ERR_UNSUPPORTED) return st;   // else the SIMT backward below
      }
    }
    auto k = heads_bwd_kernel<T, F, W>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwdSmem);
    if (e != cudaSuccess) return cuda_status(e);
    const int blocks = bwd_blocks(N);
    k<<<blocks, kBwdThreads, kBwdSmem, s>>>(gp, hp, reinterpret_cast<const float4*>(pos), N,
                                              static_cast<const T*>(tables), static_cast<const W*>(weights), latent, raw,
                                              go, grad_tables, ws, n_params);
    SPIN4D_CHECK(launch_status());
    heads_reduce_slots<<<(n_params + 255) / 256, 256, 0, s>>>(ws, blocks, n_params, grad_weights);
    return launch_status();
  }
};

template <typename T, int F>
int dispatch_w(int wdt, bool bwd, const GridParams& gp, const HeadsParams& hp, const float* pos, int64_t N,
               const void* tables, const void* weights, const HeadsOut* o, const float* latent, const float* raw, const HeadsGrads* go,
               float* gt, float* gw, float* ws, int n_params, cudaStream_t s) {
  if (wdt == SPIN4D_F16) {
    if (bwd) return HeadsLaunch<T, F, __half>::bwd(gp, hp, pos, N, tables, weights, latent, raw, *go, gt, gw, ws, n_params, s);
    return HeadsLaunch<T, F, __half>::fwd(gp, hp, pos, N, tables, weights, *o, s);
  }
  if (bwd) return HeadsLaunch<T, F, float>::bwd(gp, hp, pos, N, tables, weights, latent, raw, *go, gt, gw, ws, n_params, s);
  return HeadsLaunch<T, F, float>::fwd(gp, hp, pos, N, tables, weights, *o, s);
}

template <typename T>
int dispatch_f(int F, int wdt, bool bwd, const GridParams& gp, const HeadsParams& hp, const float* pos, int64_t N,
               const void* tables, const void* weights, const HeadsOut* o, const float* latent, const float* raw, const HeadsGrads* go,
               float* gt, float* gw, float* ws, int n_params, cudaStream_t s) {
  switch (F) {
    case 1: return dispatch_w<T, 1>(wdt, bwd, gp, hp, pos, N, tables, weights, o, latent, raw, go, gt, gw, ws, n_params, s);
    case 2: return dispatch_w<T, 2>(wdt, bwd, gp, hp, pos, N, tables, weights, o, latent, raw, go, gt, gw, ws, n_params, s);
    case 4: return dispatch_w<T, 4>(wdt, bwd, gp, hp, pos, N, tables, weights, o, latent, raw, go, gt, gw, ws, n_params, s);
    case 8: return dispatch_w<T, 8>(wdt, bwd, gp, hp, pos, N, tables, weights, o, latent, raw, go, gt, gw, ws, n_params, s);
    default: return SPIN4D_ERR_UNSUPPORTED;
  }
}

int run(const spin4d_grid_desc* g, const spin4d_heads_desc* h, bool bwd, const float* pos, int64_t N,
        const void* tables, const void* weights, const HeadsOut* o, const float* latent, const float* raw, const HeadsGrads* go,
        float* gt, float* gw, float* ws, cudaStream_t s) {
  const GridParams gp = make_grid_params(g);
  const HeadsParams hp = make_heads(h);
  const int n_params = (int)param_count(h);
  if (g->table_dtype == SPIN4D_F16)
    return dispatch_f<__half>(g->F, h->w_dtype, bwd, gp, hp, pos, N, tables, weights, o, latent, raw, go, gt, gw, ws,
                              n_params, s);
  return dispatch_f<float>(g->F, h->w_dtype, bwd, gp, hp, pos, N, tables, weights, o, latent, raw, go, gt, gw, ws,
                           n_params, s);
}

// The configuration whose forward splits into gather + tensor-core layers
// when given a workspace (otherwise it runs the fused tensor-core kernel).
bool split_forward(const spin4d_grid_desc* g, const spin4d_heads_desc* h) {
  return g->table_dtype == SPIN4D_F16 && h->w_dtype == SPIN4D_F16 && g->F == 4 && h->in_dim == 64 &&
         h->hidden == 64 && h->sh_dim == kHTMaxSh;
}

int check_inputs(const spin4d_grid_desc* g, const spin4d_heads_desc* h, const float* pos, int64_t N,
                 const void* tables, const void* weights) {
  SPIN4D_CHECK(validate_grid(g));
  SPIN4D_CHECK(validate_heads(g, h));
  if (N < 0) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  const size_t esz = g->table_dtype == SPIN4D_F16 ? 2 : 4;
  const size_t talign = esz * g->F > 16 ? 16 : esz * g->F;
  if (!pos || !tables || !weights || !aligned(pos, 16) || !aligned(tables, talign) || !aligned(weights, 4))
    return SPIN4D_ERR_INVALID;
  return SPIN4D_OK;
}

}  // namespace
}  // namespace spin4d

using namespace spin4d;

extern "C" int64_t spin4d_heads_param_count(const spin4d_heads_desc* h) {
  if (!h || h->in_dim < 1 || h->hidden < 1 || h->sh_dim < 1) return -1;
  return param_count(h);
}

extern "C" size_t spin4d_heads_fwd_workspace(const spin4d_grid_desc* g, const spin4d_heads_desc* h, int64_t N) {
  if (validate_grid(g) != SPIN4D_OK || validate_heads(g, h) != SPIN4D_OK || N <= 0) return 0;
  return split_forward(g, h) ? (size_t)N * 64 * sizeof(__half) : 0;
}

extern "C" int spin4d_heads_fwd(const spin4d_grid_desc* g, const spin4d_heads_desc* h, const float* pos, int64_t N,
                                const void* tables, const void* weights, spin4d_heads_outputs out, void* workspace,
                                size_t ws_bytes, spin4d_stream_t stream) {
  SPIN4D_CHECK(check_inputs(g, h, pos, N, tables, weights));
  if (N == 0) return SPIN4D_OK;
  if (!out.scale || !out.rot || !out.sh || !out.opacity || !out.cov || !aligned(out.rot, 16)) return SPIN4D_ERR_INVALID;
  const size_t need = spin4d_heads_fwd_workspace(g, h, N);
  if (workspace && (!aligned(workspace, 256) || ws_bytes < need)) return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_heads_fwd")) return SPIN4D_ERR_INJECTED;
  uint4* z16 = workspace && need ? static_cast<uint4*>(workspace) : nullptr;
  const HeadsOut o{out.scale, out.rot, out.sh, out.opacity, out.cov, out.latent, out.raw, z16};
  return run(g, h, false, pos, N, tables, weights, &o, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
             (cudaStream_t)stream);
}

extern "C" size_t spin4d_heads_bwd_workspace(const spin4d_grid_desc* g, const spin4d_heads_desc* h, int64_t N) {
  if (validate_grid(g) != SPIN4D_OK || validate_heads(g, h) != SPIN4D_OK || N <= 0) return 0;
  const size_t simt = (size_t)bwd_blocks(N) * slot_stride((int)param_count(h)) * sizeof(float);
  // the tensor-core backward: one padded slot per CTA, one CTA per SM
  const size_t tcb = (size_t)persistent_blocks((N + kHT - 1) / kHT, 1) * slot_stride(kHBSlot) * sizeof(float);
  return split_forward(g, h) && tcb > simt ? tcb : simt;
}

extern "C" int spin4d_heads_bwd(const spin4d_grid_desc* g, const spin4d_heads_desc* h, const float* pos, int64_t N,
                                const void* tables, const void* weights, const float* latent, const float* raw,
                                const spin4d_heads_output_grads* grad_out, float* grad_tables, float* grad_weights,
                                void* workspace, size_t ws_bytes, spin4d_stream_t stream) {
  SPIN4D_CHECK(check_inputs(g, h, pos, N, tables, weights));
  if (N == 0) return SPIN4D_OK;
  if (!grad_out || !grad_tables || !grad_weights || !workspace) return SPIN4D_ERR_INVALID;
  if (!aligned(grad_tables, 16) || !aligned(grad_weights, 4) || !aligned(workspace, 256) ||
      ws_bytes < spin4d_heads_bwd_workspace(g, h, N))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_heads_bwd")) return SPIN4D_ERR_INJECTED;
  const HeadsGrads go{grad_out->scale, grad_out->rot, grad_out->sh, grad_out->opacity, grad_out->cov};
  return run(g, h, true, pos, N, tables, weights, nullptr, latent, raw, &go, grad_tables, grad_weights,
             static_cast<float*>(workspace), (cudaStream_t)stream);
}
