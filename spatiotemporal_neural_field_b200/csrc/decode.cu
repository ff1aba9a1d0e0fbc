// Fused attribute decoder, SIMT path (SPIN-4DGS section 3.3, Eq. 7-11, and
// section 3.1, Eq. 2): normalise -> 4D hash encode -> ReLU trunk -> 11-row
// head -> activations -> Sigma, and its backward pass.
//
// One thread owns one position.  Layer activations live in shared memory,
// transposed [feature][thread] so that every thread touches its own column
// (conflict-free); weights are read through the read-only path, where all
// threads of a warp read the same address (one broadcast per warp).
//
// Backward: weight gradients are reduced per thread block over its tile of
// positions and accumulated into that block's private slot of the
// workspace; a second kernel sums the slots in a fixed order, so the weight
// gradients do not depend on scheduling.  Table gradients are scattered with
// fp32 vector atomics.
#include "host.h"

namespace spin4d {

constexpr int kFwdBlock = 64;
constexpr int kBwdBlock = 64;

struct MlpParams {
  int in_dim, hidden, n_hidden, gate;
  float tau;
};

struct OutPtrs {
  float *scale, *rot, *rgb, *opacity, *cov, *latent;
};
struct GradPtrs {
  const float *scale, *rot, *rgb, *opacity, *cov;
};

template <typename W>
__device__ __forceinline__ float ldw(const W* __restrict__ w, int i) {
  return to_f32<W>(__ldg(w + i));
}

// out[o] = act(b[o] + sum_k W[o][k] * in[k]) for this thread's column.
template <typename W>
__device__ __forceinline__ void dense_layer(const W* __restrict__ Wp, int n_out, int n_in,
                                            const float* in, float* out, int blk, int col, bool relu) {
  const W* bp = Wp + n_out * n_in;
  for (int o = 0; o < n_out; ++o) {
    float acc = ldw(bp, o);
    const W* wr = Wp + o * n_in;
    for (int k = 0; k < n_in; ++k) acc = fmaf(ldw(wr, k), in[k * blk + col], acc);
    out[o * blk + col] = relu ? fmaxf(acc, 0.0f) : acc;
  }
}

__device__ __forceinline__ void store_attr(const OutPtrs& out, int64_t n, const Attr& a) {
#pragma unroll
  for (int i = 0; i < 3; ++i) out.scale[3 * n + i] = a.s[i];
  reinterpret_cast<float4*>(out.rot)[n] = make_float4(a.r[0], a.r[1], a.r[2], a.r[3]);
#pragma unroll
  for (int i = 0; i < 3; ++i) out.rgb[3 * n + i] = a.rgb[i];
  out.opacity[n] = a.o;
#pragma unroll
  for (int i = 0; i < 6; ++i) out.cov[6 * n + i] = a.cov[i];
}

template <typename T, int F, typename W>
__global__ void __launch_bounds__(kFwdBlock) decode_fwd_simt(GridParams g, MlpParams m,
                                                             const float4* __restrict__ pos, int64_t N,
                                                             const T* __restrict__ tables,
                                                             const W* __restrict__ weights,
                                                             const float2* __restrict__ gate_cr, OutPtrs out) {
  extern __shared__ float smem[];
  const int maxw = max(m.in_dim, m.hidden);
  float* buf0 = smem;
  float* buf1 = smem + maxw * kFwdBlock;
  const int col = threadIdx.x;
  for (int64_t n0 = (int64_t)blockIdx.x * kFwdBlock; n0 < N; n0 += (int64_t)gridDim.x * kFwdBlock) {
    const int64_t n = n0 + col;
    if (n >= N) continue;   // no block-level synchronisation below
    float xt[4];
    normalise_position(pos[n], g, xt);
    for (int l = 0; l < g.L; ++l) {
      float acc[F];
      encode_level<T, F>(xt, g, l, tables, acc);
#pragma unroll
      for (int f = 0; f < F; ++f) buf0[(l * F + f) * kFwdBlock + col] = acc[f];
      if (out.latent) {
#pragma unroll
        for (int f = 0; f < F; ++f) out.latent[n * m.in_dim + l * F + f] = acc[f];
      }
    }
    const W* wp = weights;
    float* cur = buf0;
    float* nxt = buf1;
    int din = m.in_dim;
    for (int j = 0; j < m.n_hidden; ++j) {
      dense_layer<W>(wp, m.hidden, din, cur, nxt, kFwdBlock, col, true);
      wp += m.hidden * din + m.hidden;
      din = m.hidden;
      float* t = cur; cur = nxt; nxt = t;
    }
    float y[kHeadRows];
    for (int o = 0; o < kHeadRows; ++o) {
      float acc = ldw(wp + kHeadRows * din, o);
      for (int k = 0; k < din; ++k) acc = fmaf(ldw(wp + o * din, k), cur[k * kFwdBlock + col], acc);
      y[o] = acc;
    }
    float gate = 1.0f;
    if (m.gate) {
      float2 cr = gate_cr[n];
      gate = temporal_gate(xt[3], cr.x, cr.y, m.tau);
    }
    Attr a;
    heads_forward(y, gate, a);
    store_attr(out, n, a);
  }
}

// ---------------------------------------------------------------------------
// Backward
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ld_or0(const float* p, int64_t i) { return p ? __ldg(p + i) : 0.0f; }

// Adds this block's contribution to dW = sum_t d[o][t] * a[k][t] (and db) of
// one layer into the block's workspace slot.  Every thread owns a fixed set
// of parameter indices, so the slot needs no atomics.
__device__ __forceinline__ void block_weight_grad(const float* d, const float* a, int n_out, int n_in,
                                                  float* slot, int blk) {
  const int nW = n_out * n_in;
  for (int p = threadIdx.x; p < nW + n_out; p += blockDim.x) {
    float s = 0.0f;
    if (p < nW) {
      const int o = p / n_in, k = p - o * n_in;
      const float* dr = d + o * blk;
      const float* ar = a + k * blk;
      for (int t = 0; t < blk; ++t) s = fmaf(dr[t], ar[t], s);
    } else {
      const float* dr = d + (p - nW) * blk;
      for (int t = 0; t < blk; ++t) s += dr[t];
    }
    slot[p] += s;
  }
}

template <typename T, int F, typename W>
__global__ void __launch_bounds__(kBwdBlock) decode_bwd_simt(GridParams g, MlpParams m,
                                                             const float4* __restrict__ pos, int64_t N,
                                                             const T* __restrict__ tables,
                                                             const W* __restrict__ weights,
                                                             const float2* __restrict__ gate_cr,
                                                             const float* __restrict__ latent, GradPtrs go,
                                                             float* __restrict__ grad_tables,
                                                             float* __restrict__ grad_pos,
                                                             float* __restrict__ grad_gate,
                                                             float* __restrict__ ws, int n_params) {
  extern __shared__ float smem[];
  const int H = m.hidden, IN = m.in_dim, NH = m.n_hidden;
  const int maxw = max(IN, H);
  // acts: inputs of every layer (z, h_1 .. h_NH), [feature][thread]
  float* acts = smem;
  float* dA = acts + (IN + NH * H) * kBwdBlock;
  float* dB = dA + maxw * kBwdBlock;
  float* dy_s = dB + maxw * kBwdBlock;
  const int col = threadIdx.x;
  float* slot = ws + (size_t)blockIdx.x * slot_stride(n_params);
  for (int p = threadIdx.x; p < n_params; p += blockDim.x) slot[p] = 0.0f;

  // offsets of each layer's packed parameters
  int woff[6];
  {
    int o = 0, din = IN;
    for (int j = 0; j < NH; ++j) { woff[j] = o; o += H * din + H; din = H; }
    woff[NH] = o;
  }
  const int head_in = H;

  for (int64_t n0 = (int64_t)blockIdx.x * kBwdBlock; n0 < N; n0 += (int64_t)gridDim.x * kBwdBlock) {
    const int64_t n = n0 + col;
    const bool valid = n < N;
    float xt[4] = {0.f, 0.f, 0.f, 0.f};
    float gate = 1.0f;
    // ---- forward, keeping every layer input ----
    if (valid) {
      normalise_position(pos[n], g, xt);
      if (latent) {
        for (int k = 0; k < IN; ++k) acts[k * kBwdBlock + col] = __ldg(latent + n * IN + k);
      } else {
        for (int l = 0; l < g.L; ++l) {
          float acc[F];
          encode_level<T, F>(xt, g, l, tables, acc);
#pragma unroll
          for (int f = 0; f < F; ++f) acts[(l * F + f) * kBwdBlock + col] = acc[f];
        }
      }
      int din = IN;
      float* cur = acts;
      for (int j = 0; j < NH; ++j) {
        float* nxt = acts + (IN + j * H) * kBwdBlock;
        dense_layer<W>(weights + woff[j], H, din, cur, nxt, kBwdBlock, col, true);
        cur = nxt;
        din = H;
      }
      float y[kHeadRows];
      const W* wh = weights + woff[NH];
      for (int o = 0; o < kHeadRows; ++o) {
        float acc = ldw(wh + kHeadRows * head_in, o);
        for (int k = 0; k < head_in; ++k) acc = fmaf(ldw(wh + o * head_in, k), cur[k * kBwdBlock + col], acc);
        y[o] = acc;
      }
      float2 cr = make_float2(0.f, 0.f);
      if (m.gate) {
        cr = gate_cr[n];
        gate = temporal_gate(xt[3], cr.x, cr.y, m.tau);
      }
      AttrGrad ag;
#pragma unroll
      for (int i = 0; i < 3; ++i) ag.s[i] = ld_or0(go.scale, 3 * n + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) ag.r[i] = ld_or0(go.rot, 4 * n + i);
#pragma unroll
      for (int i = 0; i < 3; ++i) ag.rgb[i] = ld_or0(go.rgb, 3 * n + i);
      ag.o = ld_or0(go.opacity, n);
#pragma unroll
      for (int i = 0; i < 6; ++i) ag.cov[i] = ld_or0(go.cov, 6 * n + i);
      float dy[kHeadRows];
      heads_backward(y, gate, ag, dy);
      if (grad_gate && m.gate) {   // o = sigma(o^) w: dloss/dw = g_o sigma(o^)
        float gcr[2];
        temporal_gate_backward(xt[3], cr.x, cr.y, m.tau, ag.o * sigmoidf_(y[10]), gcr);
        grad_gate[2 * n] += gcr[0];
        grad_gate[2 * n + 1] += gcr[1];
      }
#pragma unroll
      for (int o = 0; o < kHeadRows; ++o) dy_s[o * kBwdBlock + col] = dy[o];
    } else {
      for (int k = 0; k < IN + NH * H; ++k) acts[k * kBwdBlock + col] = 0.0f;
      for (int o = 0; o < kHeadRows; ++o) dy_s[o * kBwdBlock + col] = 0.0f;
    }
    __syncthreads();
    // ---- head layer ----
    const float* h_last = acts + (IN + (NH - 1) * H) * kBwdBlock;
    block_weight_grad(dy_s, h_last, kHeadRows, head_in, slot + woff[NH], kBwdBlock);
    {
      const W* wh = weights + woff[NH];
      for (int k = 0; k < head_in; ++k) {
        float s = 0.0f;
        for (int o = 0; o < kHeadRows; ++o) s = fmaf(ldw(wh + o * head_in, k), dy_s[o * kBwdBlock + col], s);
        // through the ReLU that produced h_last
        dA[k * kBwdBlock + col] = h_last[k * kBwdBlock + col] > 0.0f ? s : 0.0f;
      }
    }
    __syncthreads();
    // ---- trunk layers, last to first; dA holds d(pre-activation) of layer j ----
    for (int j = NH - 1; j >= 0; --j) {
      const int din = j == 0 ? IN : H;
      const float* a_in = j == 0 ? acts : acts + (IN + (j - 1) * H) * kBwdBlock;
      block_weight_grad(dA, a_in, H, din, slot + woff[j], kBwdBlock);
      const W* wj = weights + woff[j];
      for (int i = 0; i < din; ++i) {
        float s = 0.0f;
        for (int o = 0; o < H; ++o) s = fmaf(ldw(wj + o * din, i), dA[o * kBwdBlock + col], s);
        if (j > 0) s = a_in[i * kBwdBlock + col] > 0.0f ? s : 0.0f;
        dB[i * kBwdBlock + col] = s;
      }
      __syncthreads();
      float* t = dA; dA = dB; dB = t;
    }
    // ---- scatter dz into the tables; position gradient ----
    if (valid) {
      float gx[4] = {0.f, 0.f, 0.f, 0.f};
      for (int l = 0; l < g.L; ++l) {
        float dz[F];
#pragma unroll
        for (int f = 0; f < F; ++f) dz[f] = dA[(l * F + f) * kBwdBlock + col];
        scatter_level<F>(xt, g, l, grad_tables, dz);
        if (grad_pos) level_position_grad<T, F>(xt, g, l, tables, dz, gx);
      }
      if (grad_pos) {
        float gp[3];
        position_grad_chain(pos[n], g, gx, gp);
#pragma unroll
        for (int i = 0; i < 3; ++i) grad_pos[3 * n + i] += gp[i];
      }
    }
    __syncthreads();
  }
}

// grad_weights[p] += sum over slots, in slot order.
__global__ void reduce_slots(const float* __restrict__ ws, int n_slots, int n_params, float* __restrict__ out) {
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < n_params; p += gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int c = 0; c < n_slots; ++c) s += ws[(size_t)c * slot_stride(n_params) + p];
    out[p] += s;
  }
}

static size_t fwd_smem(const spin4d_mlp_desc* m) {
  int maxw = m->in_dim > m->hidden ? m->in_dim : m->hidden;
  return (size_t)2 * maxw * kFwdBlock * sizeof(float);
}

static size_t bwd_smem(const spin4d_mlp_desc* m) {
  int maxw = m->in_dim > m->hidden ? m->in_dim : m->hidden;
  return ((size_t)(m->in_dim + m->n_hidden * m->hidden) + 2 * maxw + kHeadRows) * kBwdBlock * sizeof(float);
}

static int bwd_blocks(int64_t N) { return persistent_blocks((N + kBwdBlock - 1) / kBwdBlock, 2); }

template <typename T, int F, typename W>
static int launch_fwd(const GridParams& gp, const MlpParams& mp, size_t smem, const float* pos, int64_t N,
                      const void* tables, const void* weights, const float* gate_cr, OutPtrs o,
                      cudaStream_t s) {
  auto k = decode_fwd_simt<T, F, W>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_status(e);
  int blocks = persistent_blocks((N + kFwdBlock - 1) / kFwdBlock, 8);
  k<<<blocks, kFwdBlock, smem, s>>>(gp, mp, reinterpret_cast<const float4*>(pos), N,
                                    static_cast<const T*>(tables), static_cast<const W*>(weights),
                                    reinterpret_cast<const float2*>(gate_cr), o);
  return launch_status();
}

template <typename T, int F, typename W>
static int launch_bwd(const GridParams& gp, const MlpParams& mp, size_t smem, const float* pos, int64_t N,
                      const void* tables, const void* weights, const float* gate_cr, const float* latent, GradPtrs go,
                      float* grad_tables, float* grad_pos, float* grad_gate, float* grad_weights, float* ws,
                      int n_params, cudaStream_t s) {
  auto k = decode_bwd_simt<T, F, W>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_status(e);
  int blocks = bwd_blocks(N);
  k<<<blocks, kBwdBlock, smem, s>>>(gp, mp, reinterpret_cast<const float4*>(pos), N,
                                    static_cast<const T*>(tables), static_cast<const W*>(weights),
                                    reinterpret_cast<const float2*>(gate_cr), latent, go, grad_tables, grad_pos, grad_gate, ws,
                                    n_params);
  SPIN4D_CHECK(launch_status());
  int rb = (n_params + 255) / 256;
  reduce_slots<<<rb, 256, 0, s>>>(ws, blocks, n_params, grad_weights);
  return launch_status();
}

// Dispatch on (table dtype, F, weight dtype).
template <template <typename, int, typename> class Fn, typename... Args>
static int dispatch(int tdt, int F, int wdt, Args&&... args) {
#define SPIN4D_DISPATCH_W(T, FF)                                                  \
  if (wdt == SPIN4D_F16) return Fn<T, FF, __half>::run(std::forward<Args>(args)...); \
  return Fn<T, FF, float>::run(std::forward<Args>(args)...);
#define SPIN4D_DISPATCH_F(T)                      \
  switch (F) {                                    \
    case 1: { SPIN4D_DISPATCH_W(T, 1) }           \
    case 2: { SPIN4D_DISPATCH_W(T, 2) }           \
    case 4: { SPIN4D_DISPATCH_W(T, 4) }           \
    case 8: { SPIN4D_DISPATCH_W(T, 8) }           \
    default: return SPIN4D_ERR_UNSUPPORTED;       \
  }
  if (tdt == SPIN4D_F16) { SPIN4D_DISPATCH_F(__half) }
  SPIN4D_DISPATCH_F(float)
#undef SPIN4D_DISPATCH_F
#undef SPIN4D_DISPATCH_W
}

template <typename T, int F, typename W> struct FwdFn {
  template <typename... A> static int run(A&&... a) { return launch_fwd<T, F, W>(std::forward<A>(a)...); }
};
template <typename T, int F, typename W> struct BwdFn {
  template <typename... A> static int run(A&&... a) { return launch_bwd<T, F, W>(std::forward<A>(a)...); }
};

static int check_common(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos, int64_t N,
                        const void* tables, const void* weights, const float* gate_cr) {
  SPIN4D_CHECK(validate_grid(g));
  SPIN4D_CHECK(validate_mlp(g, m));
  if (N < 0) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  size_t esz = g->table_dtype == SPIN4D_F16 ? 2 : 4;
  size_t talign = esz * g->F > 16 ? 16 : esz * g->F;
  if (!pos || !tables || !weights || !aligned(pos, 16) || !aligned(tables, talign) || !aligned(weights, 16))
    return SPIN4D_ERR_INVALID;
  if (m->gate && (!gate_cr || !aligned(gate_cr, 8))) return SPIN4D_ERR_INVALID;
  return SPIN4D_OK;
}

static MlpParams make_mlp(const spin4d_mlp_desc* m) {
  MlpParams p;
  p.in_dim = m->in_dim;
  p.hidden = m->hidden;
  p.n_hidden = m->n_hidden;
  p.gate = m->gate;
  p.tau = m->tau;
  return p;
}

// Tensor-core fused forward for fp16 tables and weights (decode_tc.cu).
int decode_fwd_tc(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos, int64_t N,
                  const void* tables, const void* weights, const float* gate_cr, const spin4d_outputs& out,
                  cudaStream_t s, bool* handled);
// Tensor-core fused backward (decode_bwd_tc.cu): CTAs per SM, 0 when the shape is not covered.
int decode_bwd_tc_ctas_per_sm(const spin4d_grid_desc* g, const spin4d_mlp_desc* m);
int decode_bwd_tc(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos, int64_t N,
                  const void* tables, const void* weights, const float* gate_cr, const float* latent,
                  const spin4d_output_grads* go, float* grad_tables, float* grad_pos, float* grad_gate, float* ws,
                  int n_params, int blocks, cudaStream_t s);

// Thread blocks (= workspace slots) the backward launches for N positions.
static int bwd_slots(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, int64_t N) {
  const int c = decode_bwd_tc_ctas_per_sm(g, m);
  if (c > 0) return persistent_blocks((N + 127) / 128, c);
  return bwd_blocks(N);
}

}  // namespace spin4d

using namespace spin4d;

extern "C" int spin4d_decode_fwd(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos, int64_t N,
                                 const void* tables, const void* weights, const float* gate_cr,
                                 spin4d_outputs out, spin4d_stream_t stream) {
  SPIN4D_CHECK(check_common(g, m, pos, N, tables, weights, gate_cr));
  if (N == 0) return SPIN4D_OK;
  if (!out.scale || !out.rot || !out.rgb || !out.opacity || !out.cov || !aligned(out.rot, 16) ||
      !aligned(out.scale, 4) || !aligned(out.rgb, 4) || !aligned(out.opacity, 4) || !aligned(out.cov, 4) ||
      (out.latent && !aligned(out.latent, 16)))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_decode_fwd")) return SPIN4D_ERR_INJECTED;
  cudaStream_t s = (cudaStream_t)stream;
  bool handled = false;
  int st = decode_fwd_tc(g, m, pos, N, tables, weights, gate_cr, out, s, &handled);
  if (handled) return st;
  OutPtrs o{out.scale, out.rot, out.rgb, out.opacity, out.cov, out.latent};
  return dispatch<FwdFn>(g->table_dtype, g->F, m->w_dtype, make_grid_params(g), make_mlp(m), fwd_smem(m), pos,
                         N, tables, weights, gate_cr, o, s);
}

extern "C" size_t spin4d_decode_bwd_workspace(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, int64_t N) {
  if (validate_grid(g) != SPIN4D_OK || validate_mlp(g, m) != SPIN4D_OK || N <= 0) return 0;
  return (size_t)bwd_slots(g, m, N) * slot_stride((int)spin4d_mlp_param_count(m)) * sizeof(float);
}

namespace spin4d {

// spin4d_decode_bwd with optional extra gradients (members of `extra` may be NULL).
static int decode_bwd_impl(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos, int64_t N,
                           const void* tables, const void* weights, const float* gate_cr, const float* latent,
                           const spin4d_output_grads* grad_out, float* grad_tables, float* grad_weights,
                           const spin4d_extra_grads& extra, void* workspace, size_t ws_bytes, cudaStream_t s,
                           const char* name) {
  SPIN4D_CHECK(check_common(g, m, pos, N, tables, weights, gate_cr));
  if (N == 0) return SPIN4D_OK;
  if (!grad_out || !grad_tables || !grad_weights || !workspace) return SPIN4D_ERR_INVALID;
  if (!aligned(grad_tables, 16) || !aligned(grad_weights, 4) || !aligned(workspace, 256) ||
      (latent && !aligned(latent, 16)) || (extra.pos && !aligned(extra.pos, 4)) ||
      (extra.gate_cr && !aligned(extra.gate_cr, 4)))
    return SPIN4D_ERR_INVALID;
  if (extra.gate_cr && !m->gate) return SPIN4D_ERR_INVALID;
  if (ws_bytes < spin4d_decode_bwd_workspace(g, m, N)) return SPIN4D_ERR_INVALID;
  if (grad_out->rot && !aligned(grad_out->rot, 4)) return SPIN4D_ERR_INVALID;
  const bool tc = decode_bwd_tc_ctas_per_sm(g, m) > 0;
  if (!tc && bwd_smem(m) > 220 * 1024) return SPIN4D_ERR_UNSUPPORTED;
  if (fault_injected(name)) return SPIN4D_ERR_INJECTED;
  int n_params = (int)spin4d_mlp_param_count(m);
  if (tc) {
    const int blocks = bwd_slots(g, m, N);
    float* ws = static_cast<float*>(workspace);
    SPIN4D_CHECK(decode_bwd_tc(g, m, pos, N, tables, weights, gate_cr, latent, grad_out, grad_tables, extra.pos,
                               extra.gate_cr, ws, n_params, blocks, s));
    reduce_slots<<<(n_params + 255) / 256, 256, 0, s>>>(ws, blocks, n_params, grad_weights);
    return launch_status();
  }
  GradPtrs go{grad_out->scale, grad_out->rot, grad_out->rgb, grad_out->opacity, grad_out->cov};
  return dispatch<BwdFn>(g->table_dtype, g->F, m->w_dtype, make_grid_params(g), make_mlp(m), bwd_smem(m), pos,
                         N, tables, weights, gate_cr, latent, go, grad_tables, extra.pos, extra.gate_cr,
                         grad_weights, static_cast<float*>(workspace), n_params, s);
}

}  // namespace spin4d

extern "C" int spin4d_decode_bwd(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos, int64_t N,
                                 const void* tables, const void* weights, const float* gate_cr, const float* latent,
                                 const spin4d_output_grads* grad_out, float* grad_tables, float* grad_weights,
                                 void* workspace, size_t ws_bytes, spin4d_stream_t stream) {
  return decode_bwd_impl(g, m, pos, N, tables, weights, gate_cr, latent, grad_out, grad_tables, grad_weights,
                         spin4d_extra_grads{nullptr, nullptr}, workspace, ws_bytes, (cudaStream_t)stream,
                         "spin4d_decode_bwd");
}

extern "C" int spin4d_decode_bwd_ext(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos,
                                     int64_t N, const void* tables, const void* weights, const float* gate_cr,
                                     const float* latent, const spin4d_output_grads* grad_out, float* grad_tables,
                                     float* grad_weights, const spin4d_extra_grads* extra, void* workspace,
                                     size_t ws_bytes, spin4d_stream_t stream) {
  if (!extra) return SPIN4D_ERR_INVALID;
  return decode_bwd_impl(g, m, pos, N, tables, weights, gate_cr, latent, grad_out, grad_tables, grad_weights,
                         *extra, workspace, ws_bytes, (cudaStream_t)stream, "spin4d_decode_bwd_ext");
}

// ---------------------------------------------------------------------------
// Backward pass for callers that cannot allocate device memory.
//
// Some hosts own every byte of device memory themselves: a renderer or game
// engine that hands a plugin only the buffers it passes in, or a real-time
// loop that forbids cudaMalloc once it is running.  Such a caller cannot
// provide the workspace spin4d_decode_bwd asks for, so this entry point uses
// a fixed scratch array compiled into the library instead.  The array lives
// in every GPU that loads the library, for the life of the process.
// ---------------------------------------------------------------------------
#include <mutex>

namespace spin4d {

// The one definition of the size is the header's, so the documented limit is
// the enforced one.
constexpr size_t kStaticScratchBytes = (size_t)SPIN4D_NOALLOC_SCRATCH_BYTES;   // 16 MiB
static_assert(kStaticScratchBytes % 256 == 0, "scratch size must keep 256-byte slots aligned");
static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / sizeof(float)];

// Device address of g_static_scratch on the current device, looked up once
// per device (cudaGetSymbolAddress with that device current).
static int static_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= 64) return SPIN4D_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    addr[dev] = p;
  }
  *out = addr[dev];
  return SPIN4D_OK;
}

}  // namespace spin4d

extern "C" size_t spin4d_decode_bwd_noalloc_scratch_bytes(void) { return spin4d::kStaticScratchBytes; }

extern "C" int spin4d_decode_bwd_noalloc(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos,
                                         int64_t N, const void* tables, const void* weights, const float* gate_cr,
                                         const float* latent, const spin4d_output_grads* grad_out,
                                         float* grad_tables, float* grad_weights, spin4d_stream_t stream) {
  SPIN4D_CHECK(validate_grid(g));
  SPIN4D_CHECK(validate_mlp(g, m));
  if (N < 0) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  // The scratch needed grows with the weight count and (up to a cap) with N.
  if (spin4d_decode_bwd_workspace(g, m, N) > kStaticScratchBytes) return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_decode_bwd_noalloc")) return SPIN4D_ERR_INJECTED;
  void* scratch = nullptr;
  SPIN4D_CHECK(static_scratch_address(&scratch));
  // Every slot the kernels read is first written by the same call, so the
  // scratch needs no clearing between calls.
  return spin4d_decode_bwd(g, m, pos, N, tables, weights, gate_cr, latent, grad_out, grad_tables, grad_weights,
                           scratch, kStaticScratchBytes, stream);
}
