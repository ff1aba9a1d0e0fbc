// Fused attribute decoder on the sm_100a tensor cores, fp16 tables and
// weights with fp32 accumulation (SPIN-4DGS section 3.3, Eq. 7-11, and
// section 3.1, Eq. 2).
//
// Persistent CTAs of 256 threads; each pass handles a tile of 128 positions,
// two threads per position (each takes half of the levels):
//   1. gather: normalise the position, interpolate its levels (16 corners
//      each, x-neighbour corners paired into one 16-byte load when they share
//      a group, fp32 accumulation), round the latent z to fp16 and store it in
//      the position's row of a K-major operand tile in shared memory;
//   2. trunk: one elected thread issues tcgen05.mma (M=128, N=hidden, K=16
//      per instruction) with the weights, staged once per CTA as K-major fp16
//      tiles, as the B operand; the fp32 accumulator lives in tensor memory;
//   3. epilogue: each warp reads its 32 TMEM lanes (= its 32 positions) with
//      tcgen05.ld -- warps 0-3 the first half of the columns, warps 4-7 the
//      second -- adds the bias, applies ReLU and writes the next layer's fp16
//      operand tile;
//   4. head: an N=16 MMA (11 real rows, 5 zero rows), then per thread the
//      activations, the optional temporal gate and Sigma, written to HBM.
// Several CTAs share an SM (TMEM: 2*hidden columns each), so one CTA's
// gathers overlap another's matrix work.  Every mbarrier wait is bounded; a
// wait that runs out sets a device error word (spin4d_check_device_errors)
// and the CTA releases its tensor memory and exits.
#include "host.h"
#include "tc.cuh"

namespace spin4d {

__device__ int g_device_error = 0;

namespace {

constexpr int kTile = 128;      // positions per pass (= MMA M = TMEM lanes)
constexpr int kThreads = 256;   // two threads per position
constexpr int kHeadN = 16;
#ifndef SPIN4D_TC_PAIRED_GATHER
#define SPIN4D_TC_PAIRED_GATHER 1
#endif
constexpr uint32_t kWaitIters = 1u << 24;
constexpr int kSmemPerSM = 233472;   // 228 KiB of shared memory per SM

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }
__host__ __device__ constexpr uint32_t tmem_cols(int c) { return c <= 32 ? 32u : c <= 64 ? 64u : c <= 128 ? 128u : c <= 256 ? 256u : 512u; }

template <int IN, int H>
struct Layout {
  static constexpr int w1 = 0;                                   // [H][IN] fp16, K-major
  static constexpr int w2 = w1 + H * IN * 2;                     // [H][H]
  static constexpr int wh = w2 + H * H * 2;                      // [16][H]
  static constexpr int bias = wh + kHeadN * H * 2;               // fp32: layer 1, layer 2, head
  static constexpr int zt = align_up(bias + (2 * H + kHeadN) * 4, 128);   // [128][IN] fp16
  static constexpr int ht = zt + kTile * IN * 2;                 // [128][H] fp16
  static constexpr int misc = ht + kTile * H * 2;                // mbarrier, TMEM address
  static constexpr int bytes = misc + 16;
};

struct TcOut {
  float *scale, *rot, *rgb, *opacity, *cov, *latent;
};

// W[rows][K] (fp16, row-major, global) -> K-major tile with `rows_pad` rows.
__device__ __forceinline__ void stage_weights(uint8_t* sm, int soff, const __half* __restrict__ w, int rows,
                                              int rows_pad, int K) {
  const int chunks = K / 8;
  for (int i = threadIdx.x; i < rows_pad * chunks; i += blockDim.x) {
    const int r = i / chunks, kc = i - r * chunks;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows) v = __ldg(reinterpret_cast<const uint4*>(w + (size_t)r * K + kc * 8));
    *reinterpret_cast<uint4*>(sm + soff + tc::kmaj_off(r, kc, K)) = v;
  }
}

template <int F, int IN, int H>
__global__ void __launch_bounds__(kThreads, 512 / tmem_cols(2 * H)) decode_fwd_tc_kernel(GridParams g, int n_hidden, int gate, float tau,
                                                              const float4* __restrict__ pos, int64_t N,
                                                              const __half* __restrict__ tables,
                                                              const __half* __restrict__ weights,
                                                              const float2* __restrict__ gate_cr, TcOut out) {
  using Lay = Layout<IN, H>;
  constexpr uint32_t kCols = tmem_cols(2 * H);
  static_assert(IN % 16 == 0 && H % 16 == 0 && (8 % F == 0), "tile shape");
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int row = tid & (kTile - 1);   // position in the tile = TMEM lane
  const int half = tid / kTile;        // which half of the levels / columns
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::misc + 8);
  const uint32_t mbar = tc::smem_u32(sm + Lay::misc);
  float* bias = reinterpret_cast<float*>(sm + Lay::bias);

  // ---- weights and biases, once per CTA ----
  {
    const __half* w = weights;
    int din = IN;
    for (int j = 0; j < n_hidden; ++j) {
      stage_weights(sm, j == 0 ? Lay::w1 : Lay::w2, w, H, H, din);
      for (int o = tid; o < H; o += kThreads) bias[j * H + o] = __half2float(w[H * din + o]);
      w += H * din + H;
      din = H;
    }
    stage_weights(sm, Lay::wh, w, kHeadRows, kHeadN, H);
    for (int o = tid; o < kHeadN; o += kThreads) bias[2 * H + o] = o < kHeadRows ? __half2float(w[kHeadRows * H + o]) : 0.f;
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), kCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(mbar, 1);
    tc::mbar_fence_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
  uint32_t phase = 0;
  bool failed = false;

  const uint32_t zt = tc::smem_u32(sm + Lay::zt);
  const uint32_t ht = tc::smem_u32(sm + Lay::ht);

  for (int64_t tile = blockIdx.x; tile * kTile < N; tile += gridDim.x) {
    const int64_t n = tile * kTile + row;
    const bool valid = n < N;
    float xt[4] = {0.f, 0.f, 0.f, 0.f};
    // ---- 1. gather: this thread's half of z (fp16) into row `row` ----
    if (valid) normalise_position(pos[n], g, xt);
#pragma unroll 1
    for (int kc = half * (IN / 16); kc < (half + 1) * (IN / 16); ++kc) {
      float zv[8];
#pragma unroll
      for (int q = 0; q < 8 / F; ++q) {
        float acc[F];
        if (valid) {
#if SPIN4D_TC_PAIRED_GATHER
          encode_level_f16_paired<F>(xt, g, kc * (8 / F) + q, tables, acc);
#else
          encode_level<__half, F>(xt, g, kc * (8 / F) + q, tables, acc);
#endif
        } else {
#pragma unroll
          for (int f = 0; f < F; ++f) acc[f] = 0.f;
        }
#pragma unroll
        for (int f = 0; f < F; ++f) zv[q * F + f] = acc[f];
      }
      if (out.latent && valid) {   // z saved for the backward pass
        float4* zl = reinterpret_cast<float4*>(out.latent + n * IN + kc * 8);
        zl[0] = make_float4(zv[0], zv[1], zv[2], zv[3]);
        zl[1] = make_float4(zv[4], zv[5], zv[6], zv[7]);
      }
      *reinterpret_cast<uint4*>(sm + Lay::zt + tc::kmaj_off(row, kc, IN)) =
          make_uint4(tc::pack_half2(zv[0], zv[1]), tc::pack_half2(zv[2], zv[3]), tc::pack_half2(zv[4], zv[5]),
                     tc::pack_half2(zv[6], zv[7]));
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();

    // ---- 2./3. trunk ----
    uint32_t a_tile = zt;
    int din = IN;
    for (int j = 0; j < n_hidden; ++j) {
      const uint32_t dcol = (j & 1) ? (uint32_t)H : 0u;
      if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t b_tile = tc::smem_u32(sm + (j == 0 ? Lay::w1 : Lay::w2));
        const uint32_t sbo = (uint32_t)din * 16u;
        for (int s = 0; s < din / 16; ++s)
          tc::mma_f16(tmem + dcol, tc::smem_desc(a_tile + s * 256, 128, sbo), tc::smem_desc(b_tile + s * 256, 128, sbo),
                      tc::idesc_f16_f32(kTile, H), s > 0 ? 1u : 0u);
        tc::mma_commit(mbar);
      }
      const bool ok = tc::mbar_wait_bounded(mbar, phase, kWaitIters);
      phase ^= 1u;
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      tc::fence_after_sync();
      const float* b = bias + j * H;
#pragma unroll 1
      for (int c0 = half * (H / 2); c0 < (half + 1) * (H / 2); c0 += 32) {
        float v[32];
        tc::tmem_ld32(tmem + lane + dcol + c0, v);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = tc::pack_half2(fmaxf(v[2 * i] + b[c0 + 2 * i], 0.f), fmaxf(v[2 * i + 1] + b[c0 + 2 * i + 1], 0.f));
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(sm + Lay::ht + tc::kmaj_off(row, c0 / 8 + q, H)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      __syncthreads();
      a_tile = ht;
      din = H;
    }
    if (failed) break;

    // ---- 4. head: 16 output columns (11 used) ----
    const uint32_t hcol = (n_hidden & 1) ? (uint32_t)H : 0u;
    if (tid == 0) {
      tc::fence_after_sync();
      const uint32_t wh = tc::smem_u32(sm + Lay::wh);
      const uint32_t sbo = (uint32_t)H * 16u;
      for (int s = 0; s < H / 16; ++s)
        tc::mma_f16(tmem + hcol, tc::smem_desc(ht + s * 256, 128, sbo), tc::smem_desc(wh + s * 256, 128, sbo),
                    tc::idesc_f16_f32(kTile, kHeadN), s > 0 ? 1u : 0u);
      tc::mma_commit(mbar);
    }
    const bool ok = tc::mbar_wait_bounded(mbar, phase, kWaitIters);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    if (half == 0) {
      float v[16];
      tc::tmem_ld16(tmem + lane + hcol, v);
      tc::fence_before_sync();
      if (valid) {
      float y[kHeadRows];
#pragma unroll
      for (int i = 0; i < kHeadRows; ++i) y[i] = v[i] + bias[2 * H + i];
      float gw = 1.0f;
      if (gate) {
        const float2 cr = gate_cr[n];
        gw = temporal_gate(xt[3], cr.x, cr.y, tau);
      }
      Attr a;
      heads_forward(y, gw, a);
#pragma unroll
      for (int i = 0; i < 3; ++i) out.scale[3 * n + i] = a.s[i];
      reinterpret_cast<float4*>(out.rot)[n] = make_float4(a.r[0], a.r[1], a.r[2], a.r[3]);
#pragma unroll
      for (int i = 0; i < 3; ++i) out.rgb[3 * n + i] = a.rgb[i];
      out.opacity[n] = a.o;
#pragma unroll
      for (int i = 0; i < 6; ++i) out.cov[6 * n + i] = a.cov[i];
      }
    }
  }

  // ---- teardown: nothing of ours may still be writing TMEM when it is freed ----
  if (failed) {
    if (tid == 0) atomicExch(&g_device_error, 1);
    tc::mbar_wait_bounded(mbar, phase ^ 1u, kWaitIters);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kCols);
  }
}

template <int F, int IN, int H>
int launch_tc(const GridParams& gp, const spin4d_mlp_desc* m, const float* pos, int64_t N, const void* tables,
              const void* weights, const float* gate_cr, const spin4d_outputs& o, cudaStream_t s) {
  using Lay = Layout<IN, H>;
  constexpr int ctas = (int)(512u / tmem_cols(2 * H));
  auto k = decode_fwd_tc_kernel<F, IN, H>;
  // Shared memory large enough that no more CTAs than TMEM can host share an SM.
  int smem = align_up(Lay::bytes, 128);
  const int floor_bytes = kSmemPerSM / (ctas + 1) - 1024 + 128;
  if (smem < floor_bytes) smem = align_up(floor_bytes, 128);
  static bool configured[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_status(e);
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kThreads, smem);
    if (e != cudaSuccess) return cuda_status(e);
    if (occ > ctas || occ < 1) return SPIN4D_ERR_UNSUPPORTED;   // TMEM would be oversubscribed
    configured[dev] = true;
  }
  const int64_t tiles = (N + kTile - 1) / kTile;
  const int blocks = persistent_blocks(tiles, ctas);
  TcOut out{o.scale, o.rot, o.rgb, o.opacity, o.cov, o.latent};
  k<<<blocks, kThreads, smem, s>>>(gp, m->n_hidden, m->gate, m->tau, reinterpret_cast<const float4*>(pos), N,
                                static_cast<const __half*>(tables), static_cast<const __half*>(weights),
                                reinterpret_cast<const float2*>(gate_cr), out);
  return launch_status();
}

}  // namespace

int decode_fwd_tc(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos, int64_t N,
                  const void* tables, const void* weights, const float* gate_cr, const spin4d_outputs& out,
                  cudaStream_t s, bool* handled) {
  *handled = false;
  if (g->table_dtype != SPIN4D_F16 || m->w_dtype != SPIN4D_F16 || m->n_hidden > 2) return SPIN4D_OK;
  const GridParams gp = make_grid_params(g);
  if (g->F == 2 && m->in_dim == 32 && m->hidden == 64) {
    *handled = true;
    return launch_tc<2, 32, 64>(gp, m, pos, N, tables, weights, gate_cr, out, s);
  }
  if (g->F == 4 && m->in_dim == 64 && m->hidden == 128) {
    *handled = true;
    return launch_tc<4, 64, 128>(gp, m, pos, N, tables, weights, gate_cr, out, s);
  }
  return SPIN4D_OK;
}

int bwd_device_error(int clear);     // decode_bwd_tc.cu
int hex_device_error(int clear);     // hexplane.cu
int heads_device_error(int clear);   // decode_heads.cu
int bounds_status(int clear);        // api.cu (checked build: SPIN4D_ERR_BOUNDS)

}  // namespace spin4d

extern "C" int spin4d_check_device_errors(int clear) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, spin4d::g_device_error, sizeof(int));
  if (e != cudaSuccess) return spin4d::cuda_status(e);
  if (clear && v) {
    int zero = 0;
    e = cudaMemcpyToSymbol(spin4d::g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return spin4d::cuda_status(e);
  }
  const int b = spin4d::bwd_device_error(clear);
  const int h = spin4d::hex_device_error(clear);
  const int p = spin4d::heads_device_error(clear);
  const int c = spin4d::bounds_status(clear);
  if (c != SPIN4D_OK) return c;
  if (b != SPIN4D_OK) return b;
  if (h != SPIN4D_OK) return h;
  if (p != SPIN4D_OK) return p;
  return v ? SPIN4D_ERR_TIMEOUT : SPIN4D_OK;
}
