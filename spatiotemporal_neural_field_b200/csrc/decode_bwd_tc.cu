// Backward pass of the fused decoder on the sm_100a tensor cores (fp16
// tables and weights, fp32 gradients): the training step's gradient of
// loss = sum_k <g_k, attribute_k> with respect to the hash tables and the
// network weights (SPIN-4DGS section 3.3: tables and decoder are trained
// jointly through Eq. 7-11 and Eq. 2).
//
// Persistent CTAs of 256 threads, tiles of 128 positions (two threads per
// position, as in the forward kernel).  Per tile:
//   A. gather z (fp16 operand tile, x-neighbour pairs share 16-byte loads);
//   B-D. forward trunk and head on the tensor cores (accumulators in TMEM),
//      the trunk inputs z and h1 split into two fp16 terms (hi + lo) so the
//      ReLU masks agree with exact arithmetic; then per position the
//      activations, their adjoint and the upstream gradients give dy;
//   Every fp16 operand tile (z, h1, h2, dy, dpre2, dpre1) is stored scaled by
//   a power of two that puts its largest entry in [2^10, 2^11); epilogues and
//   the weight-gradient readback undo the scales in fp32.
//   E. dh2 = dy . Wh      (tcgen05, K = 16)  -> dpre2 = dh2 * [h2 > 0]
//   G. dh1 = dpre2 . W2   (tcgen05, K = H)   -> dpre1 = dh1 * [h1 > 0]
//   I. dz  = dpre1 . W1   (tcgen05, K = H)   -> scatter-add into the tables
//      with fp32 vector atomics; an x-neighbour pair that shares a 16-byte
//      group of the gradient table is one 16-byte atomic;
//   weight gradients dW = sum_p d_p a_p^T on the tensor core too, issued with
//      the dgrad MMA of the same stage: the K-major-by-feature operand tiles
//      are read as MN-major operands so that K runs over the tile's 128
//      positions (M = 64 accumulators sit in lanes 0-15 of each TMEM
//      quadrant); biases are column sums over positions (SIMT).  Each tile's
//      result is unscaled and added to this CTA's slot of the workspace,
//      which a second kernel adds into grad_weights in slot order.
// The dgrad MMAs use transposed copies of the weights staged as K-major
// tiles.  Every mbarrier wait is bounded (device error word on timeout).
#include "host.h"
#include "tc.cuh"

namespace spin4d {

// Set when a bounded wait of this kernel runs out (read by spin4d_check_device_errors).
__device__ int g_bwd_device_error = 0;

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kHeadN = 16;
constexpr uint32_t kWaitIters = 1u << 24;

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }
__host__ __device__ constexpr uint32_t tmem_cols(int c) {
  return c <= 32 ? 32u : c <= 64 ? 64u : c <= 128 ? 128u : c <= 256 ? 256u : 512u;
}

template <int IN, int H>
struct BLayout {
  static constexpr int w1 = 0;                       // [H][IN]   forward
  static constexpr int w2 = w1 + H * IN * 2;         // [H][H]
  static constexpr int wh = w2 + H * H * 2;          // [16][H]
  static constexpr int w1t = wh + kHeadN * H * 2;    // [IN][H]   transposed, for dz
  static constexpr int w2t = w1t + IN * H * 2;       // [H][H]    for dh1
  static constexpr int wht = w2t + H * H * 2;        // [H][16]   for dh2
  static constexpr int bias = wht + H * kHeadN * 2;  // fp32 b1 | b2 | bh
  static constexpr int zt = align_up(bias + (2 * H + kHeadN) * 4, 128);   // [128][IN]
  static constexpr int h1t = zt + kTile * IN * 2;    // [128][H]
  static constexpr int h2t = h1t + kTile * H * 2;    // [128][H], later dpre1
  static constexpr int dyt = h2t + kTile * H * 2;    // [128][16]
  static constexpr int d2t = dyt + kTile * kHeadN * 2;   // [128][H] dpre2
  static constexpr int scales = d2t + kTile * H * 2;   // fp32 [8]: per-warp maxima
  static constexpr int misc = scales + 64;
  static constexpr int bytes = misc + 16;
};

struct GradIn {
  const float *scale, *rot, *rgb, *opacity, *cov;
};

__device__ __forceinline__ float g_or0(const float* p, int64_t i) { return p ? __ldg(p + i) : 0.0f; }

// Transposed staging: Wt[n][k] = W[k][n] for W [rows][cols] row-major fp16;
// the tile has `n_pad` rows (n >= cols are zero) and K = rows_pad columns
// (k >= rows are zero).
__device__ void stage_transposed(uint8_t* sm, int soff, const __half* __restrict__ w, int rows, int cols,
                                 int n_pad, int k_pad) {
  for (int i = threadIdx.x; i < n_pad * k_pad; i += blockDim.x) {
    const int n = i / k_pad, k = i - n * k_pad;
    __half v = __float2half(0.0f);
    if (n < cols && k < rows) v = w[(size_t)k * cols + n];
    *reinterpret_cast<__half*>(sm + soff + tc::kmaj_off(n, k / 8, k_pad) + (k % 8) * 2) = v;
  }
}

__device__ void stage_plain(uint8_t* sm, int soff, const __half* __restrict__ w, int rows, int rows_pad, int K) {
  const int chunks = K / 8;
  for (int i = threadIdx.x; i < rows_pad * chunks; i += blockDim.x) {
    const int r = i / chunks, kc = i - r * chunks;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows) v = __ldg(reinterpret_cast<const uint4*>(w + (size_t)r * K + kc * 8));
    *reinterpret_cast<uint4*>(sm + soff + tc::kmaj_off(r, kc, K)) = v;
  }
}

__device__ __forceinline__ void unpack8(const uint4& u, float f[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __half2 h = *reinterpret_cast<const __half2*>(&w[q]);
    float2 a = __half22float2(h);
    f[2 * q] = a.x;
    f[2 * q + 1] = a.y;
  }
}

// db[o] += factor * sum_p d[p][o] for a K-major fp16 tile d with Kd columns
// (`rows` real): lanes run over positions, 16-byte chunk reads (conflict-free),
// then a shuffle reduction per output.
__device__ void bias_grad(const uint8_t* sm, int d_off, int Kd, int rows, float factor, float* __restrict__ slotB) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = kThreads / 32;
  for (int ob = warp; ob < Kd / 8; ob += n_warps) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < kTile / 32; ++j) {
      float d[8];
      unpack8(*reinterpret_cast<const uint4*>(sm + d_off + tc::kmaj_off(lane + 32 * j, ob, Kd)), d);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += d[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], m);
    float mine = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) mine = (lane == i) ? acc[i] : mine;
    if (lane < 8 && ob * 8 + lane < rows) slotB[ob * 8 + lane] += mine * factor;
  }
}

// Weight-gradient MMA over the tile's positions: D[m][n] = sum_p A[p][m] B[p][n]
// where A and B are the K-major-by-feature operand tiles (rows = positions,
// Fa / Fb features per row) read as MN-major operands, so K = 128 positions.
__device__ __forceinline__ void mma_wgrad(uint32_t d_tmem, uint32_t a_tile, int Fa, uint32_t b_tile, int Fb, int M,
                                          int N) {
  const uint32_t idesc = tc::idesc_f16_f32(M, N) | (1u << 15) | (1u << 16);   // A and B MN-major
  for (int s = 0; s < kTile / 16; ++s)
    tc::mma_f16(d_tmem, tc::smem_desc(a_tile + s * 32 * Fa, (uint32_t)Fa * 16u, 128),
                tc::smem_desc(b_tile + s * 32 * Fb, (uint32_t)Fb * 16u, 128), idesc, s > 0 ? 1u : 0u);
}

// Reads an M x N weight-gradient accumulator (M = 64: rows in lanes 0-15 of
// each warp quadrant; M = 128: one row per lane) and hands every element to
// fn(row, col, value).  Warps 0-3 take the first half of the columns, 4-7 the
// second; N = 16 is read by warps 0-3 alone.
template <int M, int N, typename Fn>
__device__ __forceinline__ void wgrad_readback(uint32_t tmem, uint32_t col, Fn fn) {
  const int warp = threadIdx.x >> 5, t = threadIdx.x & 31, q = warp & 3, ch = warp >> 2;
  const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
  const int row = M == 128 ? q * 32 + t : q * 16 + t;
  const bool has_row = M == 128 || t < 16;
  if constexpr (N == 16) {
    if (ch == 0) {
      float v[16];
      tc::tmem_ld16(tmem + lane_addr + col, v);
      if (has_row)
#pragma unroll
        for (int i = 0; i < 16; ++i) fn(row, i, v[i]);
    }
  } else if constexpr (N == 32) {
    float v[16];
    tc::tmem_ld16(tmem + lane_addr + col + ch * 16, v);
    if (has_row)
#pragma unroll
      for (int i = 0; i < 16; ++i) fn(row, ch * 16 + i, v[i]);
  } else {
#pragma unroll 1
    for (int c0 = ch * (N / 2); c0 < (ch + 1) * (N / 2); c0 += 32) {
      float v[32];
      tc::tmem_ld32(tmem + lane_addr + col + c0, v);
      if (has_row)
#pragma unroll
        for (int i = 0; i < 32; ++i) fn(row, c0 + i, v[i]);
    }
  }
}

// Power of two that brings a tile's largest magnitude m into [2^10, 2^11):
// every fp16 operand tile is stored scaled by it, so values that would be
// fp16-subnormal (small upstream gradients, tiny early-training activations)
// keep their 11-bit precision; rows down to 2^-24 of the tile maximum stay
// normal.  Exact (a power of two); 1 for m = 0.
__device__ __forceinline__ float pow2_scale(float m) {
  if (!(m > 0.f) || !isfinite(m)) return 1.0f;
  int e;
  frexpf(m, &e);   // m = f * 2^e, f in [0.5, 1)
  return ldexpf(1.0f, max(-100, min(100, 11 - e)));
}

// Scatter of one level's adjoint: grad[idx_c][f] += w_c * dz[f], x-pairs that
// share a 16-byte group of the fp32 gradient table merged into one atomic.
template <int F>
__device__ __forceinline__ void scatter_level_paired(const float xt[4], const GridParams& g, int l,
                                                     float* __restrict__ grad_tables, const float dz[F]) {
  uint32_t base[4];
  float frac[4];
  level_cell(xt, g, l, base, frac);
  uint32_t idx[16];
  level_indices(base, g, l, idx);
  float w[16];
  level_weights(frac, w);
  float* gl = grad_tables + ((size_t)l << g.log2_T) * F;
  if constexpr (F == 2) {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t e0 = idx[2 * p], e1 = idx[2 * p + 1];
      const float w0 = w[2 * p], w1 = w[2 * p + 1];
      if ((e0 >> 1) == (e1 >> 1)) {
        const bool lo0 = (e0 & 1u) == 0;
        const float4 v = lo0 ? make_float4(w0 * dz[0], w0 * dz[1], w1 * dz[0], w1 * dz[1])
                             : make_float4(w1 * dz[0], w1 * dz[1], w0 * dz[0], w0 * dz[1]);
        atomicAdd(reinterpret_cast<float4*>(gl + (size_t)(e0 & ~1u) * 2), v);
      } else {
        atomicAdd(reinterpret_cast<float2*>(gl + (size_t)e0 * 2), make_float2(w0 * dz[0], w0 * dz[1]));
        atomicAdd(reinterpret_cast<float2*>(gl + (size_t)e1 * 2), make_float2(w1 * dz[0], w1 * dz[1]));
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c)
      atomicAdd(reinterpret_cast<float4*>(gl + (size_t)idx[c] * 4),
                make_float4(w[c] * dz[0], w[c] * dz[1], w[c] * dz[2], w[c] * dz[3]));
  }
}

__device__ __forceinline__ void store_row8(uint8_t* sm, int off, int row, int kc, int K, const float v[8]) {
  *reinterpret_cast<uint4*>(sm + off + tc::kmaj_off(row, kc, K)) =
      make_uint4(tc::pack_half2(v[0], v[1]), tc::pack_half2(v[2], v[3]), tc::pack_half2(v[4], v[5]),
                 tc::pack_half2(v[6], v[7]));
}

// D[tmem] (+)= A . B^T over K columns, K/16 instructions of K = 16.
__device__ __forceinline__ void mma_group(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr, int K, int N,
                                          bool accumulate) {
  const uint32_t sbo = (uint32_t)K * 16u;
  for (int s = 0; s < K / 16; ++s)
    tc::mma_f16(d_tmem, tc::smem_desc(a_addr + s * 256, 128, sbo), tc::smem_desc(b_addr + s * 256, 128, sbo),
                tc::idesc_f16_f32(kTile, N), (s > 0 || accumulate) ? 1u : 0u);
}

// One MMA D = A . B^T, completion signalled on `mbar`.
__device__ __forceinline__ void issue_mma(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr, int K, int N,
                                          uint32_t mbar) {
  tc::fence_after_sync();
  mma_group(d_tmem, a_addr, b_addr, K, N, false);
  tc::mma_commit(mbar);
}

// D = (A_hi + A_lo) . B^T: an fp16 operand split into two fp16 terms, so the
// product carries ~22 bits of the activations instead of 11.
__device__ __forceinline__ void issue_mma_split(uint32_t d_tmem, uint32_t a_hi, uint32_t a_lo, uint32_t b_addr, int K,
                                                int N, uint32_t mbar) {
  tc::fence_after_sync();
  mma_group(d_tmem, a_hi, b_addr, K, N, false);
  mma_group(d_tmem, a_lo, b_addr, K, N, true);
  tc::mma_commit(mbar);
}

template <int F, int IN, int H>
__global__ void __launch_bounds__(kThreads, H <= 64 ? 2 : 1) decode_bwd_tc_kernel(
    GridParams g, int gate, float tau, const float4* __restrict__ pos, int64_t N, const __half* __restrict__ tables,
    const __half* __restrict__ weights, const float2* __restrict__ gate_cr, const float* __restrict__ latent, GradIn go,
    float* __restrict__ grad_tables, float* __restrict__ grad_pos, float* __restrict__ grad_gate,
    float* __restrict__ ws, int n_params) {
  using Lay = BLayout<IN, H>;
  // TMEM columns: two per-tile regions of H, then the weight-gradient
  // accumulators dW1 (IN), dW2 (H), dWh^T (16)
  constexpr uint32_t colA = 0, colB = H, cW1 = 2 * H, cW2 = 2 * H + IN, cW3 = 2 * H + IN + H;
  constexpr uint32_t kCols = tmem_cols(2 * H + IN + H + kHeadN);
  static_assert(IN % 16 == 0 && H % 16 == 0 && (F == 2 || F == 4) && IN <= H && (H == 64 || H == 128), "tile shape");
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (kTile - 1), half = tid / kTile;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::misc + 8);
  const uint32_t mbar = tc::smem_u32(sm + Lay::misc);
  float* bias = reinterpret_cast<float*>(sm + Lay::bias);

  // packed weight offsets: W1 | b1 | W2 | b2 | Wh | bh
  const __half* W1 = weights;
  const __half* W2 = W1 + H * IN + H;
  const __half* Wh = W2 + H * H + H;
  const int oW1 = 0, oB1 = H * IN, oW2 = oB1 + H, oB2 = oW2 + H * H, oWh = oB2 + H, oBh = oWh + kHeadRows * H;

  stage_plain(sm, Lay::w1, W1, H, H, IN);
  stage_plain(sm, Lay::w2, W2, H, H, H);
  stage_plain(sm, Lay::wh, Wh, kHeadRows, kHeadN, H);
  stage_transposed(sm, Lay::w1t, W1, H, IN, IN, H);        // [IN][H]
  stage_transposed(sm, Lay::w2t, W2, H, H, H, H);          // [H][H]
  stage_transposed(sm, Lay::wht, Wh, kHeadRows, H, H, kHeadN);   // [H][16]
  for (int o = tid; o < H; o += kThreads) {
    bias[o] = __half2float(W1[H * IN + o]);
    bias[H + o] = __half2float(W2[H * H + o]);
  }
  for (int o = tid; o < kHeadN; o += kThreads) bias[2 * H + o] = o < kHeadRows ? __half2float(Wh[kHeadRows * H + o]) : 0.f;
  float* slot = ws + (size_t)blockIdx.x * slot_stride(n_params);
  for (int p = tid; p < n_params; p += kThreads) slot[p] = 0.0f;
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
  const uint32_t a_zt = tc::smem_u32(sm + Lay::zt), a_h1 = tc::smem_u32(sm + Lay::h1t),
                 a_h2 = tc::smem_u32(sm + Lay::h2t), a_dy = tc::smem_u32(sm + Lay::dyt),
                 a_d2 = tc::smem_u32(sm + Lay::d2t);

  auto wait_mma = [&]() -> bool {
    const bool ok = tc::mbar_wait_bounded(mbar, phase, kWaitIters);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) return false;
    tc::fence_after_sync();
    return true;
  };
  auto handoff = [&]() {   // make this thread's operand writes visible to the next MMA
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
  };

  float* red = reinterpret_cast<float*>(sm + Lay::scales);   // per-warp maxima
  const int lane_id = tid & 31;
  // Largest magnitude over the whole tile (all 256 threads contribute).
  auto tile_max = [&](float m) -> float {
    const unsigned u = __reduce_max_sync(0xffffffffu, __float_as_uint(m));   // m >= 0: bit order = value order
    if (lane_id == 0) red[warp] = __uint_as_float(u);
    __syncthreads();
    float t = red[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) t = fmaxf(t, red[w]);
    return t;
  };
  // Epilogue: this thread's half of the row, fn(column, accumulator) -> value;
  // one scale for the tile; fp16 hi at `dst`, rounding remainder at `dst_lo`.
  auto store_scaled = [&](uint32_t col, int dst, int dst_lo, auto fn) -> float {
    constexpr int HH = H / 2;
    float v[HH];
#pragma unroll
    for (int c0 = 0; c0 < HH; c0 += 32) tc::tmem_ld32(tmem + lane + col + half * HH + c0, v + c0);
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < HH; ++i) {
      v[i] = fn(half * HH + i, v[i]);
      m = fmaxf(m, fabsf(v[i]));
    }
    const float sc = pow2_scale(tile_max(m));
#pragma unroll
    for (int q = 0; q < HH / 8; ++q) {
      float r[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = v[8 * q + i] * sc;
      store_row8(sm, dst, row, half * (HH / 8) + q, H, r);
      if (dst_lo >= 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) r[i] -= __half2float(__float2half_rn(r[i]));
        store_row8(sm, dst_lo, row, half * (HH / 8) + q, H, r);
      }
    }
    return sc;
  };
  // fp16 tile entry of this row at column c (for ReLU masks: sign only)
  auto tile_at = [&](int off, int c) -> float {
    return __half2float(*reinterpret_cast<const __half*>(sm + off + tc::kmaj_off(row, c / 8, H) + (c % 8) * 2));
  };

  for (int64_t tile = blockIdx.x; tile * kTile < N; tile += gridDim.x) {
    const int64_t n = tile * kTile + row;
    const bool valid = n < N;
    float xt[4] = {0.f, 0.f, 0.f, 0.f};
    // ---- A. gather this thread's half of z; one power-of-two scale per tile ----
    if (valid) normalise_position(pos[n], g, xt);
    constexpr int HZ = IN / 2;
    float zv[HZ];
    if (latent) {   // z saved by the forward pass: no second gather
#pragma unroll
      for (int q = 0; q < HZ / 4; ++q) {
        float4 v = valid ? __ldg(reinterpret_cast<const float4*>(latent + n * IN + half * HZ) + q)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        zv[4 * q] = v.x;
        zv[4 * q + 1] = v.y;
        zv[4 * q + 2] = v.z;
        zv[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < HZ / F; ++q) {
        float acc[F];
        if (valid) {
          encode_level_f16_paired<F>(xt, g, half * (HZ / F) + q, tables, acc);
        } else {
#pragma unroll
          for (int f = 0; f < F; ++f) acc[f] = 0.f;
        }
#pragma unroll
        for (int f = 0; f < F; ++f) zv[q * F + f] = acc[f];
      }
    }
    float zm = 0.f;
#pragma unroll
    for (int i = 0; i < HZ; ++i) zm = fmaxf(zm, fabsf(zv[i]));
    const float s_z = pow2_scale(tile_max(zm));
#pragma unroll
    for (int kc = 0; kc < HZ / 8; ++kc) {
      float r[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = zv[8 * kc + i] * s_z;
      store_row8(sm, Lay::zt, row, half * (HZ / 8) + kc, IN, r);
      // remainder of the fp16 rounding, in the (still unused) h2 tile
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] -= __half2float(__float2half_rn(r[i]));
      store_row8(sm, Lay::h2t, row, half * (HZ / 8) + kc, IN, r);
    }
    handoff();
    // ---- B. h1 = relu(z W1^T + b1), z as hi + lo: the ReLU masks must match
    //      those of exact arithmetic, or the gradient of a pre-activation near
    //      zero flips between 0 and its full value ----
    if (tid == 0) issue_mma_split(tmem + colA, a_zt, a_h2, tc::smem_u32(sm + Lay::w1), IN, H, mbar);
    if (!wait_mma()) { failed = true; break; }
    const float iz = 1.0f / s_z;
    const float s_h1 = store_scaled(colA, Lay::h1t, Lay::d2t,
                                    [&](int c, float v) { return fmaxf(fmaf(v, iz, bias[c]), 0.f); });
    handoff();
    // ---- C. h2 = relu(h1 W2^T + b2), h1 as hi + lo ----
    if (tid == 0) issue_mma_split(tmem + colB, a_h1, a_d2, tc::smem_u32(sm + Lay::w2), H, H, mbar);
    if (!wait_mma()) { failed = true; break; }
    const float ih1 = 1.0f / s_h1;
    const float s_h2 = store_scaled(colB, Lay::h2t, -1,
                                    [&](int c, float v) { return fmaxf(fmaf(v, ih1, bias[H + c]), 0.f); });
    handoff();
    // ---- D. head and its adjoint: dy ----
    if (tid == 0) issue_mma(tmem + colA, a_h2, tc::smem_u32(sm + Lay::wh), H, kHeadN, mbar);
    if (!wait_mma()) { failed = true; break; }
    float dy[kHeadN];
#pragma unroll
    for (int i = 0; i < kHeadN; ++i) dy[i] = 0.f;
    if (half == 0) {
      float v[16];
      tc::tmem_ld16(tmem + lane + colA, v);
      if (valid) {
        const float ih2 = 1.0f / s_h2;
        float y[kHeadRows];
#pragma unroll
        for (int i = 0; i < kHeadRows; ++i) y[i] = fmaf(v[i], ih2, bias[2 * H + i]);
        float gw = 1.0f;
        float2 cr = make_float2(0.f, 0.f);
        if (gate) {
          cr = gate_cr[n];
          gw = temporal_gate(xt[3], cr.x, cr.y, tau);
        }
        AttrGrad ag;
#pragma unroll
        for (int i = 0; i < 3; ++i) ag.s[i] = g_or0(go.scale, 3 * n + i);
#pragma unroll
        for (int i = 0; i < 4; ++i) ag.r[i] = g_or0(go.rot, 4 * n + i);
#pragma unroll
        for (int i = 0; i < 3; ++i) ag.rgb[i] = g_or0(go.rgb, 3 * n + i);
        ag.o = g_or0(go.opacity, n);
#pragma unroll
        for (int i = 0; i < 6; ++i) ag.cov[i] = g_or0(go.cov, 6 * n + i);
        heads_backward(y, gw, ag, dy);
        if (grad_gate && gate) {   // o = sigma(o^) w: dloss/dw = g_o sigma(o^)
          float gcr[2];
          temporal_gate_backward(xt[3], cr.x, cr.y, tau, ag.o * sigmoidf_(y[10]), gcr);
          grad_gate[2 * n] += gcr[0];
          grad_gate[2 * n + 1] += gcr[1];
        }
      }
    }
    float dm = 0.f;
#pragma unroll
    for (int i = 0; i < kHeadN; ++i) dm = fmaxf(dm, fabsf(dy[i]));
    const float s_dy = pow2_scale(tile_max(dm));
    if (half == 0) {
#pragma unroll
      for (int i = 0; i < kHeadN; ++i) dy[i] *= s_dy;
      *reinterpret_cast<uint4*>(sm + Lay::dyt + tc::kmaj_off(row, 0, kHeadN)) =
          make_uint4(tc::pack_half2(dy[0], dy[1]), tc::pack_half2(dy[2], dy[3]), tc::pack_half2(dy[4], dy[5]),
                     tc::pack_half2(dy[6], dy[7]));
      *reinterpret_cast<uint4*>(sm + Lay::dyt + tc::kmaj_off(row, 1, kHeadN)) =
          make_uint4(tc::pack_half2(dy[8], dy[9]), tc::pack_half2(dy[10], dy[11]), tc::pack_half2(dy[12], dy[13]),
                     tc::pack_half2(dy[14], dy[15]));
    }
    handoff();
    // ---- E. dpre2 = (dy Wh) * [h2 > 0]; dWh^T = h2^T dy on the tensor core ----
    if (tid == 0) {
      tc::fence_after_sync();
      mma_group(tmem + colB, a_dy, tc::smem_u32(sm + Lay::wht), kHeadN, H, false);
      mma_wgrad(tmem + cW3, a_h2, H, a_dy, kHeadN, H, kHeadN);
      tc::mma_commit(mbar);
    }
    bias_grad(sm, Lay::dyt, kHeadN, kHeadRows, 1.0f / s_dy, slot + oBh);
    if (!wait_mma()) { failed = true; break; }
    {
      const float f3 = 1.0f / (s_h2 * s_dy);
      wgrad_readback<H, kHeadN>(tmem, cW3, [&](int i, int o, float v) {
        if (o < kHeadRows) slot[oWh + o * H + i] += v * f3;
      });
    }
    const float idy = 1.0f / s_dy;
    const float s_d2 = store_scaled(colB, Lay::d2t, -1, [&](int c, float v) { return tile_at(Lay::h2t, c) > 0.f ? v * idy : 0.f; });
    handoff();
    // ---- G. dpre1 = (dpre2 W2) * [h1 > 0] into the h2 tile; dW2 = dpre2^T h1 ----
    if (tid == 0) {
      tc::fence_after_sync();
      mma_group(tmem + colA, a_d2, tc::smem_u32(sm + Lay::w2t), H, H, false);
      mma_wgrad(tmem + cW2, a_d2, H, a_h1, H, H, H);
      tc::mma_commit(mbar);
    }
    bias_grad(sm, Lay::d2t, H, H, 1.0f / s_d2, slot + oB2);
    if (!wait_mma()) { failed = true; break; }
    {
      const float f2 = 1.0f / (s_d2 * s_h1);
      wgrad_readback<H, H>(tmem, cW2, [&](int o, int i, float v) { slot[oW2 + o * H + i] += v * f2; });
    }
    const float id2 = 1.0f / s_d2;
    const float s_d1 = store_scaled(colA, Lay::h2t, -1, [&](int c, float v) { return tile_at(Lay::h1t, c) > 0.f ? v * id2 : 0.f; });
    handoff();
    // ---- I. dz = dpre1 W1 -> scatter; dW1 = dpre1^T z ----
    if (tid == 0) {
      tc::fence_after_sync();
      mma_group(tmem + colB, a_h2, tc::smem_u32(sm + Lay::w1t), H, IN, false);
      mma_wgrad(tmem + cW1, a_h2, H, a_zt, IN, H, IN);
      tc::mma_commit(mbar);
    }
    bias_grad(sm, Lay::h2t, H, H, 1.0f / s_d1, slot + oB1);
    if (!wait_mma()) { failed = true; break; }
    {
      const float f1 = 1.0f / (s_d1 * s_z);
      wgrad_readback<H, IN>(tmem, cW1, [&](int o, int i, float v) { slot[oW1 + o * IN + i] += v * f1; });
    }
    {
      constexpr int HALF_IN = IN / 2;
      float dzv[HALF_IN];
      if constexpr (HALF_IN == 16) {
        tc::tmem_ld16(tmem + lane + colB + half * HALF_IN, dzv);
      } else {
        tc::tmem_ld32(tmem + lane + colB + half * HALF_IN, dzv);
      }
      tc::fence_before_sync();
      const float id1 = 1.0f / s_d1;
      float gx[4] = {0.f, 0.f, 0.f, 0.f};
      if (valid) {
        constexpr int LV = HALF_IN / F;
#pragma unroll 1
        for (int q = 0; q < LV; ++q) {
          float dz[F];
#pragma unroll
          for (int f = 0; f < F; ++f) dz[f] = dzv[q * F + f] * id1;
          scatter_level_paired<F>(xt, g, half * LV + q, grad_tables, dz);
          if (grad_pos) level_position_grad<__half, F>(xt, g, half * LV + q, tables, dz, gx);
        }
      }
      if (grad_pos) {
        // the two halves' level sums meet in the (now free) dy tile; half 0
        // applies Eq. 7's Jacobian and owns the position's output
        float4* part = reinterpret_cast<float4*>(sm + Lay::dyt);
        part[half * kTile + row] = make_float4(gx[0], gx[1], gx[2], gx[3]);
        __syncthreads();
        if (half == 0 && valid) {
          const float4 o = part[kTile + row];
          const float sum[4] = {gx[0] + o.x, gx[1] + o.y, gx[2] + o.z, gx[3] + o.w};
          float gp[3];
          position_grad_chain(pos[n], g, sum, gp);
#pragma unroll
          for (int i = 0; i < 3; ++i) grad_pos[3 * n + i] += gp[i];
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();
  }

  if (failed) {
    if (tid == 0) atomicExch(&g_bwd_device_error, 1);
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
int launch_bwd_tc(const GridParams& gp, const spin4d_mlp_desc* m, const float* pos, int64_t N, const void* tables,
                  const void* weights, const float* gate_cr, const float* latent, const spin4d_output_grads* go,
                  float* grad_tables, float* grad_pos, float* grad_gate, float* ws, int n_params, int blocks,
                  cudaStream_t s) {
  using Lay = BLayout<IN, H>;
  auto k = decode_bwd_tc_kernel<F, IN, H>;
  const int smem = align_up(Lay::bytes, 128);
  static bool configured[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_status(e);
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kThreads, smem);
    if (e != cudaSuccess) return cuda_status(e);
    if (occ < 1 || occ * (int)tmem_cols(3 * H + IN + kHeadN) > 512) return SPIN4D_ERR_UNSUPPORTED;
    configured[dev] = true;
  }
  GradIn gi{go->scale, go->rot, go->rgb, go->opacity, go->cov};
  k<<<blocks, kThreads, smem, s>>>(gp, m->gate, m->tau, reinterpret_cast<const float4*>(pos), N,
                                   static_cast<const __half*>(tables), static_cast<const __half*>(weights),
                                   reinterpret_cast<const float2*>(gate_cr), latent, gi, grad_tables, grad_pos,
                                   grad_gate, ws, n_params);
  return launch_status();
}

}  // namespace

// Synchronous read (and optional reset) of this file's device error word.
int bwd_device_error(int clear) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_bwd_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_status(e);
  if (clear && v) {
    int zero = 0;
    e = cudaMemcpyToSymbol(g_bwd_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_status(e);
  }
  return v ? SPIN4D_ERR_TIMEOUT : SPIN4D_OK;
}

// CTAs per SM of the tensor-core backward for this shape (0 = not handled).
int decode_bwd_tc_ctas_per_sm(const spin4d_grid_desc* g, const spin4d_mlp_desc* m) {
  if (g->table_dtype != SPIN4D_F16 || m->w_dtype != SPIN4D_F16 || m->n_hidden != 2) return 0;
  if (g->F == 2 && m->in_dim == 32 && m->hidden == 64) return 2;
  if (g->F == 4 && m->in_dim == 64 && m->hidden == 128) return 1;
  return 0;
}

int decode_bwd_tc(const spin4d_grid_desc* g, const spin4d_mlp_desc* m, const float* pos, int64_t N,
                  const void* tables, const void* weights, const float* gate_cr, const float* latent,
                  const spin4d_output_grads* go, float* grad_tables, float* grad_pos, float* grad_gate, float* ws,
                  int n_params, int blocks, cudaStream_t s) {
  const GridParams gp = make_grid_params(g);
  if (g->F == 2 && m->in_dim == 32 && m->hidden == 64)
    return launch_bwd_tc<2, 32, 64>(gp, m, pos, N, tables, weights, gate_cr, latent, go, grad_tables, grad_pos,
                                    grad_gate, ws, n_params, blocks, s);
  if (g->F == 4 && m->in_dim == 64 && m->hidden == 128)
    return launch_bwd_tc<4, 64, 128>(gp, m, pos, N, tables, weights, gate_cr, latent, go, grad_tables, grad_pos,
                                     grad_gate, ws, n_params, blocks, s);
  return SPIN4D_ERR_UNSUPPORTED;
}

}  // namespace spin4d
