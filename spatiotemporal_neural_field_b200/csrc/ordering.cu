// Z-order (Morton) ordering of the Gaussians, for gather locality.
//
// The KineticGS notes ("overall kinetic synchronisation") serialise particle
// coordinates onto a Z-order space-filling curve because it keeps spatial
// neighbours close in 1D.  Ordering the Gaussians along that curve makes the
// 128 positions of one decoder tile neighbours in space, so their hash-table
// corners overlap and hit in L1/L2 instead of each costing a random sector.
//
// Keys: the decoder's own normalised coordinates (Eq. 7, same fp32 code),
// 10 bits per spatial axis, q = min(floor(mu_bar * 1024), 1023), bits
// interleaved x0 y0 z0 x1 ... (x lowest): a 30-bit code.  Time is left out
// (every Gaussian is decoded at every frame).
//
// Sort: least-significant-digit radix sort, 8-bit digits, four passes, each
// a histogram kernel, an exclusive scan of the (digit, block) counts and a
// scatter kernel that ranks each block's keys stably (warp match on the
// digit, then a prefix over the warps), so equal keys keep their input
// order and the permutation is deterministic.
#include "host.h"

namespace spin4d {
namespace {

constexpr int kSortThreads = 256;
constexpr int kSortPerThread = 8;
constexpr int kSortTile = kSortThreads * kSortPerThread;   // keys per block
constexpr int kDigits = 256;
constexpr int kScanThreads = 1024;
constexpr int kScanPerThread = 8;
constexpr int kScanChunk = kScanThreads * kScanPerThread;

// Spreads the low 10 bits of v so that bit b lands on bit 3b.
__device__ __forceinline__ uint32_t spread3(uint32_t v) {
  v &= 0x3FFu;
  v = (v | (v << 16)) & 0x030000FFu;
  v = (v | (v << 8)) & 0x0300F00Fu;
  v = (v | (v << 4)) & 0x030C30C3u;
  v = (v | (v << 2)) & 0x09249249u;
  return v;
}

__global__ void morton_keys_kernel(GridParams g, const float4* __restrict__ pos, int64_t N, uint32_t* __restrict__ keys) {
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N; n += (int64_t)gridDim.x * blockDim.x) {
    float xt[4];
    normalise_position(pos[n], g, xt);
    uint32_t q[3];
#pragma unroll
    for (int d = 0; d < 3; ++d) q[d] = min((uint32_t)floorf(__fmul_rn(xt[d], 1024.0f)), 1023u);
    keys[n] = spread3(q[0]) | (spread3(q[1]) << 1) | (spread3(q[2]) << 2);
  }
}

// counts[d * B + b] = keys of block b whose digit is d.
__global__ void __launch_bounds__(kSortThreads) radix_histogram(const uint32_t* __restrict__ keys, int64_t N, int shift,
                                                                uint32_t* __restrict__ counts) {
  __shared__ uint32_t h[kDigits];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int64_t t0 = (int64_t)blockIdx.x * kSortTile;
#pragma unroll
  for (int r = 0; r < kSortPerThread; ++r) {
    const int64_t i = t0 + r * kSortThreads + threadIdx.x;
    if (i < N) atomicAdd(&h[(keys[i] >> shift) & 0xFFu], 1u);
  }
  __syncthreads();
  counts[(size_t)threadIdx.x * gridDim.x + blockIdx.x] = h[threadIdx.x];
}

// Block-wide exclusive scan of one value per thread (kScanThreads threads).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* s_warp, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  total = s_warp[31];
  const uint32_t before = warp ? s_warp[warp - 1] : 0u;
  __syncthreads();
  return before + x - v;
}

// Scan step 1: partial[c] = sum of chunk c of a.
__global__ void __launch_bounds__(kScanThreads) scan_reduce(const uint32_t* __restrict__ a, int64_t n,
                                                            uint32_t* __restrict__ partial) {
  __shared__ uint32_t s_warp[32];
  const int64_t c0 = (int64_t)blockIdx.x * kScanChunk + (int64_t)threadIdx.x * kScanPerThread;
  uint32_t s = 0;
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k)
    if (c0 + k < n) s += a[c0 + k];
  uint32_t total;
  block_exclusive_scan(s, s_warp, total);
  if (threadIdx.x == 0) partial[blockIdx.x] = total;
}

// Scan step 2 (one block): partial[] -> its exclusive scan, in place.
__global__ void __launch_bounds__(kScanThreads) scan_partials(uint32_t* __restrict__ partial, int n) {
  __shared__ uint32_t s_warp[32];
  uint32_t carry = 0;
  for (int base = 0; base < n; base += kScanThreads) {
    const int i = base + threadIdx.x;
    const uint32_t v = i < n ? partial[i] : 0u;
    uint32_t total;
    const uint32_t ex = block_exclusive_scan(v, s_warp, total);
    if (i < n) partial[i] = carry + ex;
    carry += total;
  }
}

// Scan step 3: out = exclusive scan of a, chunk c starting at partial[c].
__global__ void __launch_bounds__(kScanThreads) scan_apply(const uint32_t* __restrict__ a, int64_t n,
                                                           const uint32_t* __restrict__ partial,
                                                           uint32_t* __restrict__ out) {
  __shared__ uint32_t s_warp[32];
  const int64_t c0 = (int64_t)blockIdx.x * kScanChunk + (int64_t)threadIdx.x * kScanPerThread;
  uint32_t v[kScanPerThread];
  uint32_t s = 0;
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) {
    v[k] = c0 + k < n ? a[c0 + k] : 0u;
    s += v[k];
  }
  uint32_t total;
  uint32_t run = partial[blockIdx.x] + block_exclusive_scan(s, s_warp, total);
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) {
    if (c0 + k < n) out[c0 + k] = run;
    run += v[k];
  }
}

// Stable scatter of one block's keys (and values) by digit: the rank of a key
// among the block's keys of its digit counts the earlier rounds, the earlier
// warps of its round and the earlier lanes of its warp.  vals_in == NULL
// means the values are the input indices.
__global__ void __launch_bounds__(kSortThreads) radix_scatter(const uint32_t* __restrict__ keys_in,
                                                              const uint32_t* __restrict__ vals_in, int64_t N,
                                                              int shift, const uint32_t* __restrict__ offsets,
                                                              uint32_t* __restrict__ keys_out,
                                                              uint32_t* __restrict__ vals_out) {
  constexpr int kWarps = kSortThreads / 32;
  __shared__ uint32_t base[kDigits];          // global position of this block's first key of each digit
  __shared__ uint32_t wcnt[kWarps][kDigits];  // per round: keys per (warp, digit), then their prefix
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  base[tid] = offsets[(size_t)tid * gridDim.x + blockIdx.x];
  const uint32_t lt = (1u << lane) - 1u;
  const int64_t t0 = (int64_t)blockIdx.x * kSortTile;
  for (int r = 0; r < kSortPerThread; ++r) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wcnt[w][tid] = 0u;
    __syncthreads();
    const int64_t i = t0 + r * kSortThreads + tid;
    const bool valid = i < N;
    uint32_t key = 0, val = 0, d = 0;
    if (valid) {
      key = keys_in[i];
      val = vals_in ? vals_in[i] : (uint32_t)i;
      d = (key >> shift) & 0xFFu;
    }
    // lanes holding no key form singleton groups of their own
    const uint32_t mask = __match_any_sync(0xffffffffu, valid ? d : 0x100u + (uint32_t)lane);
    const uint32_t lane_rank = __popc(mask & lt);
    if (valid && lane_rank == 0) wcnt[warp][d] = __popc(mask);
    __syncthreads();
    {
      // digit tid: prefix over the warps, then advance the block's base
      uint32_t acc = base[tid];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const uint32_t c = wcnt[w][tid];
        wcnt[w][tid] = acc;
        acc += c;
      }
      base[tid] = acc;
    }
    __syncthreads();
    if (valid) {
      const uint32_t at = wcnt[warp][d] + lane_rank;
      keys_out[at] = key;
      vals_out[at] = val;
    }
    __syncthreads();
  }
}

// dst row i = src row perm[i]; rows of `words` 4-byte words (VEC4: read as
// 16-byte vectors).  A row whose perm entry is not below src_rows is left
// unwritten.
template <bool VEC4>
__global__ void permute_rows_kernel(const uint32_t* __restrict__ src, int64_t src_rows, uint32_t* __restrict__ dst,
                                    const uint32_t* __restrict__ perm, int64_t N, int64_t words) {
  const int64_t total = N * (VEC4 ? words / 4 : words);
  const int64_t per_row = VEC4 ? words / 4 : words;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / per_row, k = e - i * per_row;
    const int64_t s = perm[i];
    if (s >= src_rows) continue;
    if constexpr (VEC4)
      reinterpret_cast<uint4*>(dst)[e] = __ldg(reinterpret_cast<const uint4*>(src) + s * per_row + k);
    else
      dst[e] = __ldg(src + s * per_row + k);
  }
}

int64_t sort_blocks(int64_t N) { return (N + kSortTile - 1) / kSortTile; }
int64_t scan_len(int64_t N) { return sort_blocks(N) * kDigits; }
int64_t scan_chunks(int64_t N) { return (scan_len(N) + kScanChunk - 1) / kScanChunk; }

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace spin4d

using namespace spin4d;

// Workspace: keys' and values' second buffers, the (digit, block) counts and
// their scan, the scan's chunk partials.
extern "C" size_t spin4d_morton_order_workspace(int64_t N) {
  if (N <= 0 || N > SPIN4D_MAX_SORT) return 0;
  return 2 * align256((size_t)N * 4) + 2 * align256((size_t)scan_len(N) * 4) + align256((size_t)scan_chunks(N) * 4);
}

extern "C" int spin4d_morton_order(const spin4d_grid_desc* g, const float* pos, int64_t N, uint32_t* keys,
                                   uint32_t* perm, void* workspace, size_t ws_bytes, spin4d_stream_t stream) {
  SPIN4D_CHECK(validate_grid(g));
  if (N < 0 || N > SPIN4D_MAX_SORT) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  if (!pos || !keys || !perm || !workspace || !aligned(pos, 16) || !aligned(keys, 4) || !aligned(perm, 4) ||
      !aligned(workspace, 256) || ws_bytes < spin4d_morton_order_workspace(N))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_morton_order")) return SPIN4D_ERR_INJECTED;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint32_t* keys_b = reinterpret_cast<uint32_t*>(w);
  uint32_t* vals_b = reinterpret_cast<uint32_t*>(w + align256((size_t)N * 4));
  uint32_t* counts = reinterpret_cast<uint32_t*>(w + 2 * align256((size_t)N * 4));
  uint32_t* offsets = counts + align256((size_t)scan_len(N) * 4) / 4;
  uint32_t* partial = offsets + align256((size_t)scan_len(N) * 4) / 4;
  const GridParams gp = make_grid_params(g);
  morton_keys_kernel<<<persistent_blocks((N + 255) / 256, 8), 256, 0, s>>>(gp, reinterpret_cast<const float4*>(pos), N,
                                                                            keys);
  SPIN4D_CHECK(launch_status());
  const int B = (int)sort_blocks(N);
  const int64_t len = scan_len(N);
  const int chunks = (int)scan_chunks(N);
  uint32_t *ka = keys, *kb = keys_b, *va = perm, *vb = vals_b;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 8 * pass;
    radix_histogram<<<B, kSortThreads, 0, s>>>(ka, N, shift, counts);
    scan_reduce<<<chunks, kScanThreads, 0, s>>>(counts, len, partial);
    scan_partials<<<1, kScanThreads, 0, s>>>(partial, chunks);
    scan_apply<<<chunks, kScanThreads, 0, s>>>(counts, len, partial, offsets);
    radix_scatter<<<B, kSortThreads, 0, s>>>(ka, pass == 0 ? nullptr : va, N, shift, offsets, kb, vb);
    SPIN4D_CHECK(launch_status());
    uint32_t* t = ka; ka = kb; kb = t;
    t = va; va = vb; vb = t;
  }
  // four passes: the sorted keys and permutation are back in keys / perm
  return SPIN4D_OK;
}

extern "C" int spin4d_permute_rows(const void* src, int64_t src_rows, void* dst, const uint32_t* perm, int64_t N,
                                   int64_t row_bytes, spin4d_stream_t stream) {
  if (N < 0 || src_rows < 0 || row_bytes <= 0 || row_bytes % 4) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  if (!src || !dst || !perm || src == dst || !aligned(src, 4) || !aligned(dst, 4) || !aligned(perm, 4))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_permute_rows")) return SPIN4D_ERR_INJECTED;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t words = row_bytes / 4;
  const bool vec = row_bytes % 16 == 0 && aligned(src, 16) && aligned(dst, 16);
  const int64_t total = N * (vec ? words / 4 : words);
  const int blocks = persistent_blocks((total + 255) / 256, 8);
  if (vec)
    permute_rows_kernel<true><<<blocks, 256, 0, s>>>(static_cast<const uint32_t*>(src), src_rows,
                                                     static_cast<uint32_t*>(dst), perm, N, words);
  else
    permute_rows_kernel<false><<<blocks, 256, 0, s>>>(static_cast<const uint32_t*>(src), src_rows,
                                                      static_cast<uint32_t*>(dst), perm, N, words);
  return launch_status();
}
