// Stable least-significant-digit radix sort of 32-bit keys with 32-bit
// values, 8-bit digits.  Each pass: a histogram kernel, a two-kernel
// exclusive scan of the (digit, block) counts and a scatter kernel that
// ranks each block's keys stably (warp match on the digit, then a prefix
// over the warps), so equal keys keep their input order and the result is
// deterministic.
//
// The grid is fixed by the capacity (at most kMaxSortBlocks blocks, a few per
// SM); each block owns one contiguous chunk of the keys, sized from the key
// count at run time.  That count may live on the device (n_dev, clamped to
// the capacity), so a sort can follow a kernel that produced a
// data-dependent number of keys without a host sync, and the scan stays
// sized by the grid, not by the capacity.  The kernels of a sort are
// launched as programmatic dependents of each other (pdl.cuh).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pdl.cuh"

namespace spin4d {
namespace radix {
namespace {   // every translation unit that sorts gets its own copy of the kernels

constexpr int kSortThreads = 256;              // keys ranked per round
constexpr int kMinKeysPerBlock = 2048;
constexpr int kMaxSortBlocks = 640;
constexpr int kDigits = 256;
constexpr int kScanThreads = 1024;
constexpr int kScanPerThread = 8;
constexpr int kScanChunk = kScanThreads * kScanPerThread;
constexpr int kFusedScanMaxChunks = 1024;      // above this the chunk partials get their own scan kernel

inline int sort_blocks(int64_t N) {
  const int64_t b = (N + kMinKeysPerBlock - 1) / kMinKeysPerBlock;
  return (int)(b < 1 ? 1 : (b > kMaxSortBlocks ? kMaxSortBlocks : b));
}
inline int64_t scan_len(int64_t N) { return (int64_t)sort_blocks(N) * kDigits; }
inline int64_t scan_chunks(int64_t len) { return (len + kScanChunk - 1) / kScanChunk; }
inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Block b's keys: [b * chunk, min((b + 1) * chunk, n)), chunk a multiple of
// kSortThreads.
__device__ __forceinline__ void block_chunk(int64_t N, const uint32_t* n_dev, int64_t& lo, int64_t& hi) {
  const int64_t n = n_dev ? min(N, (int64_t)*n_dev) : N;
  int64_t chunk = (n + gridDim.x - 1) / gridDim.x;
  chunk = (chunk + kSortThreads - 1) / kSortThreads * kSortThreads;
  lo = min((int64_t)blockIdx.x * chunk, n);
  hi = min(lo + chunk, n);
}

// counts[d * B + b] = keys of block b whose digit is d.
__global__ void __launch_bounds__(kSortThreads) radix_histogram(const uint32_t* __restrict__ keys, int64_t N,
                                                                const uint32_t* __restrict__ n_dev, int shift,
                                                                uint32_t* __restrict__ counts) {
  pdl_wait();
  pdl_release();
  __shared__ uint32_t h[kDigits];
  h[threadIdx.x] = 0;
  __syncthreads();
  int64_t lo, hi;
  block_chunk(N, n_dev, lo, hi);
  for (int64_t i = lo + threadIdx.x; i < hi; i += kSortThreads) atomicAdd(&h[(keys[i] >> shift) & 0xFFu], 1u);
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

// A scan chunk moves between global and shared memory with coalesced
// accesses (thread t touches t, t + kScanThreads, ...); each thread then
// works on its kScanPerThread consecutive values in shared memory, read with
// a padded stride so the eight-apart rows fall in different banks.
__device__ __forceinline__ int padded(int e) { return e + (e >> 5); }
constexpr int kScanShared = kScanChunk + kScanChunk / 32;

__device__ __forceinline__ void load_chunk(const uint32_t* __restrict__ a, int64_t n, uint32_t* sm) {
  const int64_t c0 = (int64_t)blockIdx.x * kScanChunk;
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) {
    const int e = k * kScanThreads + threadIdx.x;
    sm[padded(e)] = c0 + e < n ? a[c0 + e] : 0u;
  }
  __syncthreads();
}

// Scan step 1: partial[c] = sum of chunk c of a.
__global__ void __launch_bounds__(kScanThreads) scan_reduce(const uint32_t* __restrict__ a, int64_t n,
                                                            uint32_t* __restrict__ partial) {
  pdl_wait();
  pdl_release();
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t sm[kScanShared];
  load_chunk(a, n, sm);
  uint32_t s = 0;
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) s += sm[padded(threadIdx.x * kScanPerThread + k)];
  uint32_t total;
  block_exclusive_scan(s, s_warp, total);
  if (threadIdx.x == 0) partial[blockIdx.x] = total;
}

// Scan step 2 for many chunks (one block): partial[] -> its exclusive scan, in place.
__global__ void __launch_bounds__(kScanThreads) scan_partials(uint32_t* __restrict__ partial, int n) {
  pdl_wait();
  pdl_release();
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

// Last step: out = exclusive scan of a.  FUSED: chunk c's start is the sum of
// partial[0..c) (the raw chunk sums), added up here; otherwise partial[c]
// already holds it.
template <bool FUSED>
__global__ void __launch_bounds__(kScanThreads) scan_apply(const uint32_t* __restrict__ a, int64_t n,
                                                           const uint32_t* __restrict__ partial,
                                                           uint32_t* __restrict__ out) {
  pdl_wait();
  pdl_release();
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_base;
  __shared__ uint32_t sm[kScanShared];
  if (FUSED) {
    if (threadIdx.x < 32) {
      uint32_t acc = 0;
      for (int c = threadIdx.x; c < (int)blockIdx.x; c += 32) acc += partial[c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (threadIdx.x == 0) s_base = acc;
    }
  }
  load_chunk(a, n, sm);   // its barrier also publishes s_base
  uint32_t v[kScanPerThread];
  uint32_t s = 0;
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) {
    v[k] = sm[padded(threadIdx.x * kScanPerThread + k)];
    s += v[k];
  }
  uint32_t total;
  uint32_t run = (FUSED ? s_base : partial[blockIdx.x]) + block_exclusive_scan(s, s_warp, total);
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) {
    sm[padded(threadIdx.x * kScanPerThread + k)] = run;
    run += v[k];
  }
  __syncthreads();
  const int64_t c0 = (int64_t)blockIdx.x * kScanChunk;
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) {
    const int e = k * kScanThreads + threadIdx.x;
    if (c0 + e < n) out[c0 + e] = sm[padded(e)];
  }
}

// Stable scatter of one block's chunk by digit, kSortThreads keys per round:
// the rank of a key among the block's keys of its digit counts the earlier
// rounds, the earlier warps of its round and the earlier lanes of its warp.
// vals_in == NULL means the values are the input indices.
__global__ void __launch_bounds__(kSortThreads) radix_scatter(const uint32_t* __restrict__ keys_in,
                                                              const uint32_t* __restrict__ vals_in, int64_t N,
                                                              const uint32_t* __restrict__ n_dev,
                                                              int shift, const uint32_t* __restrict__ offsets,
                                                              uint32_t* __restrict__ keys_out,
                                                              uint32_t* __restrict__ vals_out) {
  pdl_wait();
  pdl_release();
  constexpr int kWarps = kSortThreads / 32;
  __shared__ uint32_t base[kDigits];          // global position of this block's next key of each digit
  __shared__ uint32_t wcnt[kWarps][kDigits];  // per round: keys per (warp, digit), then their prefix
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t lo, hi;
  block_chunk(N, n_dev, lo, hi);
  base[tid] = offsets[(size_t)tid * gridDim.x + blockIdx.x];
  const uint32_t lt = (1u << lane) - 1u;
  for (int64_t r0 = lo; r0 < hi; r0 += kSortThreads) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wcnt[w][tid] = 0u;
    __syncthreads();
    const int64_t i = r0 + tid;
    const bool valid = i < hi;
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

// Scratch for an exclusive scan of n values.
inline size_t exclusive_scan_scratch(int64_t n) { return align256((size_t)scan_chunks(n) * 4); }

// out = exclusive scan of a[0..n) (n < 2^32 / 2, sums below 2^32).
inline void exclusive_scan(const uint32_t* a, int64_t n, uint32_t* out, void* scratch, cudaStream_t s) {
  const int chunks = (int)scan_chunks(n);
  uint32_t* partial = static_cast<uint32_t*>(scratch);
  launch_pdl(scan_reduce, chunks, kScanThreads, 0, s, a, n, partial);
  if (chunks <= kFusedScanMaxChunks) {
    launch_pdl(scan_apply<true>, chunks, kScanThreads, 0, s, a, n, partial, out);
  } else {
    launch_pdl(scan_partials, 1, kScanThreads, 0, s, partial, chunks);
    launch_pdl(scan_apply<false>, chunks, kScanThreads, 0, s, a, n, partial, out);
  }
}

// Scratch for sorting up to N keys: the (digit, block) counts, their scan and
// the scan's chunk partials.
inline size_t scratch_bytes(int64_t N) {
  return 2 * align256((size_t)scan_len(N) * 4) + exclusive_scan_scratch(scan_len(N));
}

// Sorts (keys, vals) by bits [0, 8 * passes) of the keys, ping-ponging with
// (keys_b, vals_b).  With vals_are_index the first pass takes the input
// indices as values.  N is the capacity; n_dev (or N) the key count.
// Returns true when the result is in (keys, vals) (an even number of
// passes), false when in (keys_b, vals_b).
inline bool sort_pairs(uint32_t* keys, uint32_t* vals, uint32_t* keys_b, uint32_t* vals_b, bool vals_are_index,
                       int64_t N, const uint32_t* n_dev, int passes, void* scratch, cudaStream_t s) {
  uint32_t* counts = static_cast<uint32_t*>(scratch);
  uint32_t* offsets = counts + align256((size_t)scan_len(N) * 4) / 4;
  void* scan_scratch = offsets + align256((size_t)scan_len(N) * 4) / 4;
  const int B = sort_blocks(N);
  const int64_t len = scan_len(N);
  uint32_t *ka = keys, *kb = keys_b, *va = vals, *vb = vals_b;
  for (int pass = 0; pass < passes; ++pass) {
    const int shift = 8 * pass;
    launch_pdl(radix_histogram, B, kSortThreads, 0, s, ka, N, n_dev, shift, counts);
    exclusive_scan(counts, len, offsets, scan_scratch, s);
    launch_pdl(radix_scatter, B, kSortThreads, 0, s, ka, (pass == 0 && vals_are_index) ? nullptr : va, N, n_dev,
               shift, offsets, kb, vb);
    uint32_t* t = ka; ka = kb; kb = t;
    t = va; va = vb; vb = t;
  }
  return (passes % 2) == 0;
}

}  // namespace
}  // namespace radix
}  // namespace spin4d
