// Measurement probes: the denominators of the gather rooflines.
//
// The decoder's hash-grid gathers touch one 32-byte sector per table access
// at effectively random addresses, and the HexPlane encoder reads whole
// 128-byte channel rows at random rows, so neither a streaming copy (HBM
// peak) nor a dense GEMM describes their ceiling.  probe_gather measures it
// directly: independent loads at pseudo-random, width-aligned offsets of a
// buffer (32 MiB stays resident in L2; 1 GiB and up streams from HBM), eight
// in flight per thread, folded into a sink so nothing is optimised away.
// probe_atomic issues fp32 reductions (1, 2 or 4 floats, one 32-byte sector
// each) at random offsets: the ceiling of a gradient scatter.  probe_stream
// reads a buffer front to back (the sequential ceiling of
// wherever it lives) and probe_fma runs independent fp32 FMA chains (the
// CUDA-core arithmetic peak).
//
// Built into libspin4d_probe.so, a measurement and test library beside the
// decoder's libspin4d.so; it shares only the tensor-core helper header.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "spin4d_probe.h"
#include "tc.cuh"

namespace spin4d {
namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int launch_status() { return cudaGetLastError() == cudaSuccess ? SPIN4D_OK : SPIN4D_ERR_CUDA; }

// This library's device error word: set when a bounded wait runs out.
__device__ int g_probe_error = 0;

// Waits on an mbarrier that nothing ever arrives at, with the bounded wait
// of the decoder's tensor-core kernels: the wait runs out, the kernel
// records the timeout and returns.
__global__ void selftest_wait_timeout_kernel(uint32_t max_iters) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t mbar = tc::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(mbar, 1);
    tc::mbar_fence_init();
  }
  __syncthreads();
  const bool ok = tc::mbar_wait_bounded(mbar, 0, max_iters);
  if (__syncthreads_or(!ok) && threadIdx.x == 0) atomicExch(&g_probe_error, 1);
}

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  // integer finaliser of MurmurHash3 (public domain)
  x ^= x >> 16;
  x *= 0x85ebca6bu;
  x ^= x >> 13;
  x *= 0xc2b2ae35u;
  x ^= x >> 16;
  return x;
}

template <int W>
__global__ void __launch_bounds__(256) probe_gather_kernel(const uint8_t* __restrict__ buf, uint64_t n_slots,
                                                           int64_t loads_per_thread, uint32_t seed,
                                                           uint32_t* __restrict__ sink) {
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  // W = 128: the 8 lanes of a group share the random line and each loads one
  // of its 16-byte chunks, so one warp instruction reads 4 whole lines.
  const uint32_t key = W == 128 ? tid >> 3 : tid;
  uint32_t state = mix32(key * 0x9E3779B9u ^ seed);
  for (int64_t i = 0; i < loads_per_thread; i += 8) {
    uint64_t off[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      state = mix32(state + 0x6D2B79F5u);
      off[k] = ((uint64_t)state * n_slots) >> 32;   // uniform slot in [0, n_slots)
    }
    if constexpr (W == 4) {
      uint32_t v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = __ldg(reinterpret_cast<const uint32_t*>(buf) + off[k]);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc += v[k];
    } else {
      const uint64_t chunk = W == 128 ? (threadIdx.x & 7) : 0;
      uint4 v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = __ldg(reinterpret_cast<const uint4*>(buf) + off[k] * (W / 16) + chunk);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc += v[k].x ^ v[k].w;
    }
  }
  if (acc == 0x12345678u) sink[0] = acc;   // practically never taken; keeps the loads alive
}

template <int W>
__global__ void __launch_bounds__(256) probe_atomic_kernel(float* __restrict__ buf, uint64_t n_slots, int64_t ops,
                                                           uint32_t seed) {
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t state = mix32(tid * 0x9E3779B9u ^ seed);
  for (int64_t i = 0; i < ops; i += 8) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      state = mix32(state + 0x6D2B79F5u);
      const uint64_t slot = ((uint64_t)state * n_slots) >> 32;
      if constexpr (W == 4)
        atomicAdd(buf + slot, 1.0f);
      else if constexpr (W == 8)
        atomicAdd(reinterpret_cast<float2*>(buf) + slot, make_float2(1.0f, 1.0f));
      else
        atomicAdd(reinterpret_cast<float4*>(buf) + slot, make_float4(1.0f, 1.0f, 1.0f, 1.0f));
    }
  }
}

// Each thread owns a row of ones (RB bytes) in shared memory and adds it to
// random RB-byte rows of buf with bulk asynchronous reductions, at most 8 of
// its own in flight.
template <int RB>
__global__ void __launch_bounds__(128) probe_bulk_reduce_kernel(float* __restrict__ buf, uint64_t n_rows, int64_t ops,
                                                                uint32_t seed) {
  __shared__ __align__(128) float rows[128][RB / 4];
  for (int i = 0; i < RB / 4; ++i) rows[threadIdx.x][i] = 1.0f;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t state = mix32(tid * 0x9E3779B9u ^ seed);
  const uint32_t src = (uint32_t)__cvta_generic_to_shared(&rows[threadIdx.x][0]);
  for (int64_t i = 0; i < ops; ++i) {
    state = mix32(state + 0x6D2B79F5u);
    const uint64_t r = ((uint64_t)state * n_rows) >> 32;
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(buf + r * (RB / 4)),
                 "r"(src), "n"(RB)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group.read 8;" ::: "memory");
  }
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(256) probe_stream_kernel(const uint4* __restrict__ buf, uint64_t n16, int passes,
                                                           uint32_t* __restrict__ sink) {
  uint32_t acc = 0;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (int p = 0; p < passes; ++p) {
    uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n16; i += 4 * stride) {
      const uint4 a = __ldcg(buf + i), b = __ldcg(buf + i + stride), c = __ldcg(buf + i + 2 * stride),
                  d = __ldcg(buf + i + 3 * stride);
      acc += (a.x ^ b.y) + (c.z ^ d.w);
    }
    for (; i < n16; i += stride) acc += __ldcg(buf + i).x;
  }
  if (acc == 0x12345678u) sink[0] = acc;
}

__global__ void __launch_bounds__(256) probe_fma_kernel(int64_t iters, float seed, uint32_t* __restrict__ sink) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = seed + (float)(threadIdx.x + k);
  const float m = 0.999999f, c = 1e-7f;
  for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmaf(a[k], m, c);
  }
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) s += a[k];
  if (s == 1234.5f) sink[0] = 1;
}

}  // namespace
}  // namespace spin4d

using namespace spin4d;

extern "C" int spin4d_probe_gather(const void* buf, uint64_t buf_bytes, int width, int64_t loads_per_thread,
                                   int blocks, uint32_t seed, uint32_t* sink, spin4d_stream_t stream) {
  if (!buf || !sink || (width != 4 && width != 16 && width != 128) || buf_bytes < (uint64_t)width ||
      loads_per_thread < 8 || loads_per_thread % 8 || blocks < 1 || !aligned(buf, width == 128 ? 128 : 16))
    return SPIN4D_ERR_INVALID;
  const uint64_t slots = buf_bytes / (uint64_t)width;
  const uint8_t* b = static_cast<const uint8_t*>(buf);
  cudaStream_t s = (cudaStream_t)stream;
  if (width == 4)
    probe_gather_kernel<4><<<blocks, 256, 0, s>>>(b, slots, loads_per_thread, seed, sink);
  else if (width == 16)
    probe_gather_kernel<16><<<blocks, 256, 0, s>>>(b, slots, loads_per_thread, seed, sink);
  else
    probe_gather_kernel<128><<<blocks, 256, 0, s>>>(b, slots, loads_per_thread, seed, sink);
  return launch_status();
}

extern "C" int spin4d_probe_stream(const void* buf, uint64_t buf_bytes, int passes, int blocks, uint32_t* sink,
                                   spin4d_stream_t stream) {
  if (!buf || !sink || buf_bytes < 16 || buf_bytes % 16 || passes < 1 || blocks < 1 || !aligned(buf, 16))
    return SPIN4D_ERR_INVALID;
  probe_stream_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(static_cast<const uint4*>(buf), buf_bytes / 16, passes,
                                                                sink);
  return launch_status();
}

extern "C" int spin4d_probe_fma(int64_t iters, int blocks, uint32_t* sink, spin4d_stream_t stream) {
  if (!sink || iters < 1 || blocks < 1) return SPIN4D_ERR_INVALID;
  probe_fma_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(iters, 1.0f, sink);
  return launch_status();
}

extern "C" int spin4d_probe_atomic(void* buf, uint64_t buf_bytes, int width, int64_t ops_per_thread, int blocks,
                                   uint32_t seed, spin4d_stream_t stream) {
  if (!buf || (width != 4 && width != 8 && width != 16) || buf_bytes < (uint64_t)width || ops_per_thread < 8 ||
      ops_per_thread % 8 || blocks < 1 || !aligned(buf, 16))
    return SPIN4D_ERR_INVALID;
  const uint64_t slots = buf_bytes / (uint64_t)width;
  float* b = static_cast<float*>(buf);
  cudaStream_t s = (cudaStream_t)stream;
  if (width == 4)
    probe_atomic_kernel<4><<<blocks, 256, 0, s>>>(b, slots, ops_per_thread, seed);
  else if (width == 8)
    probe_atomic_kernel<8><<<blocks, 256, 0, s>>>(b, slots, ops_per_thread, seed);
  else
    probe_atomic_kernel<16><<<blocks, 256, 0, s>>>(b, slots, ops_per_thread, seed);
  return launch_status();
}

extern "C" int spin4d_probe_bulk_reduce(void* buf, uint64_t buf_bytes, int row_bytes, int64_t rows_per_thread,
                                        int blocks, uint32_t seed, spin4d_stream_t stream) {
  if (!buf || (row_bytes != 128 && row_bytes != 256) || buf_bytes < (uint64_t)row_bytes || rows_per_thread < 1 ||
      blocks < 1 || !aligned(buf, 128))
    return SPIN4D_ERR_INVALID;
  float* b = static_cast<float*>(buf);
  cudaStream_t s = (cudaStream_t)stream;
  if (row_bytes == 128)
    probe_bulk_reduce_kernel<128><<<blocks, 128, 0, s>>>(b, buf_bytes / 128, rows_per_thread, seed);
  else
    probe_bulk_reduce_kernel<256><<<blocks, 128, 0, s>>>(b, buf_bytes / 256, rows_per_thread, seed);
  return launch_status();
}

extern "C" int spin4d_selftest_wait_timeout(uint32_t max_iters, spin4d_stream_t stream) {
  if (max_iters < 1 || max_iters > (1u << 24)) return SPIN4D_ERR_INVALID;
  selftest_wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(max_iters);
  return launch_status();
}

extern "C" int spin4d_probe_check_device_errors(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_probe_error, sizeof(int)) != cudaSuccess) return SPIN4D_ERR_CUDA;
  if (clear && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_probe_error, &zero, sizeof(int)) != cudaSuccess) return SPIN4D_ERR_CUDA;
  }
  return v ? SPIN4D_ERR_TIMEOUT : SPIN4D_OK;
}
