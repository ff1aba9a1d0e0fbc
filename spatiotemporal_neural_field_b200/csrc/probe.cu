// Gather-rate probe: the denominator of the decoder's gather roofline.
//
// The decoder's hash-grid gathers touch one 32-byte sector per table access
// at effectively random addresses, so neither a streaming copy (HBM peak) nor
// a dense GEMM describes their ceiling.  This kernel measures it directly:
// every thread issues independent `width`-byte loads at pseudo-random,
// width-aligned offsets of a buffer (32 MiB stays resident in L2; 1 GiB and up
// streams from HBM), eight loads in flight per thread, and folds the loaded
// words into a sink so nothing is optimised away.
#include "host.h"

namespace spin4d {
namespace {

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
  uint32_t state = mix32(tid * 0x9E3779B9u ^ seed);
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
      uint4 v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = __ldg(reinterpret_cast<const uint4*>(buf) + off[k]);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc += v[k].x ^ v[k].w;
    }
  }
  if (acc == 0x12345678u) sink[0] = acc;   // practically never taken; keeps the loads alive
}

}  // namespace
}  // namespace spin4d

using namespace spin4d;

extern "C" int spin4d_probe_gather(const void* buf, uint64_t buf_bytes, int width, int64_t loads_per_thread,
                                   int blocks, uint32_t seed, uint32_t* sink, spin4d_stream_t stream) {
  if (!buf || !sink || (width != 4 && width != 16) || buf_bytes < (uint64_t)width || loads_per_thread < 8 ||
      loads_per_thread % 8 || blocks < 1 || !aligned(buf, 16))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_probe_gather")) return SPIN4D_ERR_INJECTED;
  const uint64_t slots = buf_bytes / (uint64_t)width;
  const uint8_t* b = static_cast<const uint8_t*>(buf);
  if (width == 4)
    probe_gather_kernel<4><<<blocks, 256, 0, (cudaStream_t)stream>>>(b, slots, loads_per_thread, seed, sink);
  else
    probe_gather_kernel<16><<<blocks, 256, 0, (cudaStream_t)stream>>>(b, slots, loads_per_thread, seed, sink);
  return launch_status();
}
