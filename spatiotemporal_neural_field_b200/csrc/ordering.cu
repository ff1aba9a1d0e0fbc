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
// (every Gaussian is decoded at every frame).  The codes are sorted by the
// stable four-pass radix sort of radix.cuh.
#include "host.h"
#include "radix.cuh"

namespace spin4d {
namespace {

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

}  // namespace
}  // namespace spin4d

using namespace spin4d;

// Workspace: keys' and values' second buffers, then the sort's scratch.
extern "C" size_t spin4d_morton_order_workspace(int64_t N) {
  if (N <= 0 || N > SPIN4D_MAX_SORT) return 0;
  return 2 * radix::align256((size_t)N * 4) + radix::scratch_bytes(N);
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
  uint32_t* vals_b = reinterpret_cast<uint32_t*>(w + radix::align256((size_t)N * 4));
  void* scratch = w + 2 * radix::align256((size_t)N * 4);
  const GridParams gp = make_grid_params(g);
  morton_keys_kernel<<<persistent_blocks((N + 255) / 256, 8), 256, 0, s>>>(gp, reinterpret_cast<const float4*>(pos), N,
                                                                            keys);
  SPIN4D_CHECK(launch_status());
  // four passes: the sorted keys and permutation end in keys / perm
  radix::sort_pairs(keys, perm, keys_b, vals_b, true, N, nullptr, 4, scratch, s);
  return launch_status();
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
