// 4D multiresolution hash encoding on its own (SPIN-4DGS section 3.3,
// Eq. 7-9) and the corner-selection test hook.
#include "host.h"

namespace spin4d {

// One thread per position, levels in order; the LF features of a position are
// written as one contiguous row of z.
template <typename T, int F>
__global__ void __launch_bounds__(128) encode_kernel(GridParams g, const float4* __restrict__ pos,
                                                     int64_t N, const T* __restrict__ tables,
                                                     float* __restrict__ z) {
  const int LF = g.L * F;
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N;
       n += (int64_t)gridDim.x * blockDim.x) {
    float xt[4];
    normalise_position(pos[n], g, xt);
    float* zr = z + n * LF;
    for (int l = 0; l < g.L; ++l) {
      float acc[F];
      encode_level<T, F>(xt, g, l, tables, acc);
#pragma unroll
      for (int f = 0; f < F; ++f) zr[l * F + f] = acc[f];
    }
  }
}

__global__ void debug_corners_kernel(GridParams g, const float4* __restrict__ pos, int64_t N,
                                     uint32_t* __restrict__ idx, float* __restrict__ frac) {
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N;
       n += (int64_t)gridDim.x * blockDim.x) {
    float xt[4];
    normalise_position(pos[n], g, xt);
    for (int l = 0; l < g.L; ++l) {
      uint32_t base[4], id[16];
      float fr[4];
      level_cell(xt, g, l, base, fr);
      level_indices(base, g, l, id);
      uint32_t* ip = idx + (n * g.L + l) * 16;
      float* fp = frac + (n * g.L + l) * 4;
#pragma unroll
      for (int c = 0; c < 16; ++c) ip[c] = id[c];
#pragma unroll
      for (int d = 0; d < 4; ++d) fp[d] = fr[d];
    }
  }
}

template <typename T>
static int launch_encode(const GridParams& p, const float* pos, int64_t N, const void* tables, float* z,
                         cudaStream_t s) {
  int blocks = persistent_blocks((N + 127) / 128, 16);
  const float4* P = reinterpret_cast<const float4*>(pos);
  const T* tab = static_cast<const T*>(tables);
  switch (p.F) {
    case 1: encode_kernel<T, 1><<<blocks, 128, 0, s>>>(p, P, N, tab, z); break;
    case 2: encode_kernel<T, 2><<<blocks, 128, 0, s>>>(p, P, N, tab, z); break;
    case 4: encode_kernel<T, 4><<<blocks, 128, 0, s>>>(p, P, N, tab, z); break;
    case 8: encode_kernel<T, 8><<<blocks, 128, 0, s>>>(p, P, N, tab, z); break;
    default: return SPIN4D_ERR_UNSUPPORTED;
  }
  return launch_status();
}

}  // namespace spin4d

using namespace spin4d;

extern "C" int spin4d_encode_fwd(const spin4d_grid_desc* g, const float* pos, int64_t N, const void* tables,
                                 float* z, spin4d_stream_t stream) {
  SPIN4D_CHECK(validate_grid(g));
  if (N < 0) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  size_t esz = g->table_dtype == SPIN4D_F16 ? 2 : 4;
  if (!pos || !tables || !z || !aligned(pos, 16) || !aligned(tables, esz * g->F > 16 ? 16 : esz * g->F) ||
      !aligned(z, 4))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_encode_fwd")) return SPIN4D_ERR_INJECTED;
  GridParams p = make_grid_params(g);
  cudaStream_t s = (cudaStream_t)stream;
  if (g->table_dtype == SPIN4D_F16) return launch_encode<__half>(p, pos, N, tables, z, s);
  return launch_encode<float>(p, pos, N, tables, z, s);
}

extern "C" int spin4d_debug_corners(const spin4d_grid_desc* g, const float* pos, int64_t N, uint32_t* idx,
                                    float* frac, spin4d_stream_t stream) {
  SPIN4D_CHECK(validate_grid(g));
  if (N < 0) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  if (!pos || !idx || !frac || !aligned(pos, 16) || !aligned(idx, 4) || !aligned(frac, 4))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_debug_corners")) return SPIN4D_ERR_INJECTED;
  GridParams p = make_grid_params(g);
  int blocks = persistent_blocks((N + 127) / 128, 16);
  debug_corners_kernel<<<blocks, 128, 0, (cudaStream_t)stream>>>(p, reinterpret_cast<const float4*>(pos), N,
                                                                 idx, frac);
  return launch_status();
}
