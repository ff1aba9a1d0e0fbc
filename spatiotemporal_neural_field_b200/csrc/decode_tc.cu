// Tensor-core fused decoder (fp16 tables and weights): placeholder until the
// tcgen05 path lands; every call falls through to the SIMT kernels.
#include "host.h"

namespace spin4d {

int decode_fwd_tc(const spin4d_grid_desc*, const spin4d_mlp_desc*, const float*, int64_t, const void*,
                  const void*, const float*, const spin4d_outputs&, cudaStream_t, bool* handled) {
  *handled = false;
  return SPIN4D_OK;
}

}  // namespace spin4d
