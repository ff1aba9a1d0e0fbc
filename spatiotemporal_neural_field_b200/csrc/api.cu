// Host-side C ABI plumbing: descriptors, validation, status strings, the
// fault-injection hook and Eq. 2 covariance assembly as a standalone call.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "host.h"

namespace spin4d {

static thread_local int g_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SPIN4D_OK;
  g_last_cuda_error = (int)e;
  return SPIN4D_ERR_CUDA;
}

int launch_status() { return cuda_status(cudaGetLastError()); }

bool fault_injected(const char* entry) {
  static std::once_flag once;
  static char name[128] = {0};
  std::call_once(once, [] {
    const char* v = getenv("SPIN4D_FAULT");
    if (v) strncpy(name, v, sizeof(name) - 1);
  });
  return name[0] != 0 && strcmp(name, entry) == 0;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int validate_grid(const spin4d_grid_desc* g) {
  if (!g) return SPIN4D_ERR_INVALID;
  if (g->L < 1 || g->L > SPIN4D_MAX_LEVELS) return SPIN4D_ERR_INVALID;
  if (!(g->F == 1 || g->F == 2 || g->F == 4 || g->F == 8)) return SPIN4D_ERR_INVALID;
  if (g->log2_T < 4 || g->log2_T > 24) return SPIN4D_ERR_INVALID;
  if (g->table_dtype != SPIN4D_F32 && g->table_dtype != SPIN4D_F16) return SPIN4D_ERR_INVALID;
  if (g->flags & ~SPIN4D_INPUT_NORMALISED) return SPIN4D_ERR_INVALID;
  if (g->reserved != 0) return SPIN4D_ERR_INVALID;
  if (!(g->t_max > g->t_min) || !isfinite(g->t_min) || !isfinite(g->t_max)) return SPIN4D_ERR_INVALID;
  for (int l = 0; l < g->L; ++l)
    for (int d = 0; d < 4; ++d)
      if (g->res[l][d] < 2 || g->res[l][d] > (1 << 24)) return SPIN4D_ERR_INVALID;
  return SPIN4D_OK;
}

int validate_mlp(const spin4d_grid_desc* g, const spin4d_mlp_desc* m) {
  if (!m) return SPIN4D_ERR_INVALID;
  if (m->in_dim != g->L * g->F) return SPIN4D_ERR_INVALID;
  if (m->in_dim < 1 || m->in_dim > SPIN4D_MAX_WIDTH) return SPIN4D_ERR_INVALID;
  if (m->hidden < 1 || m->hidden > SPIN4D_MAX_WIDTH) return SPIN4D_ERR_INVALID;
  if (m->n_hidden < 1 || m->n_hidden > 4) return SPIN4D_ERR_INVALID;
  if (m->w_dtype != SPIN4D_F32 && m->w_dtype != SPIN4D_F16) return SPIN4D_ERR_INVALID;
  if (m->gate != 0 && m->gate != 1) return SPIN4D_ERR_INVALID;
  if (m->gate && !(m->tau > 0.0f)) return SPIN4D_ERR_INVALID;
  return SPIN4D_OK;
}

int validate_hex(const spin4d_hexplane_desc* h) {
  if (!h) return SPIN4D_ERR_INVALID;
  if (h->n_scales < 1 || h->n_scales > 4) return SPIN4D_ERR_INVALID;
  for (int s = 0; s < h->n_scales; ++s)
    if (h->scales[s] < 2 || h->scales[s] > 4096) return SPIN4D_ERR_INVALID;
  if (h->time_res < 2 || h->time_res > 4096) return SPIN4D_ERR_INVALID;
  if (h->channels < 4 || h->channels > 32 || h->channels % 4) return SPIN4D_ERR_INVALID;
  if (h->n_frames < 2) return SPIN4D_ERR_INVALID;
  if (h->hidden < 1 || h->hidden > SPIN4D_MAX_WIDTH) return SPIN4D_ERR_INVALID;
  if (h->n_hidden < 1 || h->n_hidden > 4) return SPIN4D_ERR_INVALID;
  return SPIN4D_OK;
}

GridParams make_grid_params(const spin4d_grid_desc* g) {
  GridParams p;
  memset(&p, 0, sizeof(p));
  p.L = g->L;
  p.F = g->F;
  p.log2_T = g->log2_T;
  p.table_dtype = g->table_dtype;
  p.mask = (uint32_t)((1ull << g->log2_T) - 1ull);
  p.flags = g->flags;
  p.t_min = g->t_min;
  p.span = (float)(g->t_max - g->t_min);   // fp32 difference, as Eq. 8 is evaluated
  uint64_t T = 1ull << g->log2_T;
  for (int l = 0; l < g->L; ++l) {
    uint64_t prod = 1;
    for (int d = 0; d < 4; ++d) {
      p.max_cell[l][d] = g->res[l][d] - 2;
      p.scale[l][d] = (float)(g->res[l][d] - 1);
      p.stride[l][d] = (uint32_t)prod;
      prod *= (uint64_t)g->res[l][d];
      if (prod > (1ull << 40)) prod = (1ull << 40);
    }
    if (prod <= T) p.dense_bits |= 1u << l;
  }
  return p;
}

int sm_count() {
  static int cached = 0;
  if (cached) return cached;
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  cached = n;
  return n;
}

int persistent_blocks(int64_t n_tiles, int per_sm) {
  int64_t cap = (int64_t)sm_count() * per_sm;
  int64_t b = n_tiles < cap ? n_tiles : cap;
  return (int)(b < 1 ? 1 : b);
}

// ---------------------------------------------------------------------------
// Eq. 2 as a standalone call.
// ---------------------------------------------------------------------------
__global__ void cov_assemble_kernel(const float* __restrict__ scale, const float* __restrict__ rot,
                                    int64_t N, float* __restrict__ cov) {
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N;
       n += (int64_t)gridDim.x * blockDim.x) {
    float s[3] = {scale[3 * n], scale[3 * n + 1], scale[3 * n + 2]};
    float4 q4 = reinterpret_cast<const float4*>(rot)[n];
    float q[4] = {q4.x, q4.y, q4.z, q4.w};
    float c[6];
    covariance(s, q, c);
#pragma unroll
    for (int p = 0; p < 6; ++p) cov[6 * n + p] = c[p];
  }
}

}  // namespace spin4d

using namespace spin4d;

namespace spin4d {
// Readers of the translation units' bounds words (checked build only; they
// register themselves while the library loads).
static int (*g_bounds_readers[32])(int) = {nullptr};
static int g_n_bounds_readers = 0;

int register_bounds_word(int (*reader)(int clear)) {
  if (g_n_bounds_readers < 32) g_bounds_readers[g_n_bounds_readers++] = reader;
  return g_n_bounds_readers;
}

// SPIN4D_ERR_BOUNDS if a checked-build bounds check failed since the last
// clear, SPIN4D_ERR_CUDA if a word could not be read, else SPIN4D_OK.
int bounds_status(int clear) {
  int st = SPIN4D_OK;
  for (int i = 0; i < g_n_bounds_readers; ++i) {
    const int v = g_bounds_readers[i](clear);
    if (v < 0) return SPIN4D_ERR_CUDA;
    if (v) st = SPIN4D_ERR_BOUNDS;
  }
  return st;
}
}  // namespace spin4d

extern "C" {

int spin4d_grid_init(spin4d_grid_desc* g, int L, int F, int log2_T, int table_dtype, int nmin_s,
                     int nmax_s, int nmin_t, int nmax_t, float t_min, float t_max) {
  if (!g) return SPIN4D_ERR_INVALID;
  if (L < 1 || L > SPIN4D_MAX_LEVELS || nmin_s < 2 || nmax_s < nmin_s || nmin_t < 2 || nmax_t < nmin_t)
    return SPIN4D_ERR_INVALID;
  memset(g, 0, sizeof(*g));
  g->L = L;
  g->F = F;
  g->log2_T = log2_T;
  g->table_dtype = table_dtype;
  g->t_min = t_min;
  g->t_max = t_max;
  const int nmin[2] = {nmin_s, nmin_t}, nmax[2] = {nmax_s, nmax_t};
  for (int a = 0; a < 2; ++a) {
    // Instant-NGP growth factor b = exp((ln Nmax - ln Nmin)/(L-1)), in double
    double b = L > 1 ? exp((log((double)nmax[a]) - log((double)nmin[a])) / (double)(L - 1)) : 1.0;
    for (int l = 0; l < L; ++l) {
      int r = (int)floor((double)nmin[a] * pow(b, (double)l) + 1e-9);
      if (a == 0) {
        g->res[l][0] = g->res[l][1] = g->res[l][2] = r;
      } else {
        g->res[l][3] = r;
      }
    }
  }
  return validate_grid(g);
}

int64_t spin4d_mlp_param_count(const spin4d_mlp_desc* m) {
  if (!m || m->in_dim < 1 || m->hidden < 1 || m->n_hidden < 1) return -1;
  int64_t n = 0, d = m->in_dim;
  for (int j = 0; j < m->n_hidden; ++j) {
    n += (int64_t)m->hidden * d + m->hidden;
    d = m->hidden;
  }
  n += (int64_t)kHeadRows * d + kHeadRows;
  return n;
}

int spin4d_cov_assemble(const float* scale, const float* rot, int64_t N, float* cov, spin4d_stream_t stream) {
  if (N < 0) return SPIN4D_ERR_INVALID;
  if (N == 0) return SPIN4D_OK;
  if (!scale || !rot || !cov || !aligned(rot, 16) || !aligned(scale, 4) || !aligned(cov, 4))
    return SPIN4D_ERR_INVALID;
  if (fault_injected("spin4d_cov_assemble")) return SPIN4D_ERR_INJECTED;
  int blocks = persistent_blocks((N + 255) / 256, 8);
  cov_assemble_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(scale, rot, N, cov);
  return launch_status();
}

const char* spin4d_status_string(int s) {
  switch (s) {
    case SPIN4D_OK: return "ok";
    case SPIN4D_ERR_INVALID: return "invalid argument";
    case SPIN4D_ERR_UNSUPPORTED: return "unsupported shape";
    case SPIN4D_ERR_CUDA: return "CUDA error";
    case SPIN4D_ERR_NONFINITE: return "non-finite value";
    case SPIN4D_ERR_INJECTED: return "injected fault";
    case SPIN4D_ERR_TIMEOUT: return "device wait timed out";
    case SPIN4D_ERR_BOUNDS: return "device bounds check failed (checked build)";
    default: return "unknown status";
  }
}

int spin4d_last_cuda_error(void) { return g_last_cuda_error; }

int spin4d_checked_build(void) {
#ifdef SPIN4D_CHECKED
  return 1;
#else
  return 0;
#endif
}

// The persisting-L2 limit of the current context before the first window was
// set (restored by spin4d_l2_window_clear), per device.
static std::mutex g_l2_mu;
static bool g_l2_saved[64] = {false};
static size_t g_l2_prev[64] = {0};

int spin4d_l2_window_set(spin4d_stream_t stream, const void* base, size_t bytes, size_t* applied_bytes) {
  if (!stream || !base || bytes == 0) return SPIN4D_ERR_INVALID;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= 64) return SPIN4D_ERR_UNSUPPORTED;
  int max_persist = 0, max_window = 0;
  e = cudaDeviceGetAttribute(&max_persist, cudaDevAttrMaxPersistingL2CacheSize, dev);
  if (e != cudaSuccess) return cuda_status(e);
  e = cudaDeviceGetAttribute(&max_window, cudaDevAttrMaxAccessPolicyWindowSize, dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (max_persist <= 0 || max_window <= 0) return SPIN4D_ERR_UNSUPPORTED;
  const size_t window = bytes < (size_t)max_window ? bytes : (size_t)max_window;
  const size_t setaside = window < (size_t)max_persist ? window : (size_t)max_persist;
  {
    std::lock_guard<std::mutex> lock(g_l2_mu);
    if (!g_l2_saved[dev]) {
      e = cudaDeviceGetLimit(&g_l2_prev[dev], cudaLimitPersistingL2CacheSize);
      if (e != cudaSuccess) return cuda_status(e);
      g_l2_saved[dev] = true;
    }
  }
  e = cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, setaside);
  if (e != cudaSuccess) return cuda_status(e);
  cudaStreamAttrValue attr;
  memset(&attr, 0, sizeof(attr));
  attr.accessPolicyWindow.base_ptr = const_cast<void*>(base);
  attr.accessPolicyWindow.num_bytes = window;
  attr.accessPolicyWindow.hitRatio = (float)((double)setaside / (double)window);
  attr.accessPolicyWindow.hitProp = cudaAccessPropertyPersisting;
  attr.accessPolicyWindow.missProp = cudaAccessPropertyStreaming;
  e = cudaStreamSetAttribute((cudaStream_t)stream, cudaStreamAttributeAccessPolicyWindow, &attr);
  if (e != cudaSuccess) return cuda_status(e);
  if (applied_bytes) *applied_bytes = window;
  return SPIN4D_OK;
}

int spin4d_l2_window_clear(spin4d_stream_t stream) {
  if (!stream) return SPIN4D_ERR_INVALID;
  cudaStreamAttrValue attr;
  memset(&attr, 0, sizeof(attr));
  attr.accessPolicyWindow.num_bytes = 0;
  attr.accessPolicyWindow.hitProp = cudaAccessPropertyNormal;
  attr.accessPolicyWindow.missProp = cudaAccessPropertyNormal;
  cudaError_t e = cudaStreamSetAttribute((cudaStream_t)stream, cudaStreamAttributeAccessPolicyWindow, &attr);
  if (e != cudaSuccess) return cuda_status(e);
  // lines already marked persisting return to normal
  e = cudaCtxResetPersistingL2Cache();
  if (e != cudaSuccess) return cuda_status(e);
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  std::lock_guard<std::mutex> lock(g_l2_mu);
  if (dev >= 0 && dev < 64 && g_l2_saved[dev]) {
    e = cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, g_l2_prev[dev]);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return SPIN4D_OK;
}

const char* spin4d_version(void) { return "0.1.0"; }

}  // extern "C"
