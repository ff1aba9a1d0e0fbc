// Host-side helpers shared by the spin4d entry points: argument validation,
// derived grid constants, error bookkeeping and the host fault-injection hook.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "spin4d.h"

namespace spin4d {

// Records `e` as the last CUDA error of this thread and maps it to a status.
int cuda_status(cudaError_t e);
// Status after a launch: checks cudaGetLastError().
int launch_status();
// True when SPIN4D_FAULT names `entry` (read once per process).
bool fault_injected(const char* entry);

bool aligned(const void* p, size_t a);
int validate_grid(const spin4d_grid_desc* g);
int validate_mlp(const spin4d_grid_desc* g, const spin4d_mlp_desc* m);
int validate_hex(const spin4d_hexplane_desc* h);
GridParams make_grid_params(const spin4d_grid_desc* g);

// Persistent-grid size: blocks for N items of `per_block`, capped at
// `per_sm` resident blocks on every SM of the current device.
int persistent_blocks(int64_t n_tiles, int per_sm);
int sm_count();

}  // namespace spin4d

#define SPIN4D_CHECK(expr)            \
  do {                                \
    int _st = (expr);                 \
    if (_st != SPIN4D_OK) return _st; \
  } while (0)
