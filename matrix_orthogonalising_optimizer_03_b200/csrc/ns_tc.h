// Host interface of the tensor-core Newton-Schulz phases.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "muon_internal.h"

namespace muon {

// Kernel parameters: per class, the tensor maps of the A and B operands of the
// phase, plus the phase arguments. Passed as a __grid_constant__ parameter so
// the TMA unit reads the maps from parameter space.
struct TcParams {
  CUtensorMap ta[kMaxClassesPerLaunch];
  CUtensorMap tb[kMaxClassesPerLaunch];
  NsPhaseArgs args;
};

// Tile sizes of the tensor-core phases (rows x cols of an output tile, k-block).
int tc_block_m();
int tc_block_n(int phase);
int tc_block_k();

cudaError_t launch_ns_phase_tc(const TcParams& P, int num_sms, cudaStream_t s);

bool encode_slab_map_bf16(CUtensorMap* out, const void* base, int64_t inner, int64_t rows,
                          int64_t count, int64_t ld, int box_inner, int box_rows);

}  // namespace muon
