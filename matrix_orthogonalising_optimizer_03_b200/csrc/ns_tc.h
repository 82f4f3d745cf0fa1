// Host interface of the tensor-core Newton-Schulz phases.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "muon_internal.h"

namespace muon {

// Kernel parameters: per class, the tensor maps of the A and B operands, of the
// epilogue's C tile and of the output, plus the phase arguments. Passed as a __grid_constant__ parameter so
// the TMA unit reads the maps from parameter space.
struct TcParams {
  CUtensorMap ta[kMaxClassesPerLaunch];    // A operand, K-major 64 x 128 boxes
  CUtensorMap ta_t[kMaxClassesPerLaunch];  // A operand mirror blocks, 64 x 64 boxes
  CUtensorMap tb[kMaxClassesPerLaunch];    // B operand (APPLY: X, 64 x 64 boxes)
  CUtensorMap tb_t[kMaxClassesPerLaunch];  // B operand mirror blocks (POLY), 64 x 64 boxes
  CUtensorMap tc[kMaxClassesPerLaunch];    // C tile of the epilogue (POLY: S)
  CUtensorMap td[kMaxClassesPerLaunch];    // output (GRAM: S, POLY: P', APPLY: X'), 64 x 128
  NsPhaseArgs args;
};
static_assert(sizeof(TcParams) <= 4096, "kernel parameters must fit the portable 4 KB");

// Tile sizes of the tensor-core phases (rows x cols of an output tile, k-block).
int tc_block_m();
int tc_block_n(int phase);
int tc_block_k();

cudaError_t launch_ns_phase_tc(const TcParams& P, int num_sms, cudaStream_t s);

// CTA-pair launch: 256 x 256 tiles (tiles_i = ceil(m/256), tiles_j = ceil(cols/256)),
// for classes whose m is a multiple of 256. Same tensor maps as the single-CTA launch.
cudaError_t launch_ns_phase_tc_pair(const TcParams& P, int num_sms, cudaStream_t s);
constexpr int kPairTile = 256;

bool encode_slab_map_bf16(CUtensorMap* out, const void* base, int64_t inner, int64_t rows,
                          int64_t count, int64_t ld, int box_inner, int box_rows);
// 4-D view of the same slab as [count][column chunk of 64][rows][64] (innermost
// first: 64 columns, rows, chunks, matrices) with a box of 64 rows x `box_chunks`
// chunks, 128B swizzle: one load brings a block in the MN-major operand layout
// (chunk after chunk). Columns past `inner` in its last chunk are the slab's padding
// and are read as stored; they only reach output rows / columns the stores clip.
bool encode_chunk_map_bf16(CUtensorMap* out, const void* base, int64_t inner, int64_t rows,
                           int64_t count, int64_t ld, int box_chunks);

}  // namespace muon
