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

// Symmetric phases (GRAM, POLY) of single-CTA classes: the m x m output is stored as its
// 128 x 128 blocks on or above the block diagonal. Row block i (rows 128 i ..) is cut into
// column pieces from column 128 i to m, each at most 256 wide and a multiple of 64, of
// nearly equal width; a tile is one (row block, piece) pair and the MMA N is the piece
// width. The host counts tiles and the kernel decodes them with these same functions.
__host__ __device__ inline int sym_row_blocks(int m) { return (m + 127) / 128; }
__host__ __device__ inline int sym_pieces(int m, int i) { return (m - 128 * i + 255) / 256; }
__host__ __device__ inline int sym_piece_width(int m, int i) {
  const int len = m - 128 * i, np = (len + 255) / 256;
  return ((len + np - 1) / np + 63) / 64 * 64;
}
// Column start and width (a multiple of 64; the last piece may reach past m, where the
// stores are clipped) of piece j of row block i.
__host__ __device__ inline void sym_piece(int m, int i, int j, int* col0, int* width) {
  const int w = sym_piece_width(m, i);
  const int c0 = 128 * i + j * w;
  const int rest = (m - c0 + 63) / 64 * 64;
  *col0 = c0;
  *width = w < rest ? w : rest;
}
__host__ __device__ inline int sym_tiles_per_matrix(int m) {
  int t = 0;
  for (int i = 0; i < sym_row_blocks(m); ++i) t += sym_pieces(m, i);
  return t;
}

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
