// Arguments and launchers of the memory-bound kernels of libmuon (elementwise.cu).
#pragma once
#include <cstdint>

#include <cuda_runtime.h>

#include "muon_internal.h"

namespace muon {

constexpr int kOTileR = 64;   // O-only reduction: slab rows per block
constexpr int kOTileC = 256;  // O-only reduction: slab columns per tile of the walk
constexpr int kOMinBlocks = 1024;  // fewer bands than this: split each band's walk

// Sums post_apply accumulates for the statistics of Muon and the two-sided mode.
struct ApplySums {
  double w2;   // ||W_t||_F^2
  double wo;   // <W_t, D O_raw>_F (D the equilibration scaling, identity when off)
  double o2;   // ||D O_raw||_F^2
  double pad;
};

// Arguments of the memory-bound kernels.
struct ElemArgs {
  const DevMat* mats;
  const DevSlab* slabs;
  const int32_t* tile_prefix;  // n+1 entries: first elementwise tile of each matrix
  int32_t n;
  int32_t total_tiles;
  MatScalars* scal;
  MatCoef* coef;
  float* eq_o2;     // per-row / per-column sums of O^2 (then equilibration factors)
  float* eq_wo;     // per-row / per-column sums of W*O
  muon_stats_t* stats;
  uint32_t* err;
  float mu;
  float lr, wd, eps, scale_k;
  int32_t scale_rule;
  int32_t mode;
  int32_t nesterov;
  int32_t ns_only;      // X in / O out instead of the optimizer step
  int32_t x_fp32;       // slabs hold fp32 (else bf16)
  int32_t equilibrate;
  int32_t xs_from_u2;   // ns_steps == 0: the slab holds U, scale it by 1/(||U||+eps)
  int32_t sub_r, sub_c; // super-tile = sub_r x sub_c sub-tiles of 32 x 64 (1..4 each)
  int32_t staged;       // plain reduction through a shared-memory ring (aligned W rows, bf16 slab)
  int32_t staged_in;    // ingest through the ring (also bf16 G with rows of 16-byte multiples)
  // Muon and two-sided modes: the update needs no W-dependent scalar, so the reduction
  // reads the slab alone (post_reduce_o_kernel, bands of kOTileR slab rows walked in
  // kOTileC-column tiles) and post_apply accumulates the statistics' W sums
  int32_t w_free;
  int32_t apply_stats;  // w_free and statistics requested
  const int32_t* o_tile_prefix;  // n+1 entries: first O-only reduction band of each matrix
  int32_t o_total_tiles;
  ApplySums* asum;      // n entries, zeroed with the per-matrix scalars
};

cudaError_t launch_ingest(const ElemArgs& a, cudaStream_t s);
cudaError_t launch_post_reduce(const ElemArgs& a, cudaStream_t s);
cudaError_t launch_post_finalize(const ElemArgs& a, cudaStream_t s);
cudaError_t launch_post_apply(const ElemArgs& a, cudaStream_t s);
cudaError_t launch_post_stats(const ElemArgs& a, cudaStream_t s);

}  // namespace muon
