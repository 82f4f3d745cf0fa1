// Internal layout shared by the host plan and the kernels of libmuon.
#pragma once
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "muon.h"

namespace muon {

// Descriptor of one matrix as the elementwise kernels see it (stored in the
// workspace, in plan order: grouped by shape class).
enum : int32_t { MAT_TRANSPOSED = 1, MAT_G_BF16 = 2, MAT_VEC_OK = 4 };

struct DevMat {
  float* W;
  const void* G;
  float* M;
  int64_t ld_w, ld_g, ld_m;
  int32_t rows, cols;   // storage shape
  int32_t flags;
  int32_t orig;         // index in the caller's list (stats slot)
};
static_assert(sizeof(DevMat) == 64, "DevMat is 64 bytes");

// Per-matrix scalars accumulated on the device.
struct MatScalars {
  double u2;    // ||U||_F^2
  double w2;    // ||W_t||_F^2
  double wo;    // <W_t, O_raw>_F (O_raw = Newton-Schulz output, before a6/a7)
  double o2;    // ||O_raw||_F^2
};
static_assert(sizeof(MatScalars) == 32, "MatScalars is 32 bytes");

// Final per-matrix coefficients of the update W <- cw*W + co*D*O_raw, where D
// is the equilibration scaling (identity when off).
struct MatCoef {
  float cw, co;
  int32_t axis;   // 0 none, 1 rows, 2 columns (storage frame)
  int32_t pad;
};

// One shape class: all matrices with the same oriented shape m x n (m <= n).
// Their Newton-Schulz operands live in contiguous slabs [count][m][ld].
struct ClassInfo {
  int32_t m, n;        // oriented shape
  int32_t count;       // matrices in the class
  int32_t first;       // first plan index of the class
  int32_t ldx, lds;    // slab leading dimensions (elements), multiples of 64
  int64_t xbytes, sbytes;  // bytes of one matrix in the X / S slabs
  int64_t off_x[2], off_s, off_p;  // workspace byte offsets of the slabs
};

constexpr int kMaxClassesPerLaunch = 4;
constexpr int kElemTileR = 128;  // largest elementwise super-tile: rows (storage frame)
constexpr int kElemTileC = 256;  // largest elementwise super-tile: cols
constexpr int kElemSubR = 32;    // elementwise sub-tile: rows
constexpr int kElemSubC = 64;    // elementwise sub-tile: cols
// Small steps (at most this many elements over all matrices) use one-sub-tile
// super-tiles, so that more blocks share the work; larger ones use 128 x 256.
constexpr int64_t kElemSmallStep = int64_t(1) << 22;

// Workspace header: the sticky device error word and a step counter.
struct WsHeader {
  uint32_t error;
  uint32_t pad[63];
};

// Bounded spin-waits give up after this many SM clock cycles (about 1 s).
constexpr long long kWaitLimitCycles = 2000000000LL;

}  // namespace muon

namespace muon {

// Where one matrix's Newton-Schulz operand lives (plan order).
struct DevSlab {
  void* x0;        // slab entry written by the ingest kernel
  void* xf;        // slab entry holding the Newton-Schulz result
  int64_t eq_off;  // offset (floats) of this matrix's rows+cols vectors in the eq arrays
  int32_t ldx;     // leading dimension of the slab entry (elements)
  int32_t cls;     // shape class
};
static_assert(sizeof(DevSlab) == 32, "DevSlab is 32 bytes");



}  // namespace muon

namespace muon {

enum NsPhase : int32_t { PH_GRAM = 0, PH_POLY = 1, PH_APPLY = 2 };

// One shape class as a Newton-Schulz phase sees it.
struct NsClassArgs {
  int32_t m, n;            // oriented shape, m <= n
  int32_t count, first;    // matrices, first plan index
  int32_t ldx, lds;        // slab leading dimensions (elements)
  int32_t tiles_i, tiles_j;  // output tile grid of one matrix
  int32_t tiles_per_mat;   // symmetric phases: T(T+1)/2, apply: tiles_i*tiles_j
  int32_t k_blocks;        // reduction blocks (tensor-core path)
  int64_t xstride, sstride;  // elements of one matrix in the X / S slabs
  const void* x_in;        // X_k slab
  void* x_out;             // X_{k+1} slab (apply)
  void* s;                 // S slab
  void* p;                 // P slab
};

struct NsPhaseArgs {
  NsClassArgs cls[kMaxClassesPerLaunch];
  int32_t tile_base[kMaxClassesPerLaunch + 1];
  int32_t num_classes;
  int32_t phase;
  float a, b, c;           // Newton-Schulz coefficients
  int32_t first_iter;      // fold 1/(||U||+eps) into this iteration
  float eps;
  const MatScalars* scal;
  uint32_t* err;
};

cudaError_t launch_ns_phase_simt(const NsPhaseArgs& a, cudaStream_t s);

// All iterations of the fp32 Newton-Schulz of small matrices in one launch (one
// cluster of 16, or 8, blocks per matrix). cls[c] describes class c; x0 / x1 are its two X slabs
// (the iteration reads x0 on even and x1 on odd iterations); mat_base[c] is the first
// launch-local matrix of class c.
struct NsFusedArgs {
  NsClassArgs cls[kMaxClassesPerLaunch];
  void* x0[kMaxClassesPerLaunch];
  void* x1[kMaxClassesPerLaunch];
  int32_t mat_base[kMaxClassesPerLaunch + 1];
  int32_t num_classes;
  int32_t steps;
  float a, b, c;
  float eps;
  const MatScalars* scal;
};
// Whether a class of the fp32 path (oriented m x n, m <= n) takes the fused kernel:
// n <= 256, so that a tile's full-K operand panels fit in shared memory.
bool simt_fused_fits(int m, int n);
cudaError_t launch_ns_simt_fused(const NsFusedArgs& a, cudaStream_t s);

}  // namespace muon
