// fp32 Newton-Schulz phases on the CUDA cores (the MUON_NS_FP32 path).
//
// One launch per phase over every matrix of every shape class in the call:
//   GRAM   S = alpha * X X^T            (upper 64x64 tiles, mirrored on store)
//   POLY   P = b*S + c*S S              (upper tiles, mirrored)
//   APPLY  X' = gamma * (a*X + P X)
// alpha = 1/(||U||+eps)^2 and gamma = 1/(||U||+eps) on the first iteration (the
// slab then holds the unnormalised U), 1 afterwards. Recurrence: the Newton-Schulz
// listing of "LLM Pretraining Loss Spike 진단과 처방" (section "Muon head의 실체는
// 하이브리드 옵티마이저다") and section 2 of the "MUON IS SCALABLE FOR LLM TRAINING"
// review. 64x64 tile per 256-thread block, 4x4 outputs per thread, k-step 16.
#include <cuda_runtime.h>

#include "muon_internal.h"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int T = 64, KS = 16, NT = 256;

struct TileJob {
  int c, mat, ti, tj;
};

__device__ __forceinline__ TileJob decode(const NsPhaseArgs& p, int t, bool sym) {
  int c = 0;
  while (c + 1 < p.num_classes && t >= p.tile_base[c + 1]) ++c;
  const NsClassArgs& k = p.cls[c];
  const int u = t - p.tile_base[c];
  TileJob j;
  j.c = c;
  j.mat = u / k.tiles_per_mat;
  int rem = u - j.mat * k.tiles_per_mat;
  if (sym) {
    int ti = 0;
    while (rem >= k.tiles_i - ti) { rem -= k.tiles_i - ti; ++ti; }
    j.ti = ti;
    j.tj = ti + rem;
  } else {
    j.ti = rem / k.tiles_j;
    j.tj = rem - j.ti * k.tiles_j;
  }
  return j;
}

template <int PHASE>
__global__ void __launch_bounds__(NT) ns_simt_kernel(const NsPhaseArgs p) {
  constexpr bool SYM = PHASE != PH_APPLY;
  __shared__ float As[KS][T + 4];
  __shared__ float Bs[KS][T + 4];
  const TileJob job = decode(p, blockIdx.x, SYM);
  const NsClassArgs& k = p.cls[job.c];
  const int m = k.m;
  const int ncols = PHASE == PH_APPLY ? k.n : m;         // output columns
  const int K = PHASE == PH_GRAM ? k.n : m;              // reduction length
  const float* A;  // [i][kk], row-major
  const float* B;  // GRAM: [j][kk]; POLY/APPLY: [kk][j]
  int lda, ldb;
  if (PHASE == PH_GRAM) {
    A = static_cast<const float*>(k.x_in) + job.mat * k.xstride;
    B = A;
    lda = ldb = k.ldx;
  } else if (PHASE == PH_POLY) {
    A = static_cast<const float*>(k.s) + job.mat * k.sstride;
    B = A;
    lda = ldb = k.lds;
  } else {
    A = static_cast<const float*>(k.p) + job.mat * k.sstride;
    B = static_cast<const float*>(k.x_in) + job.mat * k.xstride;
    lda = k.lds;
    ldb = k.ldx;
  }
  const int i0 = job.ti * T, j0 = job.tj * T;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};

  for (int k0 = 0; k0 < K; k0 += KS) {
    {  // A tile: 64 rows x 16
      const int row = threadIdx.x >> 2, kk = (threadIdx.x & 3) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gi = i0 + row, gk = k0 + kk + e;
        As[kk + e][row] = (gi < m && gk < K) ? A[(int64_t)gi * lda + gk] : 0.f;
      }
    }
    if (PHASE == PH_GRAM) {  // B[j][k] = X[j0+j][k0+k]
      const int row = threadIdx.x >> 2, kk = (threadIdx.x & 3) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gj = j0 + row, gk = k0 + kk + e;
        Bs[kk + e][row] = (gj < ncols && gk < K) ? B[(int64_t)gj * ldb + gk] : 0.f;
      }
    } else {  // B[k][j] row-major
      const int kk = threadIdx.x >> 4, col = (threadIdx.x & 15) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gk = k0 + kk, gj = j0 + col + e;
        Bs[kk][col + e] = (gk < K && gj < ncols) ? B[(int64_t)gk * ldb + gj] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        av[e] = As[kk][ty * 4 + e];
        bv[e] = Bs[kk][tx * 4 + e];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    __syncthreads();
  }

  float scale = 1.f;
  if (p.first_iter) {
    const double inv = 1.0 / (sqrt(p.scal[k.first + job.mat].u2) + (double)p.eps);
    scale = static_cast<float>(PHASE == PH_GRAM ? inv * inv : (PHASE == PH_APPLY ? inv : 1.0));
  }
  float* out;
  const float* cin = nullptr;
  int ldo;
  if (PHASE == PH_GRAM) {
    out = static_cast<float*>(k.s) + job.mat * k.sstride;
    ldo = k.lds;
  } else if (PHASE == PH_POLY) {
    out = static_cast<float*>(k.p) + job.mat * k.sstride;
    cin = static_cast<const float*>(k.s) + job.mat * k.sstride;
    ldo = k.lds;
  } else {
    out = static_cast<float*>(k.x_out) + job.mat * k.xstride;
    cin = static_cast<const float*>(k.x_in) + job.mat * k.xstride;
    ldo = k.ldx;
  }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int i = i0 + ty * 4 + x;
    if (i >= m) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int j = j0 + tx * 4 + y;
      if (j >= ncols) continue;
      float v;
      if (PHASE == PH_GRAM) v = scale * acc[x][y];
      else if (PHASE == PH_POLY) v = fmaf(p.b, cin[(int64_t)i * ldo + j], p.c * acc[x][y]);
      else v = scale * fmaf(p.a, cin[(int64_t)i * ldo + j], acc[x][y]);
      out[(int64_t)i * ldo + j] = v;
      if (SYM && job.ti != job.tj) out[(int64_t)j * ldo + i] = v;
    }
  }
}

}  // namespace

cudaError_t launch_ns_phase_simt(const NsPhaseArgs& a, cudaStream_t s) {
  const int total = a.tile_base[a.num_classes];
  if (total <= 0) return cudaSuccess;
  switch (a.phase) {
    case PH_GRAM: ns_simt_kernel<PH_GRAM><<<total, NT, 0, s>>>(a); break;
    case PH_POLY: ns_simt_kernel<PH_POLY><<<total, NT, 0, s>>>(a); break;
    default: ns_simt_kernel<PH_APPLY><<<total, NT, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

}  // namespace muon
