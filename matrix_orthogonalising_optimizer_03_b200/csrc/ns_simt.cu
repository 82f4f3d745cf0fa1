// fp32 Newton-Schulz phases on the CUDA cores (the MUON_NS_FP32 path).
//
// The three contractions of one iteration, with fp32 storage and fp32 FMAs:
//   GRAM   S = alpha * X X^T            (upper tiles, mirrored on store)
//   POLY   P = b*S + c*S S              (upper tiles, mirrored)
//   APPLY  X' = gamma * (a*X + P X)
// alpha = 1/(||U||+eps)^2 and gamma = 1/(||U||+eps) on the first iteration (the
// slab then holds the unnormalised U), 1 afterwards. Recurrence: the Newton-Schulz
// listing of "LLM Pretraining Loss Spike 진단과 처방" (section "Muon head의 실체는
// 하이브리드 옵티마이저다") and section 2 of the "MUON IS SCALABLE FOR LLM TRAINING"
// review. Every output element is one fp32 dot product taken in k order, whatever
// the tile size, so both kernels below give the same bits.
//
// Two kernels share the tile routine:
//   ns_simt_kernel<PHASE>   one launch per phase over every matrix of the call;
//                           64x64 tiles, one per 256-thread block, 4x4 outputs per thread.
//   ns_simt_fused_kernel    small matrices (n <= 256): one cluster of 16 (or 8) blocks
//                           per matrix runs all iterations and phases in a single
//                           launch; 32x32 tiles (APPLY 32x64) from full-K
//                           operand panels in shared memory, dealt round-robin to the
//                           cluster's blocks, and a cluster barrier between phases, so a
//                           step costs one launch instead of 3 per iteration.
#include <cuda_runtime.h>

#include <atomic>

#include "muon_internal.h"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int KS = 16, NT = 256;
constexpr int kClusterCtas = 8;  // blocks per matrix in the fused kernel (portable cluster)

// Output tile (ti, tj) of one phase for one matrix: C[i0.., j0..] (+)= A B, TT x TT,
// k-step KS, 256 threads with (TT/16)^2 outputs each; the epilogue applies the phase.
// A is [i][k] row-major; B is [j][k] (GRAM) or [k][j] (POLY, APPLY). Symmetric phases
// also store the mirror of an off-diagonal tile.
template <int PHASE, int TT>
__device__ __forceinline__ void simt_tile(const float* A, int lda, const float* B, int ldb, int m,
                                          int ncols, int K, int ti, int tj, float* out, int ldo,
                                          const float* cin, float scale, float pa, float pb,
                                          float pc, float (*As)[64 + 4], float (*Bs)[64 + 4]) {
  constexpr bool SYM = PHASE != PH_APPLY;
  constexpr int R = TT / 16;  // outputs per thread along each side
  const int i0 = ti * TT, j0 = tj * TT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[R][R];
#pragma unroll
  for (int x = 0; x < R; ++x)
#pragma unroll
    for (int y = 0; y < R; ++y) acc[x][y] = 0.f;

  for (int k0 = 0; k0 < K; k0 += KS) {
    {  // A tile: TT rows x KS, R values per thread
      const int row = threadIdx.x / (KS / R), kk = (threadIdx.x % (KS / R)) * R;
#pragma unroll
      for (int e = 0; e < R; ++e) {
        const int gi = i0 + row, gk = k0 + kk + e;
        As[kk + e][row] = (gi < m && gk < K) ? A[(int64_t)gi * lda + gk] : 0.f;
      }
    }
    if (PHASE == PH_GRAM) {  // B[j][k] = X[j0+j][k0+k]
      const int row = threadIdx.x / (KS / R), kk = (threadIdx.x % (KS / R)) * R;
#pragma unroll
      for (int e = 0; e < R; ++e) {
        const int gj = j0 + row, gk = k0 + kk + e;
        Bs[kk + e][row] = (gj < ncols && gk < K) ? B[(int64_t)gj * ldb + gk] : 0.f;
      }
    } else {  // B[k][j] row-major
      const int kk = threadIdx.x >> 4, col = (threadIdx.x & 15) * R;
#pragma unroll
      for (int e = 0; e < R; ++e) {
        const int gk = k0 + kk, gj = j0 + col + e;
        Bs[kk][col + e] = (gk < K && gj < ncols) ? B[(int64_t)gk * ldb + gj] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      float av[R], bv[R];
#pragma unroll
      for (int e = 0; e < R; ++e) {
        av[e] = As[kk][ty * R + e];
        bv[e] = Bs[kk][tx * R + e];
      }
#pragma unroll
      for (int x = 0; x < R; ++x)
#pragma unroll
        for (int y = 0; y < R; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int x = 0; x < R; ++x) {
    const int i = i0 + ty * R + x;
    if (i >= m) continue;
#pragma unroll
    for (int y = 0; y < R; ++y) {
      const int j = j0 + tx * R + y;
      if (j >= ncols) continue;
      float v;
      if (PHASE == PH_GRAM) v = scale * acc[x][y];
      else if (PHASE == PH_POLY) v = fmaf(pb, cin[(int64_t)i * ldo + j], pc * acc[x][y]);
      else v = scale * fmaf(pa, cin[(int64_t)i * ldo + j], acc[x][y]);
      out[(int64_t)i * ldo + j] = v;
      if (SYM && ti != tj) out[(int64_t)j * ldo + i] = v;
    }
  }
}

// Runs output tile t of a phase of matrix `mat` of class k (tiles_i x tiles_j grid of
// TT tiles; upper triangle for the symmetric phases), reading X from x_in and writing
// X' to x_out (APPLY).
template <int PHASE, int TT>
__device__ __forceinline__ void simt_phase_tile(const NsClassArgs& k, int mat, int t,
                                                const void* x_in, void* x_out, float scale,
                                                float pa, float pb, float pc,
                                                float (*As)[64 + 4], float (*Bs)[64 + 4]) {
  constexpr bool SYM = PHASE != PH_APPLY;
  const int tiles_i = (k.m + TT - 1) / TT;
  int ti, tj;
  if (SYM) {
    int rem = t;
    ti = 0;
    while (rem >= tiles_i - ti) { rem -= tiles_i - ti; ++ti; }
    tj = ti + rem;
  } else {
    const int tiles_j = (k.n + TT - 1) / TT;
    ti = t / tiles_j;
    tj = t - ti * tiles_j;
  }
  const float* X = static_cast<const float*>(x_in) + mat * k.xstride;
  float* S = static_cast<float*>(k.s) + mat * k.sstride;
  float* Pm = static_cast<float*>(k.p) + mat * k.sstride;
  if (PHASE == PH_GRAM)
    simt_tile<PH_GRAM, TT>(X, k.ldx, X, k.ldx, k.m, k.m, k.n, ti, tj, S, k.lds, nullptr, scale,
                           pa, pb, pc, As, Bs);
  else if (PHASE == PH_POLY)
    simt_tile<PH_POLY, TT>(S, k.lds, S, k.lds, k.m, k.m, k.m, ti, tj, Pm, k.lds, S, 1.f, pa, pb,
                           pc, As, Bs);
  else
    simt_tile<PH_APPLY, TT>(Pm, k.lds, X, k.ldx, k.m, k.n, k.m, ti, tj,
                            static_cast<float*>(x_out) + mat * k.xstride, k.ldx, X, scale, pa,
                            pb, pc, As, Bs);
}

__device__ __forceinline__ float first_iter_scale(const MatScalars* scal, int idx, float eps,
                                                  int phase) {
  const double inv = 1.0 / (sqrt(scal[idx].u2) + (double)eps);
  return static_cast<float>(phase == PH_GRAM ? inv * inv : (phase == PH_APPLY ? inv : 1.0));
}

template <int PHASE>
__global__ void __launch_bounds__(NT) ns_simt_kernel(const NsPhaseArgs p) {
  constexpr bool SYM = PHASE != PH_APPLY;
  __shared__ float As[KS][64 + 4];
  __shared__ float Bs[KS][64 + 4];
  const int t = blockIdx.x;
  int c = 0;
  while (c + 1 < p.num_classes && t >= p.tile_base[c + 1]) ++c;
  const NsClassArgs& k = p.cls[c];
  const int u = t - p.tile_base[c];
  const int mat = u / k.tiles_per_mat;
  const float scale = p.first_iter ? first_iter_scale(p.scal, k.first + mat, p.eps, PHASE) : 1.f;
  (void)SYM;
  simt_phase_tile<PHASE, 64>(k, mat, u - mat * k.tiles_per_mat, k.x_in, k.x_out, scale, p.a, p.b,
                             p.c, As, Bs);
}

// Release this block's global stores and wait for every block of the cluster. Every
// reader of a phase's output is a thread of the same cluster, so the barrier's release /
// acquire at cluster scope orders the stores for them (no device-scope fence).
__device__ __forceinline__ void cluster_phase_barrier() {
  cluster_sync_all();
}

// Fused kernel tile: a 32 x 32 (GRAM, POLY) or 32 x 64 (APPLY) output tile computed from
// full-K operand panels staged in shared memory by one round of loads (K <= kFusedMaxK),
// so that the tile pays the L2 latency once instead of once per k-step. 128 threads
// compute, each a 4 x 2 (GRAM, POLY) or 4 x 4 (APPLY) block of outputs from 16-byte
// reads of both panels along k (4 k-steps per read), each output one fp32 dot product
// in k order.
//   As[i][k] = A[i0 + i][k]                      (row stride kFusedStride)
//   GRAM / POLY: Bs[j][k] = B[j0 + j][k]         (B is X, or S, which is symmetric)
//   APPLY:       Bs[k][j] = X[k][j0 + j]          (row stride 64)
// kFusedStride is a multiple of 4 (16-byte rows) whose rows are 16 bytes apart modulo
// 128: the reads of 8 consecutive rows at one k fall in different banks.
constexpr int kFusedMaxK = 256;
constexpr int kFusedStride = kFusedMaxK + 4;
constexpr int kApplyTN = 64;                  // APPLY tile columns
constexpr int kFusedMathThreads = 128;
static_assert((kFusedStride * 4) % 128 == 16, "panel rows 16 bytes apart modulo 128");

template <int PHASE>
__device__ __forceinline__ void fused_tile(const NsClassArgs& k, int mat, int t, const float* X,
                                           float* Xout, float scale, float pa, float pb, float pc,
                                           float* As, float* Bs) {
  constexpr bool SYM = PHASE != PH_APPLY;
  constexpr int TT = 32;
  const int m = k.m;
  const int tiles_i = (m + TT - 1) / TT;
  int ti, tj;
  if (SYM) {
    int rem = t;
    ti = 0;
    while (rem >= tiles_i - ti) { rem -= tiles_i - ti; ++ti; }
    tj = ti + rem;
  } else {
    const int tiles_j = (k.n + kApplyTN - 1) / kApplyTN;
    ti = t / tiles_j;
    tj = t - ti * tiles_j;
  }
  const float* S = static_cast<const float*>(k.s) + mat * k.sstride;
  float* Sw = static_cast<float*>(k.s) + mat * k.sstride;
  float* Pm = static_cast<float*>(k.p) + mat * k.sstride;
  const float* A;
  int lda, K, ncols;
  if (PHASE == PH_GRAM) { A = X; lda = k.ldx; K = k.n; ncols = m; }
  else if (PHASE == PH_POLY) { A = S; lda = k.lds; K = m; ncols = m; }
  else { A = Pm; lda = k.lds; K = m; ncols = k.n; }
  const int i0 = ti * TT, j0 = tj * (PHASE == PH_APPLY ? kApplyTN : TT);
  // panels: every load of the tile is issued before any shared-memory store (16-byte
  // loads; warp w takes rows w, w + 8, w + 16, w + 24, lanes along k). Rows start on
  // 256-byte boundaries (slab leading dimensions are multiples of 64); values past K
  // (slab padding) and rows outside the matrix are stored as 0.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  {
    const float* Bsrc = PHASE == PH_GRAM ? X : S;
    const int ldb = PHASE == PH_GRAM ? k.ldx : k.lds;
    float4 va[4][2], vb[4][2];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = warp + 8 * q;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int kk = 4 * (lane + 32 * h);
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        va[q][h] = (i0 + r < m && kk < K)
                       ? *reinterpret_cast<const float4*>(A + (int64_t)(i0 + r) * lda + kk) : z;
        vb[q][h] = (PHASE != PH_APPLY && j0 + r < ncols && kk < K)
                       ? *reinterpret_cast<const float4*>(Bsrc + (int64_t)(j0 + r) * ldb + kk) : z;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = warp + 8 * q;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int kk = 4 * (lane + 32 * h);
        if (kk >= K) continue;
        const float av[4] = {va[q][h].x, va[q][h].y, va[q][h].z, va[q][h].w};
        const float bv[4] = {vb[q][h].x, vb[q][h].y, vb[q][h].z, vb[q][h].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          As[r * kFusedStride + kk + e] = kk + e < K ? av[e] : 0.f;
          if (PHASE != PH_APPLY) Bs[r * kFusedStride + kk + e] = kk + e < K ? bv[e] : 0.f;
        }
      }
    }
  }
  if (PHASE == PH_APPLY) {  // Bs[k][j] = X[k][j0 + j]: K rows of 64, 8 loads in flight
    const int gj = j0 + 2 * lane;  // two columns per lane (8-byte loads; ldx and j0 are even)
    for (int kb = warp; kb < K; kb += 8 * (NT / 32)) {
      float2 v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int kk = kb + q * (NT / 32);
        const float* src = X + (int64_t)kk * k.ldx + gj;
        v[q] = make_float2(0.f, 0.f);
        if (kk < K && gj + 1 < ncols) v[q] = *reinterpret_cast<const float2*>(src);
        else if (kk < K && gj < ncols) v[q].x = src[0];
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int kk = kb + q * (NT / 32);
        if (kk < K) *reinterpret_cast<float2*>(Bs + kk * kApplyTN + 2 * lane) = v[q];
      }
    }
    // rows K .. K rounded up to 4 are read (times a zero of A): keep them finite
    for (int kk = K + warp; kk < ((K + 3) & ~3); kk += NT / 32)
      *reinterpret_cast<float2*>(Bs + kk * kApplyTN + 2 * lane) = make_float2(0.f, 0.f);
  }
  __syncthreads();
  if (threadIdx.x < kFusedMathThreads) {
    // rows ty + 8i (i < 4); columns tx + 16j (j < 2: GRAM, POLY) or 4tx .. 4tx + 3 (APPLY)
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    constexpr int NY = PHASE == PH_APPLY ? 4 : 2;
    const int K4 = (K + 3) & ~3;  // panel entries past K are 0 in A (and finite in B)
    float acc[4][NY];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < NY; ++y) acc[x][y] = 0.f;
    for (int kk = 0; kk < K4; kk += 4) {
      float av[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float4 q = *reinterpret_cast<const float4*>(As + (ty + 8 * x) * kFusedStride + kk);
        av[x][0] = q.x; av[x][1] = q.y; av[x][2] = q.z; av[x][3] = q.w;
      }
      float bv[4][NY];  // [k offset][column]
      if (PHASE == PH_APPLY) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 q = *reinterpret_cast<const float4*>(Bs + (kk + e) * kApplyTN + 4 * tx);
          bv[e][0] = q.x; bv[e][1] = q.y;
          bv[e][NY > 2 ? 2 : 0] = q.z; bv[e][NY > 3 ? 3 : 0] = q.w;
        }
      } else {
#pragma unroll
        for (int y = 0; y < NY; ++y) {
          const float4 q = *reinterpret_cast<const float4*>(Bs + (tx + 16 * y) * kFusedStride + kk);
          bv[0][y] = q.x; bv[1][y] = q.y; bv[2][y] = q.z; bv[3][y] = q.w;
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)  // k order
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < NY; ++y) acc[x][y] = fmaf(av[x][e], bv[e][y], acc[x][y]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int i = i0 + ty + 8 * x;
      if (i >= m) continue;
#pragma unroll
      for (int y = 0; y < NY; ++y) {
        const int j = j0 + (PHASE == PH_APPLY ? 4 * tx + y : tx + 16 * y);
        if (j >= ncols) continue;
        if (PHASE == PH_GRAM) {
          const float v = scale * acc[x][y];
          Sw[(int64_t)i * k.lds + j] = v;
          if (ti != tj) Sw[(int64_t)j * k.lds + i] = v;
        } else if (PHASE == PH_POLY) {
          const float v = fmaf(pb, S[(int64_t)i * k.lds + j], pc * acc[x][y]);
          Pm[(int64_t)i * k.lds + j] = v;
          if (ti != tj) Pm[(int64_t)j * k.lds + i] = v;
        } else {
          Xout[(int64_t)i * k.ldx + j] = scale * fmaf(pa, X[(int64_t)i * k.ldx + j], acc[x][y]);
        }
      }
    }
  }
  __syncthreads();  // the panels are reused by the next tile
}

// All iterations of one small matrix per cluster of `kFusedCtas` blocks.
__global__ void __launch_bounds__(NT) ns_simt_fused_kernel(const NsFusedArgs a) {
  extern __shared__ float fsm[];
  float* As = fsm;
  float* Bs = fsm + 32 * kFusedStride;
  const int csize = static_cast<int>(cluster_num_ctas());
  const int crank = static_cast<int>(cluster_cta_rank());
  const int gm = static_cast<int>(blockIdx.x) / csize;  // matrix of this cluster
  int c = 0;
  while (c + 1 < a.num_classes && gm >= a.mat_base[c + 1]) ++c;
  const NsClassArgs& k = a.cls[c];
  const int mat = gm - a.mat_base[c];
  const int ti = (k.m + 31) / 32;
  const int sym_tiles = ti * (ti + 1) / 2;
  const int apply_tiles = ti * ((k.n + kApplyTN - 1) / kApplyTN);
  for (int it = 0; it < a.steps; ++it) {
    const float* x_in = static_cast<const float*>((it & 1) ? a.x1[c] : a.x0[c]) + mat * k.xstride;
    float* x_out = static_cast<float*>((it & 1) ? a.x0[c] : a.x1[c]) + mat * k.xstride;
    const bool first = it == 0;
    const float sg = first ? first_iter_scale(a.scal, k.first + mat, a.eps, PH_GRAM) : 1.f;
    const float sa = first ? first_iter_scale(a.scal, k.first + mat, a.eps, PH_APPLY) : 1.f;
    for (int t = crank; t < sym_tiles; t += csize)
      fused_tile<PH_GRAM>(k, mat, t, x_in, x_out, sg, a.a, a.b, a.c, As, Bs);
    cluster_phase_barrier();
    for (int t = crank; t < sym_tiles; t += csize)
      fused_tile<PH_POLY>(k, mat, t, x_in, x_out, 1.f, a.a, a.b, a.c, As, Bs);
    cluster_phase_barrier();
    for (int t = crank; t < apply_tiles; t += csize)
      fused_tile<PH_APPLY>(k, mat, t, x_in, x_out, sa, a.a, a.b, a.c, As, Bs);
    cluster_phase_barrier();
  }
}

// As (32 rows) and the larger of the two B layouts: 32 rows of K, or K rows of 64
constexpr size_t kFusedSmem =
    sizeof(float) * (32 * kFusedStride + (32 * kFusedStride > kFusedMaxK * kApplyTN
                                              ? 32 * kFusedStride
                                              : kFusedMaxK * kApplyTN));

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

bool simt_fused_fits(int m, int n) {
  // oriented shape (m <= n): every contraction has K <= n
  return m <= n && n <= kFusedMaxK;
}

// One cluster per matrix: 16 blocks where the device allows that (non-portable size),
// else 8. Attributes are set once per device.
cudaError_t launch_ns_simt_fused(const NsFusedArgs& a, cudaStream_t s) {
  const int total = a.mat_base[a.num_classes];
  if (total <= 0 || a.steps <= 0) return cudaSuccess;
  static std::atomic<uint64_t> ready{0}, wide{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit == 0 || !(ready.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(ns_simt_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kFusedSmem));
    if (e != cudaSuccess) return e;
    if (cudaFuncSetAttribute(ns_simt_fused_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1) == cudaSuccess)
      wide.fetch_or(bit, std::memory_order_acq_rel);
    else
      cudaGetLastError();
    ready.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int csize = (wide.load(std::memory_order_acquire) & bit) ? 16 : kClusterCtas;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(total * csize), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = kFusedSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, ns_simt_fused_kernel, a);
}

}  // namespace muon
