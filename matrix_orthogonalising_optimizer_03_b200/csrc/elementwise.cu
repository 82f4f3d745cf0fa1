// Memory-bound kernels of the Muon step (CUDA cores, HBM bound).
//
//   ingest        a1 momentum M = mu*M + G, a2 Nesterov U = G + mu*M, ||U||_F^2,
//                 and U written to the Newton-Schulz slab in the oriented frame
//                 (transposed through shared memory for tall matrices).
//   post_reduce   ||W||^2, <W,O>, ||O||^2 (post_reduce_plain_kernel); with
//                 equilibration also per-row and per-column sums of O^2 and W*O in the
//                 storage frame (post_reduce_eq_kernel). Muon and the two-sided mode
//                 need no W-dependent scalar: ||O||^2 and the O^2 row / column sums
//                 from the slab alone (post_reduce_o_kernel).
//   post_finalize one block per matrix: equilibration axis and factors (a6),
//                 scale (a7), GS coefficient (a8), statistics, update coefficients.
//   post_apply    a9: W <- cw*W + co*D*O (or, Newton-Schulz only, O out); in Muon and
//                 the two-sided mode also the statistics' sums of W_t and D*O.
//   post_stats    statistics of Muon and the two-sided mode (one thread per matrix).
//
// Work unit: a 128 x 256 super-tile of the matrix in its storage frame per
// 256-thread block, walked as 4 x 4 sub-tiles of 32 x 64 (8 consecutive columns
// per thread, 128-bit accesses when aligned; the reductions and post_apply take two
// 32-row sub-tiles at a time, all their loads issued before any arithmetic). The
// super-tile of each block is found by binary search over a per-matrix tile prefix.
// With aligned rows, ingest, post_apply and (without equilibration) the W-and-O
// reduction instead stage their loads in shared memory with cp.async (the *_staged
// kernels). The slab-only reduction walks bands of 64 slab rows across the width
// (its own prefix of bands).
// Per-matrix sums use one atomic per block; the equilibration row / column sums are
// reduced inside the block (shuffles, and shared memory across warps for columns) and
// use one atomic per row and per column of the super-tile (of the band's tile, in the
// slab-only reduction).
#include <cuda_runtime.h>

#include <atomic>

#include "muon_internal.h"
#include "elementwise.h"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int kThreads = 256;
constexpr int kTR = 32;   // sub-tile rows
constexpr int kTC = 64;   // sub-tile cols
constexpr int kSubR = kElemTileR / kTR;  // at most 4 sub-tiles down a super-tile

__device__ __forceinline__ void load8_f32(const float* p, bool vec, int valid, float (&v)[8]) {
  if (vec && valid == 8) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p));
    const float4 y = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = e < valid ? p[e] : 0.f;
  }
}
__device__ __forceinline__ void store8_f32(float* p, bool vec, int valid, const float (&v)[8]) {
  if (vec && valid == 8) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (e < valid) p[e] = v[e];
  }
}
__device__ __forceinline__ void load8_bf16(const uint16_t* p, bool vec, int valid, float (&v)[8]) {
  if (vec && valid == 8) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __uint_as_float(w[e] << 16);
      v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = e < valid ? bf16_to_f32(p[e]) : 0.f;
  }
}
__device__ __forceinline__ void store8_bf16(uint16_t* p, bool vec, int valid, const float (&v)[8]) {
  if (vec && valid == 8) {
    uint4 x;
    x.x = pack_bf16x2(v[0], v[1]);
    x.y = pack_bf16x2(v[2], v[3]);
    x.z = pack_bf16x2(v[4], v[5]);
    x.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = x;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (e < valid) p[e] = f32_to_bf16(v[e]);
  }
}

// Reads 8 values of the slab entry (oriented frame) at (row, col..col+7).
__device__ __forceinline__ void load8_slab(const void* base, int x_fp32, int64_t off, int valid,
                                           float (&v)[8]) {
  if (x_fp32) load8_f32(static_cast<const float*>(base) + off, true, valid, v);
  else load8_bf16(static_cast<const uint16_t*>(base) + off, true, valid, v);
}
__device__ __forceinline__ void store8_slab(void* base, int x_fp32, int64_t off, int valid,
                                            const float (&v)[8]) {
  if (x_fp32) store8_f32(static_cast<float*>(base) + off, true, valid, v);
  else store8_bf16(static_cast<uint16_t*>(base) + off, true, valid, v);
}

template <int NV>
__device__ __forceinline__ void block_sum(double (&v)[NV], double (*sh)[kThreads / 32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    v[i] = warp_sum(v[i]);
    if (lane == 0) sh[i][warp] = v[i];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      double x = lane < kThreads / 32 ? sh[i][lane] : 0.0;
      v[i] = warp_sum(x);
    }
  }
}

__device__ __forceinline__ int find_matrix_in(const int32_t* prefix, int n, int b) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int find_matrix(const ElemArgs& a, int b) {
  return find_matrix_in(a.tile_prefix, a.n, b);
}

// ------------------------------------------------------------------ ingest
__device__ __forceinline__ float ingest_subtile(const ElemArgs& a, const DevMat& d, const DevSlab& s,
                                                int r0, int c0, float (*tile)[kTR + 1]) {
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  const int r = r0 + lr, c = c0 + lc;
  const bool vec = (d.flags & MAT_VEC_OK) != 0;
  const int valid = (r < d.rows) ? max(0, min(8, d.cols - c)) : 0;
  float u[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) u[e] = 0.f;
  if (valid > 0) {
    float g[8];
    if (d.flags & MAT_G_BF16)
      load8_bf16(static_cast<const uint16_t*>(d.G) + (int64_t)r * d.ld_g + c, vec, valid, g);
    else
      load8_f32(static_cast<const float*>(d.G) + (int64_t)r * d.ld_g + c, vec, valid, g);
    if (a.ns_only) {
#pragma unroll
      for (int e = 0; e < 8; ++e) u[e] = g[e];
    } else {
      float m[8];
      float* mp = d.M + (int64_t)r * d.ld_m + c;
      load8_f32(mp, vec, valid, m);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        m[e] = fmaf(a.mu, m[e], g[e]);                       // M_t = mu*M_{t-1} + G_t
        u[e] = a.nesterov ? fmaf(a.mu, m[e], g[e]) : m[e];  // U = G_t + mu*M_t
      }
      store8_f32(mp, vec, valid, m);
    }
  }
  float sq = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    // the slab holds U rounded to its storage type; ||U|| is taken of that value
    const float q = a.x_fp32 ? u[e] : bf16_to_f32(f32_to_bf16(u[e]));
    sq = fmaf(q, q, sq);
  }
  if (!(d.flags & MAT_TRANSPOSED)) {
    if (valid > 0) store8_slab(s.x0, a.x_fp32, (int64_t)r * s.ldx + c, valid, u);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) tile[lc + e][lr] = u[e];
    __syncthreads();
    const int sr = c0 + (threadIdx.x >> 2), sc = r0 + (threadIdx.x & 3) * 8;
    const int v2 = (sr < d.cols) ? max(0, min(8, d.rows - sc)) : 0;
    if (v2 > 0) {
      float w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = tile[threadIdx.x >> 2][(threadIdx.x & 3) * 8 + e];
      store8_slab(s.x0, a.x_fp32, (int64_t)sr * s.ldx + sc, v2, w);
    }
    __syncthreads();
  }
  return sq;
}

__global__ void __launch_bounds__(kThreads, 8) ingest_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float tile[kTC][kTR + 1];
  __shared__ double red[1][kThreads / 32];
  const int b = blockIdx.x;
  const int k = find_matrix(a, b);
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const int t = b - a.tile_prefix[k];
  const int sub_r = a.sub_r, sub_c = a.sub_c;  // 32-row / 64-column sub-tiles per super-tile
  const int tiles_c = (d.cols + sub_c * kTC - 1) / (sub_c * kTC);
  const int R0 = (t / tiles_c) * (sub_r * kTR), C0 = (t % tiles_c) * (sub_c * kTC);
  float sq = 0.f;
  for (int bi = 0; bi < sub_r && R0 + bi * kTR < d.rows; ++bi)
    for (int bj = 0; bj < sub_c && C0 + bj * kTC < d.cols; ++bj)
      sq += ingest_subtile(a, d, s, R0 + bi * kTR, C0 + bj * kTC, tile);
  double acc[1] = {sq};
  block_sum<1>(acc, red);
  if (threadIdx.x == 0) atomicAdd(&a.scal[k].u2, acc[0]);
}

__device__ __forceinline__ float slab_scale(const ElemArgs& a, int k) {
  if (!a.xs_from_u2) return 1.f;
  return static_cast<float>(1.0 / (sqrt(a.scal[k].u2) + (double)a.eps));
}

// ------------------------------------------------------------------ post_reduce (plain)
// Without equilibration only the three per-matrix sums are needed. For each 64-column
// band of the super-tile the block handles two 32-row sub-tiles at a time and issues
// all their loads (W and the slab, 96 bytes per thread) before any arithmetic; tall
// matrices transpose both slab tiles through shared memory with one barrier pair.
// The 1/(||U||+eps) slab scale multiplies the finished sums, not every element.
constexpr int kRedGroup = 2;  // sub-tile rows in flight per thread

template <bool XF32>
__global__ void __launch_bounds__(kThreads, 4) post_reduce_plain_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float tile[kRedGroup][kTC][kTR + 1];
  __shared__ double red[3][kThreads / 32];
  const int b = blockIdx.x;
  const int k = find_matrix(a, b);
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const int t = b - a.tile_prefix[k];
  const int sub_r = a.sub_r, sub_c = a.sub_c;  // 32-row / 64-column sub-tiles per super-tile
  const int tiles_c = (d.cols + sub_c * kTC - 1) / (sub_c * kTC);
  const int R0 = (t / tiles_c) * (sub_r * kTR), C0 = (t % tiles_c) * (sub_c * kTC);
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  const bool vec = (d.flags & MAT_VEC_OK) != 0;
  const bool tall = (d.flags & MAT_TRANSPOSED) != 0;
  float ww = 0.f, wo = 0.f, oo = 0.f;
  for (int bj = 0; bj < sub_c && C0 + bj * kTC < d.cols; ++bj) {
    const int c0 = C0 + bj * kTC;
    for (int g0 = 0; g0 < sub_r && R0 + g0 * kTR < d.rows; g0 += kRedGroup) {
      float w[kRedGroup][8], o[kRedGroup][8];
      // loads: W in the storage frame; the slab in the storage frame (wide) or as
      // 64 x 32 tiles of O^T (tall: slab rows = storage columns)
#pragma unroll
      for (int q = 0; q < kRedGroup; ++q) {
        const int r0 = R0 + (g0 + q) * kTR;
        const int r = r0 + lr, c = c0 + lc;
        const bool inq = g0 + q < sub_r;  // the group's second sub-tile may lie past the super-tile
        const int valid = (inq && r < d.rows) ? max(0, min(8, d.cols - c)) : 0;
        if (valid > 0) load8_f32(d.W + (int64_t)r * d.ld_w + c, vec, valid, w[q]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) w[q][e] = 0.f;
        }
        int64_t off;
        int v2;
        if (!tall) {
          off = (int64_t)r * s.ldx + c;
          v2 = valid;
        } else {
          const int sr = c0 + (threadIdx.x >> 2), sc = r0 + (threadIdx.x & 3) * 8;
          off = (int64_t)sr * s.ldx + sc;
          v2 = (inq && sr < d.cols) ? max(0, min(8, d.rows - sc)) : 0;
        }
        if (v2 > 0) load8_slab(s.xf, XF32, off, v2, o[q]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) o[q][e] = 0.f;
        }
      }
      if (tall) {  // block-uniform
#pragma unroll
        for (int q = 0; q < kRedGroup; ++q)
#pragma unroll
          for (int e = 0; e < 8; ++e) tile[q][threadIdx.x >> 2][(threadIdx.x & 3) * 8 + e] = o[q][e];
        __syncthreads();
#pragma unroll
        for (int q = 0; q < kRedGroup; ++q)
#pragma unroll
          for (int e = 0; e < 8; ++e) o[q][e] = tile[q][lc + e][lr];
        __syncthreads();  // the tiles are reused by the next group
      }
#pragma unroll
      for (int q = 0; q < kRedGroup; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) {  // elements outside the matrix are 0 on both sides
          ww = fmaf(w[q][e], w[q][e], ww);
          wo = fmaf(w[q][e], o[q][e], wo);
          oo = fmaf(o[q][e], o[q][e], oo);
        }
    }
  }
  const double xs = slab_scale(a, k);
  double acc[3] = {ww, wo * xs, oo * xs * xs};
  block_sum<3>(acc, red);
  if (threadIdx.x == 0) {
    atomicAdd(&a.scal[k].w2, acc[0]);
    atomicAdd(&a.scal[k].wo, acc[1]);
    atomicAdd(&a.scal[k].o2, acc[2]);
  }
}

// ------------------------------------------------------------------ post_reduce (equilibration)
// Equilibration and the two-sided mode: the three per-matrix sums plus the per-row and
// per-column sums of O^2 and W*O in the storage frame. Same walk and loads as the plain
// reduction (two 32-row sub-tiles in flight per thread). Each thread keeps the sums of
// its 8 columns over the band's rows and of its 4 rows over the super-tile in
// registers; a band's column sums are reduced across the 4 rows of a warp by shuffles
// and across the 8 warps through shared memory (double-buffered by band, one barrier
// per band); the row sums are reduced across the 8 lanes of a row by shuffles at the
// end. One atomic per row and per column of the super-tile. The slab scale multiplies
// the finished sums.
template <bool XF32>
__global__ void __launch_bounds__(kThreads, 3) post_reduce_eq_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float tile[kRedGroup][kTC][kTR + 1];
  __shared__ float colred[2][2][kThreads / 32][kTC];  // [band parity][sum][warp][column]
  __shared__ double red[3][kThreads / 32];
  const int b = blockIdx.x;
  const int k = find_matrix(a, b);
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const int t = b - a.tile_prefix[k];
  const int sub_r = a.sub_r, sub_c = a.sub_c;  // 32-row / 64-column sub-tiles per super-tile
  const int tiles_c = (d.cols + sub_c * kTC - 1) / (sub_c * kTC);
  const int R0 = (t / tiles_c) * (sub_r * kTR), C0 = (t % tiles_c) * (sub_c * kTC);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  const bool vec = (d.flags & MAT_VEC_OK) != 0;
  const bool tall = (d.flags & MAT_TRANSPOSED) != 0;
  const float xs = slab_scale(a, k);
  float ww = 0.f;
  float row_o2[kSubR], row_wo[kSubR];  // this thread's share of its (up to 4) rows' sums
#pragma unroll
  for (int i = 0; i < kSubR; ++i) row_o2[i] = row_wo[i] = 0.f;

  for (int bj = 0; bj < sub_c && C0 + bj * kTC < d.cols; ++bj) {  // uniform over the block
    const int c0 = C0 + bj * kTC;
    float col_o2[8], col_wo[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) col_o2[e] = col_wo[e] = 0.f;
#pragma unroll
    for (int g0 = 0; g0 < kSubR; g0 += kRedGroup) {
      if (g0 >= sub_r || R0 + g0 * kTR >= d.rows) break;  // uniform over the block
      float w[kRedGroup][8], o[kRedGroup][8];
#pragma unroll
      for (int q = 0; q < kRedGroup; ++q) {
        const int r0 = R0 + (g0 + q) * kTR;
        const int r = r0 + lr, c = c0 + lc;
        const bool inq = g0 + q < sub_r;  // the group's second sub-tile may lie past the super-tile
        const int valid = (inq && r < d.rows) ? max(0, min(8, d.cols - c)) : 0;
        if (valid > 0) load8_f32(d.W + (int64_t)r * d.ld_w + c, vec, valid, w[q]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) w[q][e] = 0.f;
        }
        int64_t off;
        int v2;
        if (!tall) {
          off = (int64_t)r * s.ldx + c;
          v2 = valid;
        } else {
          const int sr = c0 + (threadIdx.x >> 2), sc = r0 + (threadIdx.x & 3) * 8;
          off = (int64_t)sr * s.ldx + sc;
          v2 = (inq && sr < d.cols) ? max(0, min(8, d.rows - sc)) : 0;
        }
        if (v2 > 0) load8_slab(s.xf, XF32, off, v2, o[q]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) o[q][e] = 0.f;
        }
      }
      if (tall) {  // block-uniform
#pragma unroll
        for (int q = 0; q < kRedGroup; ++q)
#pragma unroll
          for (int e = 0; e < 8; ++e) tile[q][threadIdx.x >> 2][(threadIdx.x & 3) * 8 + e] = o[q][e];
        __syncthreads();
#pragma unroll
        for (int q = 0; q < kRedGroup; ++q)
#pragma unroll
          for (int e = 0; e < 8; ++e) o[q][e] = tile[q][lc + e][lr];
        __syncthreads();  // the tiles are reused by the next group
      }
#pragma unroll
      for (int q = 0; q < kRedGroup; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) {  // elements outside the matrix are 0 on both sides
          const float o2 = o[q][e] * o[q][e], wov = w[q][e] * o[q][e];
          ww = fmaf(w[q][e], w[q][e], ww);
          row_o2[g0 + q] += o2;
          row_wo[g0 + q] += wov;
          col_o2[e] += o2;
          col_wo[e] += wov;
        }
    }
    // the band's column sums: the 4 rows of a warp share columns every 8 lanes
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
      for (int m = 8; m < 32; m <<= 1) {
        col_o2[e] += __shfl_xor_sync(0xffffffffu, col_o2[e], m);
        col_wo[e] += __shfl_xor_sync(0xffffffffu, col_wo[e], m);
      }
    }
    const int buf = bj & 1;
    if (lane < 8) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        colred[buf][0][warp][lc + e] = col_o2[e];
        colred[buf][1][warp][lc + e] = col_wo[e];
      }
    }
    __syncthreads();
    if (threadIdx.x < 2 * kTC) {
      const int which = threadIdx.x / kTC, cc = threadIdx.x % kTC;
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < kThreads / 32; ++i) sum += colred[buf][which][i][cc];
      if (c0 + cc < d.cols) {
        if (which) atomicAdd(a.eq_wo + s.eq_off + d.rows + c0 + cc, sum * xs);
        else atomicAdd(a.eq_o2 + s.eq_off + d.rows + c0 + cc, sum * xs * xs);
      }
    }
    // the next band writes the other buffer; the band after it passes this band's
    // barrier only once every thread has read this buffer
  }
  // row sums: the 8 threads of a row are consecutive lanes; their totals over the
  // super-tile are the block's shares of <W,O> and ||O||^2
  float wo = 0.f, oo = 0.f;
#pragma unroll
  for (int bi = 0; bi < kSubR; ++bi) {
    float ro = row_o2[bi], rw = row_wo[bi];
    wo += rw;
    oo += ro;
#pragma unroll
    for (int m = 4; m > 0; m >>= 1) {
      ro += __shfl_xor_sync(0xffffffffu, ro, m);
      rw += __shfl_xor_sync(0xffffffffu, rw, m);
    }
    const int r = R0 + bi * kTR + lr;
    if ((threadIdx.x & 7) == 0 && bi < sub_r && r < d.rows) {
      atomicAdd(a.eq_o2 + s.eq_off + r, ro * xs * xs);
      atomicAdd(a.eq_wo + s.eq_off + r, rw * xs);
    }
  }
  double acc[3] = {ww, (double)wo * xs, (double)oo * xs * xs};
  block_sum<3>(acc, red);
  if (threadIdx.x == 0) {
    atomicAdd(&a.scal[k].w2, acc[0]);
    atomicAdd(&a.scal[k].wo, acc[1]);
    atomicAdd(&a.scal[k].o2, acc[2]);
  }
}

// ------------------------------------------------------------------ post_reduce (O only)
// Muon and the two-sided mode: ||O||^2 and the per-row and per-column sums of O^2,
// read from the Newton-Schulz slab alone (2 bytes per element in bf16) in the slab's
// own frame, where a slab row is a W row (wide) or a W column (tall: the slab holds
// O^T), so nothing is transposed. A block takes a band of kOTileR slab rows across the
// whole width (or, in a plan with too few bands to fill the GPU, one of `chunks` equal
// pieces of it), in kOTileC-column tiles: each warp 8 rows, each lane 8 consecutive
// columns of a tile (eight 16-byte loads, two each in fp32, issued before the
// arithmetic). In bf16 4 blocks per SM (64 registers) keep loads in flight while a
// block sums; two register buffers with the next tile's loads issued ahead (2 blocks
// per SM) measured 14 % slower. A tile's column partials are summed over the 8 warps
// through double-buffered shared memory (one barrier per tile) and flushed with one
// atomic per column; the row partials stay in registers over the band and are summed
// over the warp at its end by a halving exchange (each step keeps half of the rows and
// adds the partner's half: 4 + 2 + 1 shuffles, then 2 to finish). Slab columns past n
// hold whatever the Newton-Schulz stores left there and are masked.
template <bool XF32>
struct OTileRegs;
template <>
struct OTileRegs<false> {
  uint4 q[8];
};
template <>
struct OTileRegs<true> {
  float4 q[8][2];
};

template <bool XF32>
__device__ __forceinline__ void o_tile_load(OTileRegs<XF32>& b, const void* slab, int64_t ldx, int rw,
                                            int sm, int c, int sn) {
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const bool in = c < sn && rw + p < sm;
    if constexpr (XF32) {
      b.q[p][0] = b.q[p][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (in) {
        const float4* src =
            reinterpret_cast<const float4*>(static_cast<const float*>(slab) + (rw + p) * ldx + c);
        b.q[p][0] = __ldcs(src);
        b.q[p][1] = __ldcs(src + 1);
      }
    } else {
      b.q[p] = make_uint4(0u, 0u, 0u, 0u);
      if (in)
        b.q[p] = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(slab) + (rw + p) * ldx + c));
    }
  }
}

// rp[p] += sum over the lane's valid columns of row p; cp[e] += sum over the 8 rows
template <bool XF32>
__device__ __forceinline__ void o_tile_sums(const OTileRegs<XF32>& b, int nv, float (&rp)[8],
                                            float (&cp)[8]) {
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    float v[8];
    if constexpr (XF32) {
      v[0] = b.q[p][0].x; v[1] = b.q[p][0].y; v[2] = b.q[p][0].z; v[3] = b.q[p][0].w;
      v[4] = b.q[p][1].x; v[5] = b.q[p][1].y; v[6] = b.q[p][1].z; v[7] = b.q[p][1].w;
    } else {
      const uint32_t w4[4] = {b.q[p].x, b.q[p].y, b.q[p].z, b.q[p].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(w4[e] << 16);
        v[2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = e < nv ? v[e] : 0.f;
      rp[p] = fmaf(x, x, rp[p]);
      cp[e] = fmaf(x, x, cp[e]);
    }
  }
}

template <bool XF32>
__global__ void __launch_bounds__(kThreads, XF32 ? 2 : 4) post_reduce_o_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  static_assert(kOTileR == 8 * (kThreads / 32) && kOTileC == 8 * 32 && kOTileC == kThreads,
                "8 rows per warp, 8 columns per lane, one column per thread");
  __shared__ __align__(16) float colsh[2][kThreads / 32][kOTileC];
  __shared__ double red[1][kThreads / 32];
  const int b = blockIdx.x;
  const int k = find_matrix_in(a.o_tile_prefix, a.n, b);
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const bool tall = (d.flags & MAT_TRANSPOSED) != 0;
  const int sm = tall ? d.cols : d.rows, sn = tall ? d.rows : d.cols;  // slab rows, cols
  // blocks of a matrix: bands x chunks (a band's column walk in `chunks` pieces)
  const int bands = (sm + kOTileR - 1) / kOTileR;
  const int chunks = (a.o_tile_prefix[k + 1] - a.o_tile_prefix[k]) / bands;
  const int t = b - a.o_tile_prefix[k];
  const int R0 = (t / chunks) * kOTileR;
  const int ntc = (sn + kOTileC - 1) / kOTileC;
  const int per = (ntc + chunks - 1) / chunks;
  const int j0 = (t % chunks) * per, j1 = min(ntc, j0 + per);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rw = R0 + warp * 8;
  const float xs = slab_scale(a, k);
  const float xs2 = xs * xs;
  float* col_out = a.eq_o2 + s.eq_off + (tall ? 0 : d.rows);  // W rows (tall) or W columns
  float rp[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) rp[p] = 0.f;
  // c + 8 <= ldx whenever c < sn (ldx is a multiple of 64), so a whole 8-group load
  // stays inside the slab row
  auto tile = [&](const OTileRegs<XF32>& buf, int j) {
    const int c = j * kOTileC + lane * 8;
    float cp[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cp[e] = 0.f;
    o_tile_sums<XF32>(buf, max(0, min(8, sn - c)), rp, cp);
    float4* dst = reinterpret_cast<float4*>(&colsh[j & 1][warp][lane * 8]);
    dst[0] = make_float4(cp[0], cp[1], cp[2], cp[3]);
    dst[1] = make_float4(cp[4], cp[5], cp[6], cp[7]);
    __syncthreads();  // the buffer of tile j + 2 is written after the next barrier
    float col = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) col += colsh[j & 1][w][threadIdx.x];
    const int cc = j * kOTileC + threadIdx.x;
    if (cc < sn) atomicAdd(col_out + cc, col * xs2);
  };
  {
    OTileRegs<XF32> A;
    for (int j = j0; j < j1; ++j) {
      o_tile_load<XF32>(A, s.xf, s.ldx, rw, sm, j * kOTileC + lane * 8, sn);
      tile(A, j);
    }
  }
  float tot = 0.f;
#pragma unroll
  for (int p = 0; p < 8; ++p) tot += rp[p];
  // row sums over the warp: after the exchanges on lane bits 4, 3 and 2 each lane holds
  // row (lane >> 2) & 7 summed over 8 lanes; bits 1 and 0 finish the sum
  float h4[4], h2[2];
  const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0, b2 = (lane & 4) != 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b4 ? rp[i + 4] : rp[i], give = b4 ? rp[i] : rp[i + 4];
    h4[i] = keep + __shfl_xor_sync(0xffffffffu, give, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b3 ? h4[i + 2] : h4[i], give = b3 ? h4[i] : h4[i + 2];
    h2[i] = keep + __shfl_xor_sync(0xffffffffu, give, 8);
  }
  float row;
  {
    const float keep = b2 ? h2[1] : h2[0], give = b2 ? h2[0] : h2[1];
    row = keep + __shfl_xor_sync(0xffffffffu, give, 4);
  }
  row += __shfl_xor_sync(0xffffffffu, row, 2);
  row += __shfl_xor_sync(0xffffffffu, row, 1);
  {
    const int r = rw + ((lane >> 2) & 7);
    if ((lane & 3) == 0 && r < sm)
      atomicAdd(a.eq_o2 + s.eq_off + (tall ? d.rows + r : r), row * xs2);
  }
  double acc[1] = {tot};
  block_sum<1>(acc, red);
  if (threadIdx.x == 0) atomicAdd(&a.scal[k].o2, acc[0] * xs2);
}

// ------------------------------------------------------------------ post_reduce (staged)
// The three per-matrix sums with the loads moved out of the registers: every thread
// copies its share of each 32 x 64 sub-tile (W rows and slab rows, 16 bytes per copy)
// into a ring of shared-memory stages with cp.async, kStg - 1 sub-tiles ahead of the
// arithmetic, and reads its 8 elements back from shared memory. Bytes in flight per SM
// are then set by the ring (4 blocks x 4 stages of 12 KB), not by the registers that
// hold pending loads. Used when every W row segment of the plan is 16-byte aligned
// (rows of 16-byte multiples, 4 | cols), the slab is bf16 and the step has no
// equilibration (with the per-row and per-column sums as well, within 64 registers for
// 4 blocks per SM, a staged variant measured slower than the register-staged kernel
// above). For tall matrices a stage holds 64 slab rows of 64 bytes (32 storage rows of
// one storage column each), skewed by 16 bytes every 8 rows so that the column reads
// below meet no bank conflict. post_apply and ingest use the same ring.
constexpr int kStg = 4;                              // ring stages
constexpr int kStgW = kTR * kTC * 4;                 // W sub-tile, rows at 256 bytes
constexpr int kStgO = kTC * kTR * 2 + 8 * 16;        // O sub-tile (tall: skewed rows)
constexpr int kStgBytes = kStgW + kStgO;
constexpr int kStgSmem = kStg * kStgBytes + 128;     // dynamic shared memory (+ alignment)
static_assert(kStgBytes % 128 == 0, "stage alignment");

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Byte offset, in a stage's O part, of slab row k of a tall sub-tile.
__device__ __forceinline__ int o_tall_off(int k) { return k * 64 + (k >> 3) * 16; }

// This thread's copies of sub-tile (r0, c0) of matrix d into stage st: two 16-byte pieces
// of W (512 per sub-tile) and one of the slab (256). Pieces outside the matrix are not
// copied (the arithmetic masks them).
__device__ __forceinline__ void stage_subtile(const DevMat& d, const DevSlab& s, bool tall, int r0,
                                              int c0, uint8_t* st) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int q = tid + h * kThreads, row = q >> 4, col = (q & 15) * 4;
    if (r0 + row < d.rows && c0 + col < d.cols)
      cp_async16(st + row * (kTC * 4) + col * 4, d.W + static_cast<int64_t>(r0 + row) * d.ld_w + c0 + col);
  }
  const uint16_t* slab = static_cast<const uint16_t*>(s.xf);
  if (!tall) {
    const int row = tid >> 3, col = (tid & 7) * 8;
    if (r0 + row < d.rows)
      cp_async16(st + kStgW + row * (kTC * 2) + col * 2, slab + static_cast<int64_t>(r0 + row) * s.ldx + c0 + col);
  } else {
    const int k = tid >> 2, col = (tid & 3) * 8;  // slab row c0 + k, slab columns r0 + col ..
    if (c0 + k < d.cols)
      cp_async16(st + kStgW + o_tall_off(k) + col * 2, slab + static_cast<int64_t>(c0 + k) * s.ldx + r0 + col);
  }
}

__global__ void __launch_bounds__(kThreads, 4) post_reduce_staged_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  __shared__ double red[3][kThreads / 32];
  const int b = blockIdx.x;
  const int k = find_matrix(a, b);
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const int t = b - a.tile_prefix[k];
  const int sub_r = a.sub_r, sub_c = a.sub_c;
  const int tiles_c = (d.cols + sub_c * kTC - 1) / (sub_c * kTC);
  const int R0 = (t / tiles_c) * (sub_r * kTR), C0 = (t % tiles_c) * (sub_c * kTC);
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  const bool tall = (d.flags & MAT_TRANSPOSED) != 0;
  const float xs = slab_scale(a, k);  // 1/(||U||+eps) when the slab holds U (no iteration)
  // sub-tiles of the super-tile inside the matrix, band by band (64 columns each)
  const int nbr = min(sub_r, (d.rows - R0 + kTR - 1) / kTR);
  const int nbc = min(sub_c, (d.cols - C0 + kTC - 1) / kTC);
  const int nsub = nbr * nbc;
  // the first kStg - 1 stages in flight (one commit group per stage, empty ones too)
#pragma unroll
  for (int i = 0; i < kStg - 1; ++i) {
    if (i < nsub) stage_subtile(d, s, tall, R0 + (i % nbr) * kTR, C0 + (i / nbr) * kTC, ring + i * kStgBytes);
    cp_async_commit();
  }

  float ww = 0.f, wo = 0.f, oo = 0.f;
  for (int i = 0; i < nsub; ++i) {
    const int slot = i % kStg, g = i % nbr, bj = i / nbr;  // band-major order
    const int r0 = R0 + g * kTR, c0 = C0 + bj * kTC;
    const uint8_t* st = ring + slot * kStgBytes;
    {  // stage i + kStg - 1 goes into the slot freed at the end of the previous iteration
      const int in = i + kStg - 1;
      if (in < nsub)
        stage_subtile(d, s, tall, R0 + (in % nbr) * kTR, C0 + (in / nbr) * kTC, ring + (in % kStg) * kStgBytes);
      cp_async_commit();
    }
    cp_async_wait<kStg - 1>();  // this thread's copies of stage i have landed
    __syncthreads();            // and everyone's
    const int r = r0 + lr, c = c0 + lc;
    const int valid = r < d.rows ? max(0, min(8, d.cols - c)) : 0;
    float w[8], o[8];
    {
      const float4 x = *reinterpret_cast<const float4*>(st + lr * (kTC * 4) + lc * 4);
      const float4 y = *reinterpret_cast<const float4*>(st + lr * (kTC * 4) + lc * 4 + 16);
      w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
      w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
    }
    if (!tall) {
      const uint4 ov = *reinterpret_cast<const uint4*>(st + kStgW + lr * (kTC * 2) + lc * 2);
      const uint32_t q[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        o[2 * e] = __uint_as_float(q[e] << 16);
        o[2 * e + 1] = __uint_as_float(q[e] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        o[e] = __uint_as_float(static_cast<uint32_t>(
                   *reinterpret_cast<const uint16_t*>(st + kStgW + o_tall_off(lc + e) + lr * 2))
               << 16);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {  // stale shared memory outside the matrix counts as 0
      const float we = e < valid ? w[e] : 0.f, oe = e < valid ? o[e] : 0.f;
      const float o2 = oe * oe, wov = we * oe;
      ww = fmaf(we, we, ww);
      wo += wov;
      oo += o2;
    }
    // every thread is done with this stage before it is refilled
    __syncthreads();
  }
  cp_async_wait<0>();
  double acc[3] = {ww, (double)wo * xs, (double)oo * xs * xs};
  block_sum<3>(acc, red);
  if (threadIdx.x == 0) {
    atomicAdd(&a.scal[k].w2, acc[0]);
    atomicAdd(&a.scal[k].wo, acc[1]);
    atomicAdd(&a.scal[k].o2, acc[2]);
  }
}

// ------------------------------------------------------------------ post_finalize
__device__ __forceinline__ double block_sum2(double& x, double& y, double (*sh)[kThreads / 32]) {
  double v[2] = {x, y};
  block_sum<2>(v, sh);
  __shared__ double out[2];
  if (threadIdx.x == 0) { out[0] = v[0]; out[1] = v[1]; }
  __syncthreads();
  x = out[0];
  y = out[1];
  __syncthreads();
  return x;
}

// a7: the scale s of the orthogonalised update
__device__ __forceinline__ double step_scale(const ElemArgs& a, const DevMat& d) {
  const double rows = d.rows, cols = d.cols;
  if (a.scale_rule == MUON_SCALE_MOONLIGHT) return (double)a.scale_k * sqrt(fmax(rows, cols));
  if (a.scale_rule == MUON_SCALE_KELLER) return sqrt(fmax(1.0, rows / cols));
  return 1.0;
}

__global__ void __launch_bounds__(kThreads) post_finalize_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ double red[2][kThreads / 32];
  const int k = blockIdx.x;
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const MatScalars sc = a.scal[k];
  const double rows = d.rows, cols = d.cols;
  const double scale = step_scale(a, d);

  double wdo = sc.wo, doo = sc.o2;  // <W, D O>, ||D O||^2
  int axis = 0;
  if (a.mode == MUON_MODE_TWOSIDED) {
    // N_ij = X_ij rho / ((sqrt(r_i)+eps)(sqrt(c_j)+eps)): the row factor (with rho)
    // and the column factor go to the two halves of eq_o2
    const double rho = sqrt(sc.o2 / (rows * cols));
    for (int i = threadIdx.x; i < d.rows; i += kThreads)
      a.eq_o2[s.eq_off + i] =
          static_cast<float>(rho / (sqrt((double)a.eq_o2[s.eq_off + i] / cols) + (double)a.eps));
    for (int j = threadIdx.x; j < d.cols; j += kThreads)
      a.eq_o2[s.eq_off + d.rows + j] = static_cast<float>(
          1.0 / (sqrt((double)a.eq_o2[s.eq_off + d.rows + j] / rows) + (double)a.eps));
    if (threadIdx.x != 0) return;
    MatCoef cf;
    cf.cw = static_cast<float>(1.0 - (double)a.lr * (double)a.wd);
    cf.co = static_cast<float>(-(double)a.lr * scale);
    cf.axis = 3;
    cf.pad = 0;
    a.coef[k] = cf;
    if (a.stats != nullptr && !a.w_free) {
      const float nan = __int_as_float(0x7fc00000);
      muon_stats_t st;
      st.w_norm = static_cast<float>(sqrt(sc.w2));
      st.w_dot_o = nan;
      st.o_norm = nan;
      st.update_rms = nan;
      st.equil_axis = 3;
      st.reserved = 0;
      a.stats[d.orig] = st;
    }
    return;
  }
  if (a.equilibrate) {
    // imbalance = std / mean of the row RMS and of the column RMS vectors
    double sr = 0, sr2 = 0, scs = 0, sc2 = 0;
    for (int i = threadIdx.x; i < d.rows; i += kThreads) {
      const double v = sqrt((double)a.eq_o2[s.eq_off + i] / cols);
      sr += v;
      sr2 += v * v;
    }
    for (int j = threadIdx.x; j < d.cols; j += kThreads) {
      const double v = sqrt((double)a.eq_o2[s.eq_off + d.rows + j] / rows);
      scs += v;
      sc2 += v * v;
    }
    block_sum2(sr, sr2, red);
    block_sum2(scs, sc2, red);
    const double mr = sr / rows, mc = scs / cols;
    const double ir = mr > 0 ? sqrt(fmax(sr2 / rows - mr * mr, 0.0)) / mr : 0.0;
    const double ic = mc > 0 ? sqrt(fmax(sc2 / cols - mc * mc, 0.0)) / mc : 0.0;
    axis = (ir >= ic) ? 1 : 2;
    const double rho = sqrt(sc.o2 / (rows * cols));
    const int len = axis == 1 ? d.rows : d.cols;
    const double line = axis == 1 ? cols : rows;
    const int64_t base = s.eq_off + (axis == 1 ? 0 : d.rows);
    double dwo = 0, dd = 0;
    for (int i = threadIdx.x; i < len; i += kThreads) {
      const double o2 = a.eq_o2[base + i];
      const double f = rho / (sqrt(o2 / line) + (double)a.eps);
      dwo += f * (double)a.eq_wo[base + i];
      dd += f * f * o2;
      a.eq_o2[base + i] = static_cast<float>(f);  // factors for post_apply
    }
    block_sum2(dwo, dd, red);
    wdo = dwo;
    doo = dd;
  }
  if (threadIdx.x != 0) return;
  wdo *= scale;                 // <W, O> with O = s*D*O_raw
  const double oo = scale * scale * doo;
  const double lr = a.lr, cw0 = 1.0 - lr * (double)a.wd;
  double g = 0.0;
  if (a.mode == MUON_MODE_MUONGS && sc.w2 > 0.0) g = wdo / sc.w2;
  double cw = cw0 + lr * g, co = -lr * scale;
  if (a.mode == MUON_MODE_MUONH) {
    // W' = cw0 W - lr O; rescale to the current radius ||W_t||
    const double n2 = cw0 * cw0 * sc.w2 - 2.0 * cw0 * lr * wdo + lr * lr * oo;
    const double f = n2 > 0.0 ? sqrt(sc.w2 / n2) : 1.0;
    cw *= f;
    co *= f;
  }
  MatCoef cf;
  cf.cw = static_cast<float>(cw);
  cf.co = static_cast<float>(co);
  cf.axis = axis;
  cf.pad = 0;
  a.coef[k] = cf;
  if (a.stats != nullptr && !a.w_free) {  // else post_stats, after post_apply
    double ot2 = oo;
    if (a.mode == MUON_MODE_MUONGS && sc.w2 > 0.0) ot2 = oo - wdo * wdo / sc.w2;
    muon_stats_t st;
    st.w_norm = static_cast<float>(sqrt(sc.w2));
    st.w_dot_o = static_cast<float>(wdo);
    st.o_norm = static_cast<float>(sqrt(fmax(ot2, 0.0)));
    st.update_rms = static_cast<float>(sqrt(fmax(ot2, 0.0) / (rows * cols)));
    st.equil_axis = axis;
    st.reserved = 0;
    a.stats[d.orig] = st;
  }
}

// ------------------------------------------------------------------ post_apply
// Same walk as the plain reduction: per 64-column band, two 32-row sub-tiles at a time
// with all loads issued before the arithmetic and, for tall matrices, one shared-memory
// transpose of the two slab tiles.
// The statistics' sums of Muon and the two-sided mode, per block: ||W_t||^2,
// <W_t, D O_raw> and ||D O_raw||^2 (post_stats applies the scale).
__device__ __forceinline__ void apply_stats_flush(const ElemArgs& a, int k, float sw2, float swo,
                                                  float so2, double (*red)[kThreads / 32]) {
  double acc[3] = {sw2, swo, so2};
  block_sum<3>(acc, red);
  if (threadIdx.x == 0) {
    atomicAdd(&a.asum[k].w2, acc[0]);
    atomicAdd(&a.asum[k].wo, acc[1]);
    atomicAdd(&a.asum[k].o2, acc[2]);
  }
}

template <bool XF32>
__global__ void __launch_bounds__(kThreads, 4) post_apply_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float tile[kRedGroup][kTC][kTR + 1];
  __shared__ double red[3][kThreads / 32];
  const int b = blockIdx.x;
  const int k = find_matrix(a, b);
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const int t = b - a.tile_prefix[k];
  const int sub_r = a.sub_r, sub_c = a.sub_c;  // 32-row / 64-column sub-tiles per super-tile
  const int tiles_c = (d.cols + sub_c * kTC - 1) / (sub_c * kTC);
  const int R0 = (t / tiles_c) * (sub_r * kTR), C0 = (t % tiles_c) * (sub_c * kTC);
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  const bool vec = (d.flags & MAT_VEC_OK) != 0;
  const bool tall = (d.flags & MAT_TRANSPOSED) != 0;
  const bool ns_only = a.ns_only != 0;
  const bool st = a.apply_stats != 0;  // block-uniform
  float sw2 = 0.f, swo = 0.f, so2 = 0.f;
  const float xs = slab_scale(a, k);
  MatCoef cf;
  cf.cw = cf.co = 0.f;
  cf.axis = 0;
  if (!ns_only) cf = a.coef[k];
  for (int bj = 0; bj < sub_c && C0 + bj * kTC < d.cols; ++bj) {
    const int c0 = C0 + bj * kTC;
    const int c = c0 + lc;
    for (int g0 = 0; g0 < sub_r && R0 + g0 * kTR < d.rows; g0 += kRedGroup) {
      float w[kRedGroup][8], o[kRedGroup][8];
      int valid[kRedGroup];
#pragma unroll
      for (int q = 0; q < kRedGroup; ++q) {
        const int r0 = R0 + (g0 + q) * kTR;
        const int r = r0 + lr;
        const bool inq = g0 + q < sub_r;  // the group's second sub-tile may lie past the super-tile
        valid[q] = (inq && r < d.rows) ? max(0, min(8, d.cols - c)) : 0;
        if (!ns_only && valid[q] > 0) load8_f32(d.W + (int64_t)r * d.ld_w + c, vec, valid[q], w[q]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) w[q][e] = 0.f;
        }
        int64_t off;
        int v2;
        if (!tall) {
          off = (int64_t)r * s.ldx + c;
          v2 = valid[q];
        } else {
          const int sr = c0 + (threadIdx.x >> 2), sc = r0 + (threadIdx.x & 3) * 8;
          off = (int64_t)sr * s.ldx + sc;
          v2 = (inq && sr < d.cols) ? max(0, min(8, d.rows - sc)) : 0;
        }
        if (v2 > 0) load8_slab(s.xf, XF32, off, v2, o[q]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) o[q][e] = 0.f;
        }
      }
      if (tall) {  // block-uniform
#pragma unroll
        for (int q = 0; q < kRedGroup; ++q)
#pragma unroll
          for (int e = 0; e < 8; ++e) tile[q][threadIdx.x >> 2][(threadIdx.x & 3) * 8 + e] = o[q][e];
        __syncthreads();
#pragma unroll
        for (int q = 0; q < kRedGroup; ++q)
#pragma unroll
          for (int e = 0; e < 8; ++e) o[q][e] = tile[q][lc + e][lr];
        __syncthreads();  // the tiles are reused by the next group
      }
#pragma unroll
      for (int q = 0; q < kRedGroup; ++q) {
        if (valid[q] <= 0) continue;
        const int r = R0 + (g0 + q) * kTR + lr;
        if (ns_only) {
#pragma unroll
          for (int e = 0; e < 8; ++e) o[q][e] *= xs;
          if (d.flags & MAT_G_BF16)
            store8_bf16(reinterpret_cast<uint16_t*>(d.W) + (int64_t)r * d.ld_w + c, vec, valid[q], o[q]);
          else
            store8_f32(d.W + (int64_t)r * d.ld_w + c, vec, valid[q], o[q]);
          continue;
        }
        const float rowf = (cf.axis & 1) ? a.eq_o2[s.eq_off + r] : 1.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float f = xs * rowf;
          if ((cf.axis & 2) && e < valid[q]) f *= a.eq_o2[s.eq_off + d.rows + c + e];
          if (st && e < valid[q]) {
            const float ot = f * o[q][e];  // D O_raw
            sw2 = fmaf(w[q][e], w[q][e], sw2);
            swo = fmaf(w[q][e], ot, swo);
            so2 = fmaf(ot, ot, so2);
          }
          w[q][e] = fmaf(cf.cw, w[q][e], cf.co * f * o[q][e]);
        }
        store8_f32(d.W + (int64_t)r * d.ld_w + c, vec, valid[q], w[q]);
      }
    }
  }
  if (st) apply_stats_flush(a, k, sw2, swo, so2, red);
}

// post_apply with the W and slab loads staged in shared memory (cp.async, the ring of
// post_reduce_staged_kernel); the updated W goes straight from the registers to memory.
__global__ void __launch_bounds__(kThreads, 4) post_apply_staged_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  extern __shared__ uint8_t dsm_raw[];
  __shared__ double red[3][kThreads / 32];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  const int b = blockIdx.x;
  const int k = find_matrix(a, b);
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const int t = b - a.tile_prefix[k];
  const int sub_r = a.sub_r, sub_c = a.sub_c;
  const int tiles_c = (d.cols + sub_c * kTC - 1) / (sub_c * kTC);
  const int R0 = (t / tiles_c) * (sub_r * kTR), C0 = (t % tiles_c) * (sub_c * kTC);
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  const bool tall = (d.flags & MAT_TRANSPOSED) != 0;
  const MatCoef cf = a.coef[k];
  const float xs = slab_scale(a, k);  // 1/(||U||+eps) when the slab holds U (no iteration)
  const bool st = a.apply_stats != 0;  // block-uniform
  float sw2 = 0.f, swo = 0.f, so2 = 0.f;
  const int nbr = min(sub_r, (d.rows - R0 + kTR - 1) / kTR);
  const int nbc = min(sub_c, (d.cols - C0 + kTC - 1) / kTC);
  const int nsub = nbr * nbc;
#pragma unroll
  for (int i = 0; i < kStg - 1; ++i) {
    if (i < nsub) stage_subtile(d, s, tall, R0 + (i % nbr) * kTR, C0 + (i / nbr) * kTC, ring + i * kStgBytes);
    cp_async_commit();
  }
  for (int i = 0; i < nsub; ++i) {
    const int slot = i % kStg;
    const int r0 = R0 + (i % nbr) * kTR, c0 = C0 + (i / nbr) * kTC;
    const uint8_t* st = ring + slot * kStgBytes;
    {
      const int in = i + kStg - 1;
      if (in < nsub)
        stage_subtile(d, s, tall, R0 + (in % nbr) * kTR, C0 + (in / nbr) * kTC, ring + (in % kStg) * kStgBytes);
      cp_async_commit();
    }
    cp_async_wait<kStg - 1>();
    __syncthreads();
    const int r = r0 + lr, c = c0 + lc;
    const int valid = r < d.rows ? max(0, min(8, d.cols - c)) : 0;
    if (valid > 0) {
      float w[8], o[8];
      {
        const float4 x = *reinterpret_cast<const float4*>(st + lr * (kTC * 4) + lc * 4);
        const float4 y = *reinterpret_cast<const float4*>(st + lr * (kTC * 4) + lc * 4 + 16);
        w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
        w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
      }
      if (!tall) {
        const uint4 ov = *reinterpret_cast<const uint4*>(st + kStgW + lr * (kTC * 2) + lc * 2);
        const uint32_t q[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o[2 * e] = __uint_as_float(q[e] << 16);
          o[2 * e + 1] = __uint_as_float(q[e] & 0xFFFF0000u);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          o[e] = __uint_as_float(static_cast<uint32_t>(
                     *reinterpret_cast<const uint16_t*>(st + kStgW + o_tall_off(lc + e) + lr * 2))
                 << 16);
      }
      const float fr = xs * ((cf.axis & 1) ? a.eq_o2[s.eq_off + r] : 1.f);
      if (cf.axis & 2) {  // block-uniform: a factor per column
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float f = fr;
          if (e < valid) f *= a.eq_o2[s.eq_off + d.rows + c + e];
          if (st && e < valid) {
            const float ot = f * o[e];  // D O_raw
            sw2 = fmaf(w[e], w[e], sw2);
            swo = fmaf(w[e], ot, swo);
            so2 = fmaf(ot, ot, so2);
          }
          w[e] = fmaf(cf.cw, w[e], cf.co * f * o[e]);
        }
      } else {  // one factor for the thread's 8 elements
        if (st) {
          float two = 0.f, too = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (e < valid) {
              sw2 = fmaf(w[e], w[e], sw2);
              two = fmaf(w[e], o[e], two);
              too = fmaf(o[e], o[e], too);
            }
          swo = fmaf(fr, two, swo);
          so2 = fmaf(fr * fr, too, so2);
        }
        const float cof = cf.co * fr;
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = fmaf(cf.cw, w[e], cof * o[e]);
      }
      store8_f32(d.W + static_cast<int64_t>(r) * d.ld_w + c, true, valid, w);
    }
    __syncthreads();  // every thread is done with this stage before it is refilled
  }
  cp_async_wait<0>();
  if (st) apply_stats_flush(a, k, sw2, swo, so2, red);
}

// ------------------------------------------------------------------ post_stats
// Statistics of Muon and the two-sided mode from the sums post_apply accumulated:
// ||W_t||, <W_t, O> and ||O~|| with O = s D O_raw (O~ = O: no projection in these
// modes). The two-sided mode reports ||W_t|| only, as post_finalize does for it.
__global__ void __launch_bounds__(kThreads) post_stats_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  const int k = blockIdx.x * kThreads + threadIdx.x;
  if (k >= a.n) return;
  const DevMat d = a.mats[k];
  const ApplySums sc = a.asum[k];
  muon_stats_t st;
  st.w_norm = static_cast<float>(sqrt(sc.w2));
  st.reserved = 0;
  if (a.mode == MUON_MODE_TWOSIDED) {
    const float nan = __int_as_float(0x7fc00000);
    st.w_dot_o = st.o_norm = st.update_rms = nan;
    st.equil_axis = 3;
  } else {
    const double scale = step_scale(a, d);
    const double oo = scale * scale * sc.o2;
    st.w_dot_o = static_cast<float>(scale * sc.wo);
    st.o_norm = static_cast<float>(sqrt(oo));
    st.update_rms = static_cast<float>(sqrt(oo / (double(d.rows) * d.cols)));
    st.equil_axis = a.coef[k].axis;
  }
  a.stats[d.orig] = st;
}

}  // namespace

// Launch with programmatic stream serialisation: the kernel may start while its
// predecessor finishes and waits for it in griddep_wait().
// ------------------------------------------------------------------ ingest (staged)
// ingest with the G (bf16) and M loads staged in shared memory by cp.async, the ring of
// the staged post-processing kernels with a stage of G (4 KB) and M (8 KB). M goes
// back from the registers; U goes to the slab directly (wide) or through a bf16
// transpose tile with the skewed rows of the staged reads (tall).
constexpr int kStgInG = kTR * kTC * 2;               // G sub-tile (bf16), rows at 128 bytes
constexpr int kStgInBytes = kStgInG + kTR * kTC * 4; // + M sub-tile, rows at 256 bytes
constexpr int kStgInSmem = kStg * kStgInBytes + kStgO + 128;  // + the transpose tile
static_assert(kStgInBytes % 128 == 0 && kStgO % 128 == 0, "stage alignment");

__device__ __forceinline__ void stage_ingest(const DevMat& d, int r0, int c0, uint8_t* st) {
  const int tid = threadIdx.x;
  {  // G: 32 rows x 8 pieces of 8 bf16
    const int row = tid >> 3, col = (tid & 7) * 8;
    if (r0 + row < d.rows && c0 + col < d.cols)
      cp_async16(st + row * (kTC * 2) + col * 2,
                 static_cast<const uint16_t*>(d.G) + static_cast<int64_t>(r0 + row) * d.ld_g + c0 + col);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {  // M: 32 rows x 16 pieces of 4 floats
    const int q = tid + h * kThreads, row = q >> 4, col = (q & 15) * 4;
    if (r0 + row < d.rows && c0 + col < d.cols)
      cp_async16(st + kStgInG + row * (kTC * 4) + col * 4, d.M + static_cast<int64_t>(r0 + row) * d.ld_m + c0 + col);
  }
}

__global__ void __launch_bounds__(kThreads, 4) ingest_staged_kernel(const ElemArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  uint8_t* tt = ring + kStg * kStgInBytes;  // tall: U transposed, skewed 64-byte rows
  __shared__ double red[1][kThreads / 32];
  const int b = blockIdx.x;
  const int k = find_matrix(a, b);
  const DevMat d = a.mats[k];
  const DevSlab s = a.slabs[k];
  const int t = b - a.tile_prefix[k];
  const int sub_r = a.sub_r, sub_c = a.sub_c;
  const int tiles_c = (d.cols + sub_c * kTC - 1) / (sub_c * kTC);
  const int R0 = (t / tiles_c) * (sub_r * kTR), C0 = (t % tiles_c) * (sub_c * kTC);
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  const bool tall = (d.flags & MAT_TRANSPOSED) != 0;
  const int nbr = min(sub_r, (d.rows - R0 + kTR - 1) / kTR);
  const int nbc = min(sub_c, (d.cols - C0 + kTC - 1) / kTC);
  const int nsub = nbr * nbc;
  uint16_t* slab = static_cast<uint16_t*>(s.x0);
#pragma unroll
  for (int i = 0; i < kStg - 1; ++i) {
    if (i < nsub) stage_ingest(d, R0 + (i % nbr) * kTR, C0 + (i / nbr) * kTC, ring + i * kStgInBytes);
    cp_async_commit();
  }
  float sq = 0.f;
  for (int i = 0; i < nsub; ++i) {
    const int r0 = R0 + (i % nbr) * kTR, c0 = C0 + (i / nbr) * kTC;
    const uint8_t* st = ring + (i % kStg) * kStgInBytes;
    {
      const int in = i + kStg - 1;
      if (in < nsub) stage_ingest(d, R0 + (in % nbr) * kTR, C0 + (in / nbr) * kTC, ring + (in % kStg) * kStgInBytes);
      cp_async_commit();
    }
    cp_async_wait<kStg - 1>();
    __syncthreads();
    const int r = r0 + lr, c = c0 + lc;
    const int valid = r < d.rows ? max(0, min(8, d.cols - c)) : 0;
    float u[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) u[e] = 0.f;
    if (valid > 0) {
      float g[8], m[8];
      {
        const uint4 gv = *reinterpret_cast<const uint4*>(st + lr * (kTC * 2) + lc * 2);
        const uint32_t q[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          g[2 * e] = __uint_as_float(q[e] << 16);
          g[2 * e + 1] = __uint_as_float(q[e] & 0xFFFF0000u);
        }
        const float4 x = *reinterpret_cast<const float4*>(st + kStgInG + lr * (kTC * 4) + lc * 4);
        const float4 y = *reinterpret_cast<const float4*>(st + kStgInG + lr * (kTC * 4) + lc * 4 + 16);
        m[0] = x.x; m[1] = x.y; m[2] = x.z; m[3] = x.w;
        m[4] = y.x; m[5] = y.y; m[6] = y.z; m[7] = y.w;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        m[e] = fmaf(a.mu, m[e], g[e]);                       // M_t = mu*M_{t-1} + G_t
        u[e] = a.nesterov ? fmaf(a.mu, m[e], g[e]) : m[e];  // U = G_t + mu*M_t
        if (e >= valid) u[e] = 0.f;
      }
      store8_f32(d.M + static_cast<int64_t>(r) * d.ld_m + c, true, valid, m);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {  // ||U|| of the slab's bf16 values
      const float q = bf16_to_f32(f32_to_bf16(u[e]));
      sq = fmaf(q, q, sq);
    }
    if (!tall) {
      if (valid > 0) store8_bf16(slab + static_cast<int64_t>(r) * s.ldx + c, true, valid, u);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        *reinterpret_cast<uint16_t*>(tt + o_tall_off(lc + e) + lr * 2) = f32_to_bf16(u[e]);
      __syncthreads();
      const int k2 = threadIdx.x >> 2, col = (threadIdx.x & 3) * 8;  // slab row c0 + k2
      const int v2 = c0 + k2 < d.cols ? max(0, min(8, d.rows - (r0 + col))) : 0;
      if (v2 == 8) {
        *reinterpret_cast<uint4*>(slab + static_cast<int64_t>(c0 + k2) * s.ldx + r0 + col) =
            *reinterpret_cast<const uint4*>(tt + o_tall_off(k2) + col * 2);
      } else {
        for (int e = 0; e < v2; ++e)
          slab[static_cast<int64_t>(c0 + k2) * s.ldx + r0 + col + e] =
              *reinterpret_cast<const uint16_t*>(tt + o_tall_off(k2) + (col + e) * 2);
      }
    }
    __syncthreads();  // the stage (and the transpose tile) are free again
  }
  cp_async_wait<0>();
  double acc[1] = {sq};
  block_sum<1>(acc, red);
  if (threadIdx.x == 0) atomicAdd(&a.scal[k].u2, acc[0]);
}

template <typename... Args>
cudaError_t launch_pdl(void (*kern)(Args...), unsigned grid, cudaStream_t s, const ElemArgs& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// Shared-memory staged kernels: they need more than the default 48 KB of dynamic shared
// memory; the opt-in is a per-device attribute, set once on each device (per kernel).
template <void (*kern)(ElemArgs), int kSmem = kStgSmem, bool kPdl = true>
cudaError_t launch_staged_impl(const ElemArgs& a, cudaStream_t s) {
  static std::atomic<uint64_t> attr_devices{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit == 0 || !(attr_devices.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    attr_devices.fetch_or(bit, std::memory_order_acq_rel);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.total_tiles, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kPdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

cudaError_t launch_ingest(const ElemArgs& a, cudaStream_t s) {
  if (a.total_tiles <= 0) return cudaSuccess;
  // the first kernel of a step: no programmatic overlap with what precedes it
  if (a.staged_in) return launch_staged_impl<ingest_staged_kernel, kStgInSmem, false>(a, s);
  ingest_kernel<<<a.total_tiles, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}
cudaError_t launch_post_reduce(const ElemArgs& a, cudaStream_t s) {
  if (a.total_tiles <= 0) return cudaSuccess;
  if (a.w_free)
    return a.x_fp32 ? launch_pdl(post_reduce_o_kernel<true>, a.o_total_tiles, s, a)
                    : launch_pdl(post_reduce_o_kernel<false>, a.o_total_tiles, s, a);
  if (a.staged && !a.x_fp32 && !a.equilibrate) return launch_staged_impl<post_reduce_staged_kernel>(a, s);
  if (a.equilibrate)
    return a.x_fp32 ? launch_pdl(post_reduce_eq_kernel<true>, a.total_tiles, s, a)
                    : launch_pdl(post_reduce_eq_kernel<false>, a.total_tiles, s, a);
  return a.x_fp32 ? launch_pdl(post_reduce_plain_kernel<true>, a.total_tiles, s, a)
                  : launch_pdl(post_reduce_plain_kernel<false>, a.total_tiles, s, a);
}
cudaError_t launch_post_finalize(const ElemArgs& a, cudaStream_t s) {
  if (a.n <= 0) return cudaSuccess;
  return launch_pdl(post_finalize_kernel, a.n, s, a);
}
cudaError_t launch_post_apply(const ElemArgs& a, cudaStream_t s) {
  if (a.total_tiles <= 0) return cudaSuccess;
  if (a.staged && !a.x_fp32 && !a.ns_only) return launch_staged_impl<post_apply_staged_kernel>(a, s);
  return a.x_fp32 ? launch_pdl(post_apply_kernel<true>, a.total_tiles, s, a)
                  : launch_pdl(post_apply_kernel<false>, a.total_tiles, s, a);
}
cudaError_t launch_post_stats(const ElemArgs& a, cudaStream_t s) {
  if (a.n <= 0 || !a.apply_stats) return cudaSuccess;
  return launch_pdl(post_stats_kernel, (a.n + kThreads - 1) / kThreads, s, a);
}

}  // namespace muon
