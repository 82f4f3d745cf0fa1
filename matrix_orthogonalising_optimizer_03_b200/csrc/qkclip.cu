// QK-Clip (MuonClip): per-head rescale of the query / key projection weights after
// an optimizer step, from "LLM Pretraining Loss Spike 진단과 처방", section
// "Moonlight와 MuonClip이 추가한 것" (QK-Clip listing): gamma_h = min(1, tau / S_max[h]);
// non-rotary q and k rows of head h are multiplied by gamma_h^0.5, its rotary q rows
// by gamma_h, the shared rotary key is left alone.
//
// One launch per 448 slices: block (slice, 16-row chunk) reads S_max of its head on
// the device; heads at or below tau return without touching memory. fp32 weights,
// 16-byte accesses when aligned, 8 loads in flight per thread before their stores.
// Memory bound: 8 B per scaled element.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

#include "muon.h"

namespace {

constexpr int kSlicesPerLaunch = 448;  // kernel parameters stay below 32 KB
constexpr int kRowsPerBlock = 16;
constexpr int kThreads = 256;
constexpr int kBatch = 8;              // 16-byte loads in flight per thread

struct QkLaunch {
  muon_qk_slice_t s[kSlicesPerLaunch];
  int32_t block_base[kSlicesPerLaunch + 1];  // first block of each slice
  int32_t n;
  float tau;
  const float* s_max;
  int32_t n_heads;
};
static_assert(sizeof(QkLaunch) < 32000, "kernel parameter space");

__global__ void __launch_bounds__(kThreads) qk_clip_kernel(const __grid_constant__ QkLaunch L) {
  int lo = 0, hi = L.n - 1;  // the slice of this block: last base <= blockIdx.x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (L.block_base[mid] <= static_cast<int>(blockIdx.x)) lo = mid; else hi = mid - 1;
  }
  const muon_qk_slice_t& sl = L.s[lo];
  const float smax = __ldg(L.s_max + sl.head);
  if (!(smax > L.tau)) return;  // gamma = 1 (NaN S_max leaves the weights alone)
  const float gamma = L.tau / smax;
  const float f = (sl.power == 1.0f) ? gamma : powf(gamma, sl.power);
  const int64_t r0 = sl.row0 + static_cast<int64_t>(blockIdx.x - L.block_base[lo]) * kRowsPerBlock;
  const int64_t left = sl.row0 + sl.rows - r0;
  const int nr = static_cast<int>(left < kRowsPerBlock ? left : kRowsPerBlock);
  float* W = static_cast<float*>(sl.W);
  const bool vec = (reinterpret_cast<uintptr_t>(W) % 16 == 0) && (sl.ld % 4 == 0);
  const int cols = static_cast<int>(sl.cols);
  if (vec) {
    // the block's rows as one run of 16-byte pieces: kBatch loads in flight per thread
    // before their stores
    const int nv = cols / 4, total = nr * nv;
    for (int base = 0; base < total; base += kThreads * kBatch) {
      float4 x[kBatch];
      float4* p[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = base + u * kThreads + threadIdx.x;
        p[u] = nullptr;
        if (j < total) {
          const int r = j / nv, c = j - r * nv;
          p[u] = reinterpret_cast<float4*>(W + (r0 + r) * sl.ld) + c;
          x[u] = *p[u];
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (p[u] == nullptr) continue;
        x[u].x *= f; x[u].y *= f; x[u].z *= f; x[u].w *= f;
        *p[u] = x[u];
      }
    }
    for (int j = threadIdx.x; j < nr * (cols - nv * 4); j += kThreads) {  // ragged columns
      const int r = j / (cols - nv * 4), c = nv * 4 + (j - r * (cols - nv * 4));
      W[(r0 + r) * sl.ld + c] *= f;
    }
  } else {
    for (int j = threadIdx.x; j < nr * cols; j += kThreads) {
      const int r = j / cols, c = j - r * cols;
      W[(r0 + r) * sl.ld + c] *= f;
    }
  }
}

}  // namespace

extern "C" MUON_API muon_status_t muon_qk_clip(const muon_qk_slice_t* slices, int n,
                                               const float* s_max_dev, int n_heads, float tau,
                                               void* stream) {
  if (n < 0 || (n > 0 && (slices == nullptr || s_max_dev == nullptr)) || n_heads < 1 ||
      !(tau > 0.f) || !std::isfinite(tau))
    return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const muon_qk_slice_t& s = slices[i];
    if (s.W == nullptr || s.head < 0 || s.head >= n_heads) return MUON_ERR_INVALID_ARG;
    if (!(s.power >= 0.f) || !std::isfinite(s.power)) return MUON_ERR_INVALID_ARG;
    if (s.row0 < 0 || s.rows < 0 || s.cols < 1 || s.ld < s.cols) return MUON_ERR_SHAPE;
    if (s.cols > (int64_t(1) << 30) / kRowsPerBlock) return MUON_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(s.W) % 4) return MUON_ERR_INVALID_ARG;
  }
  // overlapping slices would scale rows twice: sorted by (matrix, first row), a slice
  // overlaps an earlier one of its matrix iff it starts before the furthest row end so
  // far (empty slices scale nothing and are skipped)
  std::vector<int> order;
  order.reserve(n);
  for (int i = 0; i < n; ++i)
    if (slices[i].rows > 0) order.push_back(i);
  std::sort(order.begin(), order.end(), [&](int x, int y) {
    const uintptr_t wx = reinterpret_cast<uintptr_t>(slices[x].W);
    const uintptr_t wy = reinterpret_cast<uintptr_t>(slices[y].W);
    return wx != wy ? wx < wy : slices[x].row0 < slices[y].row0;
  });
  const void* cur = nullptr;
  int64_t end = 0;
  for (const int i : order) {
    const muon_qk_slice_t& a = slices[i];
    if (a.W != cur) {
      cur = a.W;
      end = 0;
    } else if (a.row0 < end) {
      return MUON_ERR_ALIAS;
    }
    end = std::max(end, a.row0 + a.rows);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int i0 = 0; i0 < n; i0 += kSlicesPerLaunch) {
    QkLaunch L{};
    L.n = n - i0 < kSlicesPerLaunch ? n - i0 : kSlicesPerLaunch;
    L.tau = tau;
    L.s_max = s_max_dev;
    L.n_heads = n_heads;
    int64_t blocks = 0;
    for (int i = 0; i < L.n; ++i) {
      L.s[i] = slices[i0 + i];
      L.block_base[i] = static_cast<int32_t>(blocks);
      blocks += (L.s[i].rows + kRowsPerBlock - 1) / kRowsPerBlock;
    }
    L.block_base[L.n] = static_cast<int32_t>(blocks);
    if (blocks == 0) continue;
    if (blocks > (int64_t(1) << 30)) return MUON_ERR_SHAPE;
    qk_clip_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(L);
    if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  }
  return MUON_OK;
}
