// QK-Clip (MuonClip): per-head rescale of the query / key projection weights after
// an optimizer step, from "LLM Pretraining Loss Spike 진단과 처방", section
// "Moonlight와 MuonClip이 추가한 것" (QK-Clip listing): gamma_h = min(1, tau / S_max[h]);
// non-rotary q and k rows of head h are multiplied by gamma_h^0.5, its rotary q rows
// by gamma_h, the shared rotary key is left alone.
//
// One launch over every slice: block (slice, row chunk) reads S_max of its head on
// the device; heads at or below tau return without touching memory. fp32 weights,
// 128-bit accesses when aligned. Memory bound: 8 B per scaled element.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "muon.h"

namespace {

constexpr int kSlicesPerLaunch = 64;
constexpr int kRowsPerBlock = 8;
constexpr int kThreads = 256;

struct QkLaunch {
  muon_qk_slice_t s[kSlicesPerLaunch];
  int32_t block_base[kSlicesPerLaunch + 1];  // first block of each slice
  int32_t n;
  float tau;
  const float* s_max;
  int32_t n_heads;
};

__global__ void __launch_bounds__(kThreads) qk_clip_kernel(const QkLaunch L) {
  int i = 0;
  while (i + 1 < L.n && static_cast<int>(blockIdx.x) >= L.block_base[i + 1]) ++i;
  const muon_qk_slice_t sl = L.s[i];
  const float smax = __ldg(L.s_max + sl.head);
  if (!(smax > L.tau)) return;  // gamma = 1 (NaN S_max leaves the weights alone)
  const float gamma = L.tau / smax;
  const float f = (sl.power == 1.0f) ? gamma : powf(gamma, sl.power);
  const int64_t r0 = sl.row0 + static_cast<int64_t>(blockIdx.x - L.block_base[i]) * kRowsPerBlock;
  float* W = static_cast<float*>(sl.W);
  const bool vec = (reinterpret_cast<uintptr_t>(W) % 16 == 0) && (sl.ld % 4 == 0);
  for (int rr = 0; rr < kRowsPerBlock; ++rr) {
    const int64_t r = r0 + rr;
    if (r >= sl.row0 + sl.rows) break;
    float* row = W + r * sl.ld;
    if (vec) {
      const int64_t nv = sl.cols / 4;
      for (int64_t c = threadIdx.x; c < nv; c += kThreads) {
        float4 x = reinterpret_cast<float4*>(row)[c];
        x.x *= f; x.y *= f; x.z *= f; x.w *= f;
        reinterpret_cast<float4*>(row)[c] = x;
      }
      for (int64_t c = nv * 4 + threadIdx.x; c < sl.cols; c += kThreads) row[c] *= f;
    } else {
      for (int64_t c = threadIdx.x; c < sl.cols; c += kThreads) row[c] *= f;
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
    if (reinterpret_cast<uintptr_t>(s.W) % 4) return MUON_ERR_INVALID_ARG;
  }
  // overlapping slices would scale rows twice
  for (int i = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j)
      if (slices[i].W == slices[j].W && slices[i].row0 < slices[j].row0 + slices[j].rows &&
          slices[j].row0 < slices[i].row0 + slices[i].rows)
        return MUON_ERR_ALIAS;
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
