// Self-test of the bounded-wait mechanism every pipelined kernel of the library
// relies on: a single thread waits on an mbarrier that nothing ever arrives at,
// with a caller-chosen (short) limit, and reports the timeout through the
// workspace error word exactly as the GEMM kernels do. Nothing faults or hangs.
#include <cuda_runtime.h>

#include "muon.h"
#include "muon_internal.h"
#include "ptx.cuh"

namespace muon {
namespace {

__global__ void wait_probe_kernel(uint32_t* err, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait(&bar, 0, nullptr, limit)) set_error(err, MUON_ERR_TIMEOUT);
  mbar_arrive(&bar);  // leave the barrier in a completed state
}

}  // namespace
}  // namespace muon

extern "C" MUON_API muon_status_t muon_wait_probe(void* workspace, int64_t limit_cycles,
                                                  void* stream) {
  if (workspace == nullptr || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
    return MUON_ERR_WORKSPACE;
  if (limit_cycles < 1 || limit_cycles > muon::kWaitLimitCycles) return MUON_ERR_INVALID_ARG;
  muon::wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint32_t*>(workspace), static_cast<long long>(limit_cycles));
  return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}
