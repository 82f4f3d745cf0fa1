// muon_newton_schulz_noalloc: the Newton-Schulz orthogonalisation of one matrix
// with the library's own scratch memory instead of a caller workspace.
//
// Who needs it: code that cannot call cudaMalloc. Examples are code running under
// a memory pool or framework allocator that owns all device memory and must not be
// bypassed, and code that cannot afford the device-wide synchronisation that
// cudaMalloc / cudaFree may imply in the middle of a step. Such a caller passes
// only its input and output matrices.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes. Every
// GPU that loads the library holds it until the process exits. All calls share
// it and it keeps the last call's contents; each call clears what must start at
// zero. Calls whose work overlaps on the GPU (two streams, or two host threads)
// race on it and must be serialised by the caller.
//
// In host code the array's name is only a host-side stand-in for the device
// symbol. Its device address is obtained once per device, with that device
// current, by cudaGetSymbolAddress on the first call made on that device; that
// first call should therefore come before any stream capture.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>

#include <cstdint>
#include <cstring>

#include "muon.h"
#include "muon_internal.h"
#include "elementwise.h"
#include "ns_tc.h"
#include "validate.h"

namespace muon {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kNoAllocMaxDevices = 64;

// Layout of the scratch (byte offsets).
constexpr size_t kOffHeader = 0;
constexpr size_t kOffScal = 256;
constexpr size_t kOffCoef = 512;
constexpr size_t kOffDesc = 768;
constexpr size_t kOffSlabDesc = 1024;
constexpr size_t kOffTiles = 1280;
constexpr size_t kOffSlabs = 2048;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace
}  // namespace muon

static __device__ __align__(256) unsigned char g_noalloc_scratch[muon::kNoAllocScratchBytes];

namespace muon {
namespace {

// Per device: the device address of g_noalloc_scratch (published last) and the SM count.
std::atomic<void*> g_scratch_addr[kNoAllocMaxDevices];
std::atomic<int> g_num_sms[kNoAllocMaxDevices];

// Writes the one-matrix descriptor tables and clears the scalars and status words.
__global__ void noalloc_setup_kernel(unsigned char* base, DevMat d, DevSlab s, int32_t tiles,
                                     uint32_t* status) {
  if (threadIdx.x != 0) return;
  reinterpret_cast<WsHeader*>(base + kOffHeader)->error = 0;
  MatScalars* sc = reinterpret_cast<MatScalars*>(base + kOffScal);
  sc->u2 = sc->w2 = sc->wo = sc->o2 = 0.0;
  *reinterpret_cast<DevMat*>(base + kOffDesc) = d;
  *reinterpret_cast<DevSlab*>(base + kOffSlabDesc) = s;
  int32_t* t = reinterpret_cast<int32_t*>(base + kOffTiles);
  t[0] = 0;
  t[1] = tiles;
  if (status != nullptr) *status = 0;
}

muon_status_t scratch_for_current_device(unsigned char** out, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MUON_ERR_UNSUPPORTED;
  void* addr = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (addr == nullptr) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MUON_ERR_CUDA;
    if (major != 10 || minor != 0) return MUON_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return MUON_ERR_CUDA;
    g_num_sms[dev].store(sms, std::memory_order_relaxed);
    g_scratch_addr[dev].store(p, std::memory_order_release);
    addr = p;
  }
  *out = static_cast<unsigned char*>(addr);
  *num_sms = g_num_sms[dev].load(std::memory_order_relaxed);
  return MUON_OK;
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" MUON_API muon_status_t muon_newton_schulz_noalloc(const muon_ns_matrix_t* mat,
                                                              const muon_hparams_t* hp,
                                                              uint32_t* status_dev, void* stream) {
  // ---- host validation (nothing is enqueued on error): the same checks as
  // muon_newton_schulz_batched, so one set of arguments gets one status from both
  if (mat == nullptr) return MUON_ERR_INVALID_ARG;
  muon_status_t st = validate_ns(mat, 1, hp);
  if (st != MUON_OK) return st;
  const int64_t rows = mat->rows, cols = mat->cols;
  const int esz = mat->dtype == MUON_BF16 ? 2 : 4;
  const uintptr_t xa = reinterpret_cast<uintptr_t>(mat->X), oa = reinterpret_cast<uintptr_t>(mat->O);

  const bool fp32 = (hp->flags & MUON_NS_FP32) != 0;
  const int ex = fp32 ? 4 : 2;
  const int m = static_cast<int>(rows < cols ? rows : cols);
  const int n = static_cast<int>(rows < cols ? cols : rows);
  const int ldx = static_cast<int>(round_up(n, 64)), lds = static_cast<int>(round_up(m, 64));
  const size_t xbytes = size_t(m) * ldx * ex, sbytes = size_t(m) * lds * ex;
  const bool iterate = hp->ns_steps > 0;
  size_t off_x0 = kOffSlabs, off_x1 = off_x0, off_s = off_x0, off_p = off_x0;
  size_t end = round_up(off_x0 + xbytes, 1024);
  if (iterate) {
    off_x1 = end;
    end = round_up(off_x1 + xbytes, 1024);
    off_s = end;
    end = round_up(off_s + sbytes, 1024);
    off_p = end;
    end = round_up(off_p + sbytes, 1024);
  }
  if (end > kNoAllocScratchBytes) return MUON_ERR_WORKSPACE;  // beyond the static scratch

  unsigned char* base = nullptr;
  int num_sms = 0;
  st = scratch_for_current_device(&base, &num_sms);
  if (st != MUON_OK) return st;
  if (status_dev != nullptr) {
    // the setup kernel stores to it: it must be device memory of the current device
    int dev = 0;
    cudaPointerAttributes pa;
    if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
    if (cudaPointerGetAttributes(&pa, status_dev) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_INVALID_ARG;
    }
    if ((pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged) || pa.device != dev ||
        reinterpret_cast<uintptr_t>(status_dev) % 4 != 0)
      return MUON_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* err = status_dev != nullptr ? status_dev : reinterpret_cast<uint32_t*>(base + kOffHeader);

  // ---- descriptor of the single matrix (same conventions as the batched path)
  DevMat d{};
  d.W = static_cast<float*>(mat->O);
  d.G = mat->X;
  d.M = nullptr;
  d.ld_w = mat->ld_o;
  d.ld_g = mat->ld_x;
  d.rows = static_cast<int32_t>(rows);
  d.cols = static_cast<int32_t>(cols);
  const bool vec = xa % 16 == 0 && oa % 16 == 0 && (mat->ld_x * esz) % 16 == 0 &&
                   (mat->ld_o * esz) % 16 == 0;
  d.flags = (rows > cols ? MAT_TRANSPOSED : 0) | (esz == 2 ? MAT_G_BF16 : 0) | (vec ? MAT_VEC_OK : 0);
  d.orig = 0;
  DevSlab sl{};
  sl.x0 = base + off_x0;
  sl.xf = base + ((hp->ns_steps % 2) ? off_x1 : off_x0);
  sl.eq_off = 0;
  sl.ldx = ldx;
  sl.cls = 0;
  // elementwise super-tiles as the batched path picks them for a one-matrix step
  const bool small = rows * cols <= kElemSmallStep;
  const int sub_r = small ? 1 : kElemTileR / kElemSubR, sub_c = small ? 1 : kElemTileC / kElemSubC;
  const int64_t tiles = ((rows + sub_r * kElemSubR - 1) / (sub_r * kElemSubR)) *
                        ((cols + sub_c * kElemSubC - 1) / (sub_c * kElemSubC));
  noalloc_setup_kernel<<<1, 32, 0, s>>>(base, d, sl, static_cast<int32_t>(tiles), status_dev);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;

  ElemArgs ea{};
  ea.mats = reinterpret_cast<const DevMat*>(base + kOffDesc);
  ea.slabs = reinterpret_cast<const DevSlab*>(base + kOffSlabDesc);
  ea.tile_prefix = reinterpret_cast<const int32_t*>(base + kOffTiles);
  ea.n = 1;
  ea.total_tiles = static_cast<int32_t>(tiles);
  ea.scal = reinterpret_cast<MatScalars*>(base + kOffScal);
  ea.coef = reinterpret_cast<MatCoef*>(base + kOffCoef);
  ea.err = err;
  ea.eps = hp->eps;
  ea.ns_only = 1;
  ea.x_fp32 = fp32 ? 1 : 0;
  ea.xs_from_u2 = iterate ? 0 : 1;
  ea.sub_r = sub_r;
  ea.sub_c = sub_c;
  if (launch_ingest(ea, s) != cudaSuccess) return MUON_ERR_CUDA;

  // the same kernels and tile shapes the batched path picks for this shape: CTA
  // pairs with 256 x 256 tiles when m is a multiple of 256, single CTAs otherwise
  const bool pair = !fp32 && m % kPairTile == 0;
  for (int it = 0; it < hp->ns_steps; ++it) {
    for (int phase = PH_GRAM; phase <= PH_APPLY; ++phase) {
      const int bm = fp32 ? 64 : (pair ? kPairTile : tc_block_m());
      const int bn = fp32 ? 64 : (pair ? kPairTile : tc_block_n(phase));
      const int bk = fp32 ? 16 : tc_block_k();
      TcParams P;
      std::memset(&P, 0, sizeof(P));
      NsPhaseArgs& a = P.args;
      a.num_classes = 1;
      a.phase = phase;
      a.a = hp->ns_coeffs[0];
      a.b = hp->ns_coeffs[1];
      a.c = hp->ns_coeffs[2];
      a.first_iter = it == 0 ? 1 : 0;
      a.eps = hp->eps;
      a.scal = ea.scal;
      a.err = err;
      NsClassArgs& k = a.cls[0];
      k.m = m;
      k.n = n;
      k.count = 1;
      k.first = 0;
      k.ldx = ldx;
      k.lds = lds;
      k.xstride = int64_t(m) * ldx;
      k.sstride = int64_t(m) * lds;
      k.x_in = base + ((it % 2) ? off_x1 : off_x0);
      k.x_out = base + ((it % 2) ? off_x0 : off_x1);
      k.s = base + off_s;
      k.p = base + off_p;
      const int ncols = phase == PH_APPLY ? n : m;
      k.tiles_i = (m + bm - 1) / bm;
      k.tiles_j = (ncols + bn - 1) / bn;
      k.tiles_per_mat = phase == PH_APPLY ? k.tiles_i * k.tiles_j : k.tiles_i * (k.tiles_i + 1) / 2;
      if (!fp32 && !pair && phase != PH_APPLY) k.tiles_per_mat = sym_tiles_per_matrix(m);
      k.k_blocks = ((phase == PH_GRAM ? n : m) + bk - 1) / bk;
      a.tile_base[0] = 0;
      a.tile_base[1] = k.tiles_per_mat;
      if (fp32) {
        if (launch_ns_phase_simt(a, s) != cudaSuccess) return MUON_ERR_CUDA;
        continue;
      }
      const void* x_in = k.x_in;
      bool ok = true;
      // S and P' hold only their blocks on or above the diagonal; *_t maps fetch mirrors
      // (single-CTA symmetric phases take B in 64-row units: 64 x 64 boxes or
      // one-chunk mirrors)
      if (phase == PH_GRAM) {
        ok = encode_slab_map_bf16(&P.ta[0], x_in, n, m, 1, ldx, 64, 128) &&
             encode_slab_map_bf16(&P.tb[0], x_in, n, m, 1, ldx, 64, pair ? 128 : 64) &&
             encode_slab_map_bf16(&P.tc[0], k.s, m, m, 1, lds, 64, 128) &&
             encode_slab_map_bf16(&P.td[0], k.s, m, m, 1, lds, 64, 32);
        P.ta_t[0] = P.ta[0];
        P.tb_t[0] = P.tb[0];
      } else if (phase == PH_POLY) {
        ok = encode_slab_map_bf16(&P.ta[0], k.s, m, m, 1, lds, 64, 128) &&
             encode_chunk_map_bf16(&P.ta_t[0], k.s, m, m, 1, lds, 2) &&
             encode_slab_map_bf16(&P.tb[0], k.s, m, m, 1, lds, 64, pair ? 128 : 64) &&
             encode_chunk_map_bf16(&P.tb_t[0], k.s, m, m, 1, lds, pair ? 2 : 1) &&
             encode_slab_map_bf16(&P.td[0], k.p, m, m, 1, lds, 64, 32);
        P.tc[0] = P.ta[0];
      } else {
        ok = encode_slab_map_bf16(&P.ta[0], k.p, m, m, 1, lds, 64, 128) &&
             encode_chunk_map_bf16(&P.ta_t[0], k.p, m, m, 1, lds, 2) &&
             encode_chunk_map_bf16(&P.tb[0], x_in, n, m, 1, ldx,
                                   pair ? 2 : tc_block_n(PH_APPLY) / 64) &&
             encode_slab_map_bf16(&P.tc[0], x_in, n, m, 1, ldx, 64, 128) &&
             encode_slab_map_bf16(&P.td[0], k.x_out, n, m, 1, ldx, 64, 32);
        P.tb_t[0] = P.tb[0];
      }
      if (!ok) return MUON_ERR_CUDA;
      const cudaError_t e = pair ? launch_ns_phase_tc_pair(P, num_sms, s)
                                 : launch_ns_phase_tc(P, num_sms, s);
      if (e != cudaSuccess) return MUON_ERR_CUDA;
    }
  }
  if (launch_post_apply(ea, s) != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}
