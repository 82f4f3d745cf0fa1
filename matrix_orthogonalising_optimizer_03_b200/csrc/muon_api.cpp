// Host side of libmuon: validation, shape grouping (the plan), workspace layout,
// descriptor upload and the launch sequence of one Muon step.
//
// Step order (the update order of "[Deep Learning] Muon — 행렬 업데이트를 직교화하는
// 옵티마이저", section 3): ingest (momentum, Nesterov, ||U||^2) -> ns_steps x
// {GRAM, POLY, APPLY} -> post_reduce -> post_finalize -> post_apply.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <new>
#include <tuple>
#include <vector>

#include "muon.h"
#include "muon_internal.h"
#include "elementwise.h"
#include "ns_tc.h"
#include "validate.h"

using namespace muon;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kSlabAlign = 1024;
constexpr int kMaxDevices = 64;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t round_up64(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

struct ClassMaps {
  CUtensorMap x128[2];  // X slabs, 64 x 128 boxes (K-major operand, output)
  CUtensorMap xmn[2];   // X slabs, chunk view (MN-major operand of APPLY)
  CUtensorMap s128;     // S slab, 64 x 128 boxes
  CUtensorMap smir;     // S slab, chunk view (mirror blocks below the diagonal)
  CUtensorMap p128;     // P' slab, 64 x 128 boxes
  CUtensorMap pmir;     // P' slab, chunk view
  CUtensorMap x32[2];   // output boxes of one epilogue warp: 64 x 32
  CUtensorMap s32;
  CUtensorMap p32;
  // single-CTA symmetric phases load B in 64-row units
  CUtensorMap x64[2];   // X slabs, 64 x 64 boxes
  CUtensorMap s64;      // S slab, 64 x 64 boxes
  CUtensorMap smir1;    // S slab, chunk view, one chunk
};

}  // namespace

struct muon_plan_s {
  bool ns_only = false;
  int n = 0;
  muon_hparams_t hp{};
  int ns_steps = 0;  // Newton-Schulz iterations actually run (0 in the two-sided mode)
  bool x_fp32 = false;
  bool equilibrate = false;
  std::vector<ClassInfo> classes;
  std::vector<DevMat> dev;         // plan order
  std::vector<int64_t> eq_off;     // plan order
  std::vector<int32_t> tile_prefix;
  std::vector<int32_t> o_tile_prefix;  // O-only reduction tiles (slab frame)
  int64_t eq_total = 0;
  int sub_r = 4, sub_c = 4;  // elementwise super-tile in 32 x 64 sub-tiles
  bool staged = false;       // staged (shared-memory ring) post_reduce and post_apply
  bool staged_in = false;    // staged ingest
  size_t off_scal = 0, off_coef = 0, off_desc = 0, off_slabs = 0, off_tiles = 0, off_otiles = 0;
  size_t off_asum = 0;
  size_t off_eq_o2 = 0, off_eq_wo = 0, ws_bytes = 0;
  // cached per workspace pointer and device
  void* ws_cached = nullptr;
  int dev_cached = -1;
  int num_sms = 0;
  std::vector<ClassMaps> maps;
  // optional per-launch event timing
  struct ProfRec {
    cudaEvent_t a, b;
    int kind;
    double flops, bytes;
  };
  bool prof = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> event_pool;
  // A cached plan replays its step as a CUDA graph (one launch instead of ~20) while
  // the workspace, the stats pointer, the device and the hyper-parameters stay the
  // same. The first step runs eagerly (lazy per-device setup); the next one is captured
  // on a private stream; a failed capture leaves the plan eager for good.
  bool use_graph = false;
  bool graph_ok = true;
  bool graph_stale = false;  // hyper-parameters changed: update the executable in place
  int eager_steps = 0;
  cudaGraphExec_t graph_exec = nullptr;
  void* graph_ws = nullptr;
  muon_stats_t* graph_stats = nullptr;
  int graph_dev = -1;
  cudaStream_t cap_stream = nullptr;
  void drop_graph() {
    if (graph_exec != nullptr) cudaGraphExecDestroy(graph_exec);
    graph_exec = nullptr;
    graph_stale = false;
  }
  ~muon_plan_s() {
    for (const ProfRec& r : recs) {
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
    for (cudaEvent_t e : event_pool) cudaEventDestroy(e);
    drop_graph();
    if (cap_stream != nullptr) cudaStreamDestroy(cap_stream);
  }
};

namespace {

bool valid_enum_hp(const muon_hparams_t* hp) {
  if (hp->ns_steps < 0 || hp->ns_steps > 64) return false;
  if (hp->mode != MUON_MODE_MUON && hp->mode != MUON_MODE_MUONGS && hp->mode != MUON_MODE_MUONH &&
      hp->mode != MUON_MODE_TWOSIDED)
    return false;
  if (hp->scale != MUON_SCALE_MOONLIGHT && hp->scale != MUON_SCALE_KELLER &&
      hp->scale != MUON_SCALE_NONE)
    return false;
  const uint32_t known = MUON_NESTEROV | MUON_EQUILIBRATE | MUON_NS_FP32 | MUON_WANT_STATS;
  if (hp->flags & ~known) return false;
  if (!(hp->eps >= 0.f) || !std::isfinite(hp->eps)) return false;
  return true;
}

struct Interval {
  uintptr_t lo, hi;
  bool writable;
};

// Overlap of a written range with any other range is an error; read-only ranges may overlap.
bool any_alias(std::vector<Interval>& iv) {
  std::sort(iv.begin(), iv.end(), [](const Interval& a, const Interval& b) { return a.lo < b.lo; });
  uintptr_t end_any = 0, end_w = 0;
  bool first = true;
  for (const Interval& x : iv) {
    if (!first) {
      if (x.lo < end_w) return true;
      if (x.writable && x.lo < end_any) return true;
    }
    first = false;
    end_any = std::max(end_any, x.hi);
    if (x.writable) end_w = std::max(end_w, x.hi);
  }
  return false;
}

uintptr_t span_end(const void* p, int64_t rows, int64_t cols, int64_t ld, int esz) {
  return reinterpret_cast<uintptr_t>(p) + static_cast<uintptr_t>(((rows - 1) * ld + cols) * esz);
}

muon_status_t check_shape(int64_t rows, int64_t cols) {
  if (rows < 1 || cols < 1) return MUON_ERR_SHAPE;
  if (rows > (1 << 24) || cols > (1 << 24) || rows * cols >= (int64_t(1) << 31)) return MUON_ERR_SHAPE;
  return MUON_OK;
}

muon_status_t validate_step(const muon_matrix_t* mats, int n, const muon_hparams_t* hp) {
  if (hp == nullptr || n < 0 || (n > 0 && mats == nullptr)) return MUON_ERR_INVALID_ARG;
  if (!valid_enum_hp(hp)) return MUON_ERR_INVALID_ARG;
  std::vector<Interval> iv;
  iv.reserve(3 * static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    const muon_matrix_t& m = mats[i];
    if (m.W == nullptr || m.grad == nullptr || m.momentum == nullptr) return MUON_ERR_INVALID_ARG;
    muon_status_t s = check_shape(m.rows, m.cols);
    if (s != MUON_OK) return s;
    if (m.ld_w < m.cols || m.ld_g < m.cols || m.ld_m < m.cols) return MUON_ERR_SHAPE;
    if (m.w_dtype != MUON_F32) return MUON_ERR_DTYPE;
    if (m.g_dtype != MUON_F32 && m.g_dtype != MUON_BF16) return MUON_ERR_DTYPE;
    const int gsz = m.g_dtype == MUON_BF16 ? 2 : 4;
    if (reinterpret_cast<uintptr_t>(m.W) % 4 || reinterpret_cast<uintptr_t>(m.momentum) % 4 ||
        reinterpret_cast<uintptr_t>(m.grad) % gsz)
      return MUON_ERR_INVALID_ARG;
    iv.push_back({reinterpret_cast<uintptr_t>(m.W), span_end(m.W, m.rows, m.cols, m.ld_w, 4), true});
    iv.push_back({reinterpret_cast<uintptr_t>(m.momentum),
                  span_end(m.momentum, m.rows, m.cols, m.ld_m, 4), true});
    iv.push_back({reinterpret_cast<uintptr_t>(m.grad), span_end(m.grad, m.rows, m.cols, m.ld_g, gsz),
                  false});
  }
  if (any_alias(iv)) return MUON_ERR_ALIAS;
  return MUON_OK;
}

}  // namespace

// Host validation of a Newton-Schulz-only list, shared by muon_newton_schulz_batched,
// muon_ns_workspace_size and muon_newton_schulz_noalloc (declared in muon_internal.h).
muon_status_t muon::validate_ns(const muon_ns_matrix_t* mats, int n, const muon_hparams_t* hp) {
  if (hp == nullptr || n < 0 || (n > 0 && mats == nullptr)) return MUON_ERR_INVALID_ARG;
  if (!valid_enum_hp(hp)) return MUON_ERR_INVALID_ARG;
  std::vector<Interval> iv;
  for (int i = 0; i < n; ++i) {
    const muon_ns_matrix_t& m = mats[i];
    if (m.X == nullptr || m.O == nullptr) return MUON_ERR_INVALID_ARG;
    muon_status_t s = check_shape(m.rows, m.cols);
    if (s != MUON_OK) return s;
    if (m.ld_x < m.cols || m.ld_o < m.cols) return MUON_ERR_SHAPE;
    if (m.dtype != MUON_F32 && m.dtype != MUON_BF16) return MUON_ERR_DTYPE;
    const int esz = m.dtype == MUON_BF16 ? 2 : 4;
    if (reinterpret_cast<uintptr_t>(m.X) % esz || reinterpret_cast<uintptr_t>(m.O) % esz)
      return MUON_ERR_INVALID_ARG;
    iv.push_back({reinterpret_cast<uintptr_t>(m.O), span_end(m.O, m.rows, m.cols, m.ld_o, esz), true});
    iv.push_back({reinterpret_cast<uintptr_t>(m.X), span_end(m.X, m.rows, m.cols, m.ld_x, esz), false});
  }
  if (any_alias(iv)) return MUON_ERR_ALIAS;
  return MUON_OK;
}

namespace {

// Groups matrices by oriented shape and lays out the workspace.
void build_plan(muon_plan_s* p) {
  const int n = p->n;
  const bool x_fp32 = p->x_fp32;
  const int esz = x_fp32 ? 4 : 2;
  // class key: (m, n) oriented; heavier classes first (longer reductions first
  // in the persistent tile order)
  std::map<std::pair<int, int>, std::vector<int>> groups;
  for (int i = 0; i < n; ++i) {
    const int r = p->dev[i].rows, c = p->dev[i].cols;
    groups[{std::min(r, c), std::max(r, c)}].push_back(i);
  }
  std::vector<std::pair<std::pair<int, int>, std::vector<int>>> order(groups.begin(), groups.end());
  std::stable_sort(order.begin(), order.end(), [](const auto& a, const auto& b) {
    const double wa = double(a.first.first) * a.first.first * a.first.second;
    const double wb = double(b.first.first) * b.first.first * b.first.second;
    return wa > wb;
  });
  std::vector<DevMat> sorted;
  std::vector<int64_t> eq_off;
  sorted.reserve(n);
  p->classes.clear();
  int64_t eq_total = 0;
  for (auto& g : order) {
    ClassInfo ci{};
    ci.m = g.first.first;
    ci.n = g.first.second;
    ci.count = static_cast<int32_t>(g.second.size());
    ci.first = static_cast<int32_t>(sorted.size());
    ci.ldx = static_cast<int32_t>(round_up64(ci.n, 64));
    ci.lds = static_cast<int32_t>(round_up64(ci.m, 64));
    ci.xbytes = int64_t(ci.m) * ci.ldx * esz;
    ci.sbytes = int64_t(ci.m) * ci.lds * esz;
    for (int idx : g.second) {
      sorted.push_back(p->dev[idx]);
      eq_off.push_back(eq_total);
      eq_total += p->dev[idx].rows + p->dev[idx].cols;
    }
    p->classes.push_back(ci);
  }
  p->dev.swap(sorted);
  p->eq_off.swap(eq_off);
  p->eq_total = p->equilibrate ? eq_total : 0;
  // elementwise tiles: one-sub-tile super-tiles for small steps, 128 x 256 otherwise
  int64_t elems = 0;
  for (int i = 0; i < n; ++i) elems += int64_t(p->dev[i].rows) * p->dev[i].cols;
  p->sub_r = elems <= kElemSmallStep ? 1 : kElemTileR / kElemSubR;
  p->sub_c = elems <= kElemSmallStep ? 1 : kElemTileC / kElemSubC;
  const int tr = p->sub_r * kElemSubR, tc = p->sub_c * kElemSubC;
  // the staged (plain) reduction copies W rows and slab rows in 16-byte pieces with
  // cp.async: 16-byte aligned rows of 16-byte multiples; worth it only with several
  // sub-tiles per block
  p->staged = !p->x_fp32 && p->sub_r * p->sub_c > 1;
  for (int i = 0; i < n; ++i)
    p->staged = p->staged && (p->dev[i].flags & MAT_VEC_OK) != 0 && p->dev[i].cols % 4 == 0;
  // staged ingest: bf16 gradients whose rows are 16-byte multiples, and a momentum
  p->staged_in = p->staged && !p->ns_only;
  for (int i = 0; i < n; ++i)
    p->staged_in = p->staged_in && (p->dev[i].flags & MAT_G_BF16) != 0 && p->dev[i].cols % 8 == 0;
  p->tile_prefix.assign(n + 1, 0);
  for (int i = 0; i < n; ++i) {
    const int64_t t = int64_t((p->dev[i].rows + tr - 1) / tr) * ((p->dev[i].cols + tc - 1) / tc);
    p->tile_prefix[i + 1] = static_cast<int32_t>(p->tile_prefix[i] + t);
  }
  // slab-only reduction: a block walks a band of kOTileR slab rows across the whole
  // width; a plan with fewer than kOMinBlocks bands cuts each band's walk into up to
  // `split` pieces (one block each), so that a few large matrices still fill the GPU
  int64_t bands_total = 0;
  for (int i = 0; i < n; ++i)
    bands_total += (std::min(p->dev[i].rows, p->dev[i].cols) + kOTileR - 1) / kOTileR;
  const int64_t split =
      (bands_total == 0 || bands_total >= kOMinBlocks) ? 1 : (kOMinBlocks + bands_total - 1) / bands_total;
  p->o_tile_prefix.assign(n + 1, 0);
  for (int i = 0; i < n; ++i) {
    const int sm = std::min(p->dev[i].rows, p->dev[i].cols), sn = std::max(p->dev[i].rows, p->dev[i].cols);
    const int64_t chunks = std::min<int64_t>(split, (sn + kOTileC - 1) / kOTileC);
    p->o_tile_prefix[i + 1] = static_cast<int32_t>(p->o_tile_prefix[i] + ((sm + kOTileR - 1) / kOTileR) * chunks);
  }
  // workspace layout
  size_t off = align_up(sizeof(WsHeader), kAlign);
  p->off_scal = off;   off = align_up(off + sizeof(MatScalars) * n, kAlign);
  p->off_asum = off;   off = align_up(off + sizeof(ApplySums) * n, kAlign);
  p->off_coef = off;   off = align_up(off + sizeof(MatCoef) * n, kAlign);
  p->off_desc = off;   off = align_up(off + sizeof(DevMat) * n, kAlign);
  p->off_slabs = off;  off = align_up(off + sizeof(DevSlab) * n, kAlign);
  p->off_tiles = off;  off = align_up(off + sizeof(int32_t) * (n + 1), kAlign);
  p->off_otiles = off; off = align_up(off + sizeof(int32_t) * (n + 1), kAlign);
  p->off_eq_o2 = off;  off = align_up(off + sizeof(float) * p->eq_total, kAlign);
  p->off_eq_wo = off;  off = align_up(off + sizeof(float) * p->eq_total, kAlign);
  off = align_up(off, kSlabAlign);
  const bool two_x = p->ns_steps > 0;
  for (ClassInfo& ci : p->classes) {
    ci.off_x[0] = static_cast<int64_t>(off);
    off = align_up(off + ci.xbytes * ci.count, kSlabAlign);
    if (two_x) {
      ci.off_x[1] = static_cast<int64_t>(off);
      off = align_up(off + ci.xbytes * ci.count, kSlabAlign);
    } else {
      ci.off_x[1] = ci.off_x[0];
    }
    if (p->ns_steps > 0) {
      ci.off_s = static_cast<int64_t>(off);
      off = align_up(off + ci.sbytes * ci.count, kSlabAlign);
      ci.off_p = static_cast<int64_t>(off);
      off = align_up(off + ci.sbytes * ci.count, kSlabAlign);
    } else {
      ci.off_s = ci.off_p = ci.off_x[0];
    }
  }
  p->ws_bytes = off;
}

int32_t vec_flag(const void* a, const void* b, const void* c, int64_t la, int64_t lb, int64_t lc,
                 int ea, int eb, int ec) {
  auto ok = [](const void* ptr, int64_t ld, int esz) {
    if (ptr == nullptr) return true;
    return reinterpret_cast<uintptr_t>(ptr) % 16 == 0 && (ld * esz) % 16 == 0;
  };
  return (ok(a, la, ea) && ok(b, lb, eb) && ok(c, lc, ec)) ? MAT_VEC_OK : 0;
}

muon_plan_s* make_step_plan(const muon_matrix_t* mats, int n, const muon_hparams_t* hp) {
  muon_plan_s* p = new (std::nothrow) muon_plan_s();
  if (p == nullptr) return nullptr;
  p->ns_only = false;
  p->n = n;
  p->hp = *hp;
  const bool two_sided = hp->mode == MUON_MODE_TWOSIDED;
  p->ns_steps = two_sided ? 0 : hp->ns_steps;
  // the two-sided mode keeps U in fp32 and needs the row / column sums
  p->x_fp32 = (hp->flags & MUON_NS_FP32) != 0 || two_sided;
  p->equilibrate = (hp->flags & MUON_EQUILIBRATE) != 0 || two_sided;
  p->dev.resize(n);
  for (int i = 0; i < n; ++i) {
    const muon_matrix_t& m = mats[i];
    DevMat d{};
    d.W = static_cast<float*>(m.W);
    d.G = m.grad;
    d.M = static_cast<float*>(m.momentum);
    d.ld_w = m.ld_w;
    d.ld_g = m.ld_g;
    d.ld_m = m.ld_m;
    d.rows = static_cast<int32_t>(m.rows);
    d.cols = static_cast<int32_t>(m.cols);
    const bool gb = m.g_dtype == MUON_BF16;
    d.flags = (m.rows > m.cols ? MAT_TRANSPOSED : 0) | (gb ? MAT_G_BF16 : 0) |
              vec_flag(m.W, m.grad, m.momentum, m.ld_w, m.ld_g, m.ld_m, 4, gb ? 2 : 4, 4);
    d.orig = i;
    p->dev[i] = d;
  }
  build_plan(p);
  return p;
}

muon_plan_s* make_ns_plan(const muon_ns_matrix_t* mats, int n, const muon_hparams_t* hp) {
  muon_plan_s* p = new (std::nothrow) muon_plan_s();
  if (p == nullptr) return nullptr;
  p->ns_only = true;
  p->n = n;
  p->hp = *hp;
  p->ns_steps = hp->ns_steps;
  p->x_fp32 = (hp->flags & MUON_NS_FP32) != 0;
  p->equilibrate = false;
  p->dev.resize(n);
  for (int i = 0; i < n; ++i) {
    const muon_ns_matrix_t& m = mats[i];
    const bool b = m.dtype == MUON_BF16;
    DevMat d{};
    d.W = static_cast<float*>(m.O);  // output
    d.G = m.X;                        // input
    d.M = nullptr;
    d.ld_w = m.ld_o;
    d.ld_g = m.ld_x;
    d.ld_m = 0;
    d.rows = static_cast<int32_t>(m.rows);
    d.cols = static_cast<int32_t>(m.cols);
    d.flags = (m.rows > m.cols ? MAT_TRANSPOSED : 0) | (b ? MAT_G_BF16 : 0) |
              vec_flag(m.O, m.X, nullptr, m.ld_o, m.ld_x, 0, b ? 2 : 4, b ? 2 : 4, 4);
    d.orig = i;
    p->dev[i] = d;
  }
  build_plan(p);
  return p;
}

// Per-device facts, queried once. `info` packs them (bit 31: queried, bit 30: sm_100,
// low bits: SM count) so that a thread reads either nothing or the whole record.
std::atomic<uint32_t> g_dev_info[kMaxDevices];

muon_status_t current_device(int* dev, int* num_sms) {
  if (cudaGetDevice(dev) != cudaSuccess) return MUON_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return MUON_ERR_UNSUPPORTED;
  uint32_t info = g_dev_info[*dev].load(std::memory_order_acquire);
  if (!(info & 0x80000000u)) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
      return MUON_ERR_CUDA;
    info = 0x80000000u | ((major == 10 && minor == 0) ? 0x40000000u : 0u) |
           (static_cast<uint32_t>(sms) & 0xFFFFu);
    g_dev_info[*dev].store(info, std::memory_order_release);
  }
  if (!(info & 0x40000000u)) return MUON_ERR_UNSUPPORTED;
  *num_sms = static_cast<int>(info & 0xFFFFu);
  return MUON_OK;
}

// Binds the plan to a workspace: absolute slab pointers, tensor maps, and the
// device copy of the descriptor tables.
muon_status_t bind_workspace(muon_plan_s* p, void* ws, int dev, cudaStream_t stream) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int n = p->n;
  const int steps = p->ns_steps;
  std::vector<DevSlab> slabs(n);
  for (size_t c = 0; c < p->classes.size(); ++c) {
    const ClassInfo& ci = p->classes[c];
    for (int i = 0; i < ci.count; ++i) {
      DevSlab s{};
      s.x0 = base + ci.off_x[0] + ci.xbytes * i;
      s.xf = base + ci.off_x[steps % 2] + ci.xbytes * i;
      s.ldx = ci.ldx;
      s.cls = static_cast<int32_t>(c);
      s.eq_off = p->eq_off[ci.first + i];
      slabs[ci.first + i] = s;
    }
  }
  p->maps.clear();
  if (!p->x_fp32 && steps > 0) {
    p->maps.resize(p->classes.size());
    for (size_t c = 0; c < p->classes.size(); ++c) {
      const ClassInfo& ci = p->classes[c];
      ClassMaps& cm = p->maps[c];
      bool ok = true;
      for (int b = 0; b < 2; ++b) {
        ok = ok && encode_slab_map_bf16(&cm.x128[b], base + ci.off_x[b], ci.n, ci.m, ci.count, ci.ldx, 64, 128);
        ok = ok && encode_chunk_map_bf16(&cm.xmn[b], base + ci.off_x[b], ci.n, ci.m, ci.count, ci.ldx,
                                         ci.m % kPairTile == 0 ? 2 : tc_block_n(PH_APPLY) / 64);
        ok = ok && encode_slab_map_bf16(&cm.x32[b], base + ci.off_x[b], ci.n, ci.m, ci.count, ci.ldx, 64, 32);
        ok = ok && encode_slab_map_bf16(&cm.x64[b], base + ci.off_x[b], ci.n, ci.m, ci.count, ci.ldx, 64, 64);
      }
      ok = ok && encode_slab_map_bf16(&cm.s64, base + ci.off_s, ci.m, ci.m, ci.count, ci.lds, 64, 64);
      ok = ok && encode_chunk_map_bf16(&cm.smir1, base + ci.off_s, ci.m, ci.m, ci.count, ci.lds, 1);
      ok = ok && encode_slab_map_bf16(&cm.s32, base + ci.off_s, ci.m, ci.m, ci.count, ci.lds, 64, 32);
      ok = ok && encode_slab_map_bf16(&cm.p32, base + ci.off_p, ci.m, ci.m, ci.count, ci.lds, 64, 32);
      ok = ok && encode_slab_map_bf16(&cm.s128, base + ci.off_s, ci.m, ci.m, ci.count, ci.lds, 64, 128);
      ok = ok && encode_chunk_map_bf16(&cm.smir, base + ci.off_s, ci.m, ci.m, ci.count, ci.lds, 2);
      ok = ok && encode_slab_map_bf16(&cm.p128, base + ci.off_p, ci.m, ci.m, ci.count, ci.lds, 64, 128);
      ok = ok && encode_chunk_map_bf16(&cm.pmir, base + ci.off_p, ci.m, ci.m, ci.count, ci.lds, 2);
      if (!ok) return MUON_ERR_CUDA;
    }
  }
  // one upload of [desc | slabs | tiles]
  const size_t lo = p->off_desc, hi = p->off_otiles + sizeof(int32_t) * (n + 1);
  std::vector<uint8_t> host(hi - lo, 0);
  std::memcpy(host.data() + (p->off_desc - lo), p->dev.data(), sizeof(DevMat) * n);
  std::memcpy(host.data() + (p->off_slabs - lo), slabs.data(), sizeof(DevSlab) * n);
  std::memcpy(host.data() + (p->off_tiles - lo), p->tile_prefix.data(), sizeof(int32_t) * (n + 1));
  std::memcpy(host.data() + (p->off_otiles - lo), p->o_tile_prefix.data(), sizeof(int32_t) * (n + 1));
  if (cudaMemcpyAsync(base + lo, host.data(), host.size(), cudaMemcpyHostToDevice, stream) !=
      cudaSuccess)
    return MUON_ERR_CUDA;
  // a fresh workspace starts with a clear device error word
  if (cudaMemsetAsync(base, 0, sizeof(WsHeader), stream) != cudaSuccess) return MUON_ERR_CUDA;
  p->ws_cached = ws;
  p->dev_cached = dev;
  return MUON_OK;
}

// var_sym: the single-CTA tensor-core kernel, whose symmetric phases cut each 128-row
// block into variable-width pieces (sym_piece) instead of bn x bn tiles.
void fill_class_args(const muon_plan_s* p, uint8_t* base, size_t c, int phase, int it,
                     NsClassArgs* k, int bm, int bn, int bk, bool var_sym = false) {
  const ClassInfo& ci = p->classes[c];
  const int esz = p->x_fp32 ? 4 : 2;
  k->m = ci.m;
  k->n = ci.n;
  k->count = ci.count;
  k->first = ci.first;
  k->ldx = ci.ldx;
  k->lds = ci.lds;
  k->xstride = ci.xbytes / esz;
  k->sstride = ci.sbytes / esz;
  k->x_in = base + ci.off_x[it % 2];
  k->x_out = base + ci.off_x[(it + 1) % 2];
  k->s = base + ci.off_s;
  k->p = base + ci.off_p;
  const int ncols = phase == PH_APPLY ? ci.n : ci.m;
  k->tiles_i = (ci.m + bm - 1) / bm;
  k->tiles_j = (ncols + bn - 1) / bn;
  k->tiles_per_mat = phase == PH_APPLY ? k->tiles_i * k->tiles_j : k->tiles_i * (k->tiles_i + 1) / 2;
  if (var_sym && phase != PH_APPLY) k->tiles_per_mat = sym_tiles_per_matrix(ci.m);
  const int K = phase == PH_GRAM ? ci.n : ci.m;
  k->k_blocks = (K + bk - 1) / bk;
}

enum ProfKind { PK_INGEST = 0, PK_GRAM, PK_POLY, PK_APPLY, PK_REDUCE, PK_FINALIZE, PK_POST,
                PK_NS_FUSED, PK_STATS, PK_COUNT };
const char* const kProfNames[PK_COUNT] = {"ingest", "ns_gram", "ns_poly", "ns_apply",
                                          "post_reduce", "post_finalize", "post_apply",
                                          "ns_fused", "post_stats"};
constexpr size_t kMaxProfRecs = 1 << 16;

cudaEvent_t prof_event(muon_plan_s* p) {
  if (!p->event_pool.empty()) {
    cudaEvent_t e = p->event_pool.back();
    p->event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets one launch with events when profiling is on.
struct ProfScope {
  muon_plan_s* p;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  ProfScope(muon_plan_s* plan, cudaStream_t stream) : p(plan), s(stream) {
    if (p->prof && p->recs.size() < kMaxProfRecs) {
      a = prof_event(p);
      if (a != nullptr && cudaEventRecord(a, s) != cudaSuccess) {
        p->event_pool.push_back(a);
        a = nullptr;
      }
    }
  }
  void done(int kind, double flops, double bytes) {
    if (a == nullptr) return;
    cudaEvent_t b = prof_event(p);
    if (b == nullptr || cudaEventRecord(b, s) != cudaSuccess) {
      p->event_pool.push_back(a);
      if (b) p->event_pool.push_back(b);
      a = nullptr;
      return;
    }
    p->recs.push_back({a, b, kind, flops, bytes});
    a = nullptr;
  }
};

double class_phase_flops(const ClassInfo& ci, int phase) {
  const double m = ci.m, n = ci.n;
  double f = phase == PH_GRAM ? m * (m + 1) * n : (phase == PH_POLY ? m * m * (m + 1) : 2 * m * m * n);
  return f * ci.count;
}

// Muon and the two-sided mode: no step scalar depends on W, so the reduction reads
// the Newton-Schulz slab alone and post_apply gathers the statistics' W sums.
bool w_free_mode(const muon_plan_s* p) {
  return !p->ns_only && (p->hp.mode == MUON_MODE_MUON || p->hp.mode == MUON_MODE_TWOSIDED);
}

double elem_bytes(const muon_plan_s* p, int kind) {
  const int ex = p->x_fp32 ? 4 : 2;
  double total = 0;
  for (const DevMat& d : p->dev) {
    const double e = double(d.rows) * d.cols;
    const int eg = (d.flags & MAT_G_BF16) ? 2 : 4;
    if (kind == PK_INGEST) total += e * (p->ns_only ? eg + ex : eg + 8 + ex);
    else if (kind == PK_REDUCE) total += e * (w_free_mode(p) ? ex : 4 + ex);
    else if (kind == PK_POST) total += e * (p->ns_only ? eg + ex : 8 + ex);
  }
  return total;
}

// Enqueues one step (memsets and kernel launches only, so it can be captured) on
// `stream`, for a plan already bound to workspace `ws` on the current device.
muon_status_t enqueue_step(muon_plan_s* p, void* ws, muon_stats_t* stats, int num_sms,
                           cudaStream_t stream) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int n = p->n;
  const muon_hparams_t& hp = p->hp;
  // the per-matrix scalars and the statistics' sums of post_apply (adjacent)
  if (cudaMemsetAsync(base + p->off_scal, 0, p->off_asum - p->off_scal + sizeof(ApplySums) * n, stream) !=
      cudaSuccess)
    return MUON_ERR_CUDA;
  if (p->eq_total > 0) {
    if (cudaMemsetAsync(base + p->off_eq_o2, 0, p->off_eq_wo - p->off_eq_o2 + sizeof(float) * p->eq_total,
                        stream) != cudaSuccess)
      return MUON_ERR_CUDA;
  }
  ElemArgs ea{};
  ea.mats = reinterpret_cast<const DevMat*>(base + p->off_desc);
  ea.slabs = reinterpret_cast<const DevSlab*>(base + p->off_slabs);
  ea.tile_prefix = reinterpret_cast<const int32_t*>(base + p->off_tiles);
  ea.n = n;
  ea.total_tiles = p->tile_prefix[n];
  ea.scal = reinterpret_cast<MatScalars*>(base + p->off_scal);
  ea.coef = reinterpret_cast<MatCoef*>(base + p->off_coef);
  ea.eq_o2 = reinterpret_cast<float*>(base + p->off_eq_o2);
  ea.eq_wo = reinterpret_cast<float*>(base + p->off_eq_wo);
  ea.stats = p->ns_only ? nullptr : stats;
  ea.err = reinterpret_cast<uint32_t*>(base);
  ea.mu = hp.momentum;
  ea.lr = hp.lr;
  ea.wd = hp.weight_decay;
  ea.eps = hp.eps;
  ea.scale_k = hp.scale_k;
  ea.scale_rule = hp.scale;
  ea.mode = hp.mode;
  ea.nesterov = (hp.flags & MUON_NESTEROV) ? 1 : 0;
  ea.ns_only = p->ns_only ? 1 : 0;
  ea.x_fp32 = p->x_fp32 ? 1 : 0;
  ea.equilibrate = p->equilibrate ? 1 : 0;
  ea.xs_from_u2 = p->ns_steps == 0 ? 1 : 0;
  ea.sub_r = p->sub_r;
  ea.sub_c = p->sub_c;
  ea.staged = p->staged ? 1 : 0;
  ea.staged_in = p->staged_in ? 1 : 0;
  ea.w_free = w_free_mode(p) ? 1 : 0;
  ea.apply_stats = (ea.w_free && stats != nullptr) ? 1 : 0;
  ea.o_tile_prefix = reinterpret_cast<const int32_t*>(base + p->off_otiles);
  ea.o_total_tiles = p->o_tile_prefix[n];
  ea.asum = reinterpret_cast<ApplySums*>(base + p->off_asum);

  {
    ProfScope ps(p, stream);
    if (launch_ingest(ea, stream) != cudaSuccess) return MUON_ERR_CUDA;
    ps.done(PK_INGEST, 0.0, elem_bytes(p, PK_INGEST));
  }

  // Newton-Schulz phases, at most kMaxClassesPerLaunch classes per launch
  const int nc = static_cast<int>(p->classes.size());
  // fp32 path: small classes run every iteration in one fused launch; the others take
  // one launch per phase
  std::vector<int> fp32_small, fp32_large;
  for (int c = 0; p->x_fp32 && c < nc; ++c)
    (simt_fused_fits(p->classes[c].m, p->classes[c].n) ? fp32_small : fp32_large).push_back(c);
  for (size_t g0 = 0; p->ns_steps > 0 && g0 < fp32_small.size(); g0 += kMaxClassesPerLaunch) {
    const int cn = static_cast<int>(std::min<size_t>(kMaxClassesPerLaunch, fp32_small.size() - g0));
    NsFusedArgs a{};
    a.num_classes = cn;
    a.steps = p->ns_steps;
    a.a = hp.ns_coeffs[0];
    a.b = hp.ns_coeffs[1];
    a.c = hp.ns_coeffs[2];
    a.eps = hp.eps;
    a.scal = ea.scal;
    int mats = 0;
    double fl = 0;
    for (int c = 0; c < cn; ++c) {
      const int cid = fp32_small[g0 + c];
      fill_class_args(p, base, cid, PH_GRAM, 0, &a.cls[c], 32, 32, 16);
      a.x0[c] = base + p->classes[cid].off_x[0];
      a.x1[c] = base + p->classes[cid].off_x[1];
      a.mat_base[c] = mats;
      mats += a.cls[c].count;
      for (int ph = PH_GRAM; ph <= PH_APPLY; ++ph) fl += p->ns_steps * class_phase_flops(p->classes[cid], ph);
    }
    a.mat_base[cn] = mats;
    ProfScope ps(p, stream);
    if (launch_ns_simt_fused(a, stream) != cudaSuccess) return MUON_ERR_CUDA;
    ps.done(PK_NS_FUSED, fl, 0.0);
  }
  for (int it = 0; it < p->ns_steps; ++it) {
    for (int phase = PH_GRAM; phase <= PH_APPLY; ++phase) {
      for (size_t g0 = 0; g0 < fp32_large.size(); g0 += kMaxClassesPerLaunch) {
        const int cn = static_cast<int>(std::min<size_t>(kMaxClassesPerLaunch, fp32_large.size() - g0));
        {
          NsPhaseArgs a{};
          a.num_classes = cn;
          a.phase = phase;
          a.a = hp.ns_coeffs[0];
          a.b = hp.ns_coeffs[1];
          a.c = hp.ns_coeffs[2];
          a.first_iter = it == 0 ? 1 : 0;
          a.eps = hp.eps;
          a.scal = ea.scal;
          a.err = ea.err;
          int tiles = 0;
          for (int c = 0; c < cn; ++c) {
            fill_class_args(p, base, fp32_large[g0 + c], phase, it, &a.cls[c], 64, 64, 16);
            a.tile_base[c] = tiles;
            tiles += a.cls[c].count * a.cls[c].tiles_per_mat;
          }
          a.tile_base[cn] = tiles;
          ProfScope ps(p, stream);
          if (launch_ns_phase_simt(a, stream) != cudaSuccess) return MUON_ERR_CUDA;
          double fl = 0;
          for (int c = 0; c < cn; ++c) fl += class_phase_flops(p->classes[fp32_large[g0 + c]], phase);
          ps.done(PK_GRAM + phase, fl, 0.0);
        }
      }
      if (!p->x_fp32) {
        // tensor cores: classes with m a multiple of 256 run on CTA pairs (256 x 256
        // tiles), the others on single CTAs; at most kMaxClassesPerLaunch per launch
        for (int pair = 1; pair >= 0; --pair) {
          std::vector<int> ids;
          for (int c = 0; c < nc; ++c)
            if ((p->classes[c].m % kPairTile == 0) == (pair == 1)) ids.push_back(c);
          for (size_t g0 = 0; g0 < ids.size(); g0 += kMaxClassesPerLaunch) {
            const int cn = static_cast<int>(std::min<size_t>(kMaxClassesPerLaunch, ids.size() - g0));
            TcParams P;
            std::memset(&P, 0, sizeof(P));
            NsPhaseArgs& a = P.args;
            a.num_classes = cn;
            a.phase = phase;
            a.a = hp.ns_coeffs[0];
            a.b = hp.ns_coeffs[1];
            a.c = hp.ns_coeffs[2];
            a.first_iter = it == 0 ? 1 : 0;
            a.eps = hp.eps;
            a.scal = ea.scal;
            a.err = ea.err;
            int tiles = 0;
            double fl = 0;
            for (int c = 0; c < cn; ++c) {
              const int cid = ids[g0 + c];
              const ClassMaps& cm = p->maps[cid];
              const int bm = pair ? kPairTile : tc_block_m();
              const int bn = pair ? kPairTile : tc_block_n(phase);
              fill_class_args(p, base, cid, phase, it, &a.cls[c], bm, bn, tc_block_k(), !pair);
              a.tile_base[c] = tiles;
              tiles += a.cls[c].count * a.cls[c].tiles_per_mat;
              fl += class_phase_flops(p->classes[cid], phase);
              // S and P' hold only their blocks on or above the (tile) diagonal; the
              // *_t maps fetch mirror blocks for the operands below it
              // (single-CTA symmetric phases take B in 64-row units: 64 x 64 boxes or
              // one-chunk mirrors)
              if (phase == PH_GRAM) {
                P.ta[c] = P.ta_t[c] = cm.x128[it % 2];
                P.tb[c] = P.tb_t[c] = pair ? cm.x128[it % 2] : cm.x64[it % 2];
                P.tc[c] = cm.s128;
                P.td[c] = cm.s32;
              } else if (phase == PH_POLY) {
                P.ta[c] = cm.s128;
                P.ta_t[c] = cm.smir;
                P.tb[c] = pair ? cm.s128 : cm.s64;
                P.tb_t[c] = pair ? cm.smir : cm.smir1;
                P.tc[c] = cm.s128;
                P.td[c] = cm.p32;
              } else {
                P.ta[c] = cm.p128;
                P.ta_t[c] = cm.pmir;
                P.tb[c] = P.tb_t[c] = cm.xmn[it % 2];
                P.tc[c] = cm.x128[it % 2];
                P.td[c] = cm.x32[(it + 1) % 2];
              }
            }
            a.tile_base[cn] = tiles;
            ProfScope ps(p, stream);
            const cudaError_t e = pair ? launch_ns_phase_tc_pair(P, num_sms, stream)
                                       : launch_ns_phase_tc(P, num_sms, stream);
            if (e != cudaSuccess) return MUON_ERR_CUDA;
            ps.done(PK_GRAM + phase, fl, 0.0);
          }
        }
      }
    }
  }

  if (!p->ns_only) {
    // MuonGS and MuonH need <W,O> and ||W|| before the update; Muon and the two-sided
    // mode need O sums only with equilibration (their statistics come from post_apply)
    const bool need_reduce = ea.w_free ? p->equilibrate : true;
    if (need_reduce) {
      ProfScope ps(p, stream);
      if (launch_post_reduce(ea, stream) != cudaSuccess) return MUON_ERR_CUDA;
      ps.done(PK_REDUCE, 0.0, elem_bytes(p, PK_REDUCE));
    }
    ProfScope ps(p, stream);
    if (launch_post_finalize(ea, stream) != cudaSuccess) return MUON_ERR_CUDA;
    ps.done(PK_FINALIZE, 0.0, 0.0);
  }
  {
    ProfScope ps(p, stream);
    if (launch_post_apply(ea, stream) != cudaSuccess) return MUON_ERR_CUDA;
    ps.done(PK_POST, 0.0, elem_bytes(p, PK_POST));
  }
  if (ea.apply_stats) {
    ProfScope ps(p, stream);
    if (launch_post_stats(ea, stream) != cudaSuccess) return MUON_ERR_CUDA;
    ps.done(PK_STATS, 0.0, 0.0);
  }
  return MUON_OK;
}

// Captures one step of a bound plan into a CUDA graph on the plan's private stream.
// With an executable of the same launch sequence already instantiated (only scalar
// kernel arguments changed, e.g. a learning-rate schedule), the executable is updated
// in place (cudaGraphExecUpdate) instead of being instantiated again.
muon_status_t capture_step(muon_plan_s* p, void* ws, muon_stats_t* stats, int dev, int num_sms) {
  cudaGraphExec_t old_exec = p->graph_stale ? p->graph_exec : nullptr;
  if (old_exec == nullptr) p->drop_graph();
  p->graph_stale = false;
  if (p->cap_stream == nullptr &&
      cudaStreamCreateWithFlags(&p->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  if (cudaStreamBeginCapture(p->cap_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  const muon_status_t st = enqueue_step(p, ws, stats, num_sms, p->cap_stream);
  cudaGraph_t graph = nullptr;
  const cudaError_t e = cudaStreamEndCapture(p->cap_stream, &graph);
  if (st != MUON_OK || e != cudaSuccess || graph == nullptr) {
    if (graph != nullptr) cudaGraphDestroy(graph);
    cudaGetLastError();
    p->drop_graph();
    return MUON_ERR_CUDA;
  }
  if (old_exec != nullptr) {
    cudaGraphExecUpdateResultInfo info;
    if (cudaGraphExecUpdate(old_exec, graph, &info) == cudaSuccess) {
      cudaGraphDestroy(graph);
      p->graph_ws = ws;
      p->graph_stats = stats;
      p->graph_dev = dev;
      return MUON_OK;  // same executable, new arguments
    }
    cudaGetLastError();
    p->drop_graph();   // topology differs: instantiate afresh
  }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t ei = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (ei != cudaSuccess || exec == nullptr) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  p->graph_exec = exec;
  p->graph_ws = ws;
  p->graph_stats = stats;
  p->graph_dev = dev;
  return MUON_OK;
}

muon_status_t run_plan(muon_plan_s* p, void* ws, size_t ws_bytes, muon_stats_t* stats,
                       cudaStream_t stream) {
  if (p->n == 0) return MUON_OK;
  if (ws == nullptr || reinterpret_cast<uintptr_t>(ws) % kAlign != 0 || ws_bytes < p->ws_bytes)
    return MUON_ERR_WORKSPACE;
  int dev = 0, num_sms = 0;
  muon_status_t st = current_device(&dev, &num_sms);
  if (st != MUON_OK) return st;
  p->num_sms = num_sms;
  if (p->ws_cached != ws || p->dev_cached != dev) {
    p->drop_graph();
    st = bind_workspace(p, ws, dev, stream);
    if (st != MUON_OK) return st;
  }
  if (p->use_graph && p->graph_ok && !p->prof) {
    const bool same = p->graph_exec != nullptr && !p->graph_stale && p->graph_ws == ws &&
                      p->graph_stats == stats && p->graph_dev == dev;
    if (!same && p->eager_steps > 0 && capture_step(p, ws, stats, dev, num_sms) != MUON_OK)
      p->graph_ok = false;  // stay eager
    if (p->graph_ok && p->graph_exec != nullptr && p->graph_ws == ws && p->graph_stats == stats &&
        p->graph_dev == dev)
      return cudaGraphLaunch(p->graph_exec, stream) == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
  }
  ++p->eager_steps;
  return enqueue_step(p, ws, stats, num_sms, stream);
}

}  // namespace

extern "C" {

int muon_abi_version(void) { return MUON_ABI_VERSION; }

const char* muon_status_string(muon_status_t s) {
  switch (s) {
    case MUON_OK: return "MUON_OK";
    case MUON_ERR_INVALID_ARG: return "MUON_ERR_INVALID_ARG";
    case MUON_ERR_SHAPE: return "MUON_ERR_SHAPE";
    case MUON_ERR_DTYPE: return "MUON_ERR_DTYPE";
    case MUON_ERR_ALIAS: return "MUON_ERR_ALIAS";
    case MUON_ERR_WORKSPACE: return "MUON_ERR_WORKSPACE";
    case MUON_ERR_CUDA: return "MUON_ERR_CUDA";
    case MUON_ERR_TIMEOUT: return "MUON_ERR_TIMEOUT";
    case MUON_ERR_UNSUPPORTED: return "MUON_ERR_UNSUPPORTED";
  }
  return "MUON_ERR_UNKNOWN";
}

muon_status_t muon_hparams_default(muon_hparams_t* hp) {
  if (hp == nullptr) return MUON_ERR_INVALID_ARG;
  std::memset(hp, 0, sizeof(*hp));
  hp->lr = 0.02f;
  hp->momentum = 0.95f;
  hp->weight_decay = 0.f;
  hp->ns_coeffs[0] = 3.4445f;
  hp->ns_coeffs[1] = -4.7750f;
  hp->ns_coeffs[2] = 2.0315f;
  hp->ns_steps = 5;
  hp->eps = 1e-7f;
  hp->mode = MUON_MODE_MUON;
  hp->scale = MUON_SCALE_MOONLIGHT;
  hp->scale_k = 0.2f;
  hp->flags = MUON_NESTEROV;
  return MUON_OK;
}

muon_status_t muon_validate(const muon_matrix_t* mats, int n, const muon_hparams_t* hp) {
  return validate_step(mats, n, hp);
}

size_t muon_workspace_size(const muon_matrix_t* mats, int n, const muon_hparams_t* hp) {
  if (validate_step(mats, n, hp) != MUON_OK) return 0;
  muon_plan_s* p = make_step_plan(mats, n, hp);
  if (p == nullptr) return 0;
  const size_t s = p->ws_bytes;
  delete p;
  return s;
}

muon_status_t muon_step_batched(const muon_matrix_t* mats, int n, const muon_hparams_t* hp,
                                void* workspace, size_t ws_bytes, muon_stats_t* stats_dev,
                                void* stream) {
  muon_status_t st = validate_step(mats, n, hp);
  if (st != MUON_OK || n == 0) return st;
  muon_plan_s* p = make_step_plan(mats, n, hp);
  if (p == nullptr) return MUON_ERR_INVALID_ARG;
  st = run_plan(p, workspace, ws_bytes, stats_dev, static_cast<cudaStream_t>(stream));
  delete p;
  return st;
}

muon_status_t muon_plan_create(const muon_matrix_t* mats, int n, const muon_hparams_t* hp,
                               muon_plan_t* out) {
  if (out == nullptr) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  muon_status_t st = validate_step(mats, n, hp);
  if (st != MUON_OK) return st;
  muon_plan_s* p = make_step_plan(mats, n, hp);
  if (p == nullptr) return MUON_ERR_INVALID_ARG;
  p->use_graph = true;
  *out = p;
  return MUON_OK;
}

size_t muon_plan_workspace_size(muon_plan_t plan) { return plan ? plan->ws_bytes : 0; }

muon_status_t muon_plan_set_hparams(muon_plan_t plan, const muon_hparams_t* hp) {
  if (plan == nullptr || hp == nullptr || !valid_enum_hp(hp)) return MUON_ERR_INVALID_ARG;
  const uint32_t layout = MUON_NS_FP32 | MUON_EQUILIBRATE;
  if ((hp->flags & layout) != (plan->hp.flags & layout)) return MUON_ERR_INVALID_ARG;
  if ((hp->mode == MUON_MODE_TWOSIDED) != (plan->hp.mode == MUON_MODE_TWOSIDED))
    return MUON_ERR_INVALID_ARG;
  const int steps = hp->mode == MUON_MODE_TWOSIDED ? 0 : hp->ns_steps;
  if ((steps == 0) != (plan->ns_steps == 0)) return MUON_ERR_INVALID_ARG;
  const bool parity_changed = (steps % 2) != (plan->ns_steps % 2);
  const bool same_launches = steps == plan->ns_steps && hp->mode == plan->hp.mode &&
                             (hp->mode == MUON_MODE_MUON) == (plan->hp.mode == MUON_MODE_MUON);
  plan->hp = *hp;
  plan->ns_steps = steps;
  // the captured launches hold the old values: with the same launch sequence the next
  // step updates the executable in place, otherwise it is captured afresh
  if (same_launches && plan->graph_exec != nullptr) plan->graph_stale = true;
  else plan->drop_graph();
  if (parity_changed) plan->ws_cached = nullptr;  // the result slab moved: re-upload
  return MUON_OK;
}

muon_status_t muon_plan_step(muon_plan_t plan, void* workspace, size_t ws_bytes,
                             muon_stats_t* stats_dev, void* stream) {
  if (plan == nullptr) return MUON_ERR_INVALID_ARG;
  return run_plan(plan, workspace, ws_bytes, stats_dev, static_cast<cudaStream_t>(stream));
}

void muon_plan_destroy(muon_plan_t plan) { delete plan; }

muon_status_t muon_plan_profile_enable(muon_plan_t plan, int enable) {
  if (plan == nullptr) return MUON_ERR_INVALID_ARG;
  plan->prof = enable != 0;
  return MUON_OK;
}

int muon_plan_profile_read(muon_plan_t plan, muon_profile_entry_t* out, int max_entries) {
  if (plan == nullptr || (out == nullptr && max_entries > 0) || max_entries < 0) return -1;
  muon_profile_entry_t acc[PK_COUNT];
  std::memset(acc, 0, sizeof(acc));
  for (int k = 0; k < PK_COUNT; ++k) std::strncpy(acc[k].name, kProfNames[k], sizeof(acc[k].name) - 1);
  bool ok = true;
  for (const auto& r : plan->recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      ok = false;
    acc[r.kind].launches += 1;
    acc[r.kind].total_ms += ms;
    acc[r.kind].flops += r.flops;
    acc[r.kind].bytes += r.bytes;
    plan->event_pool.push_back(r.a);
    plan->event_pool.push_back(r.b);
  }
  plan->recs.clear();
  if (!ok) return -1;
  const int nw = std::min(max_entries, static_cast<int>(PK_COUNT));
  for (int k = 0; k < nw; ++k) out[k] = acc[k];
  return nw;
}

size_t muon_ns_workspace_size(const muon_ns_matrix_t* mats, int n, const muon_hparams_t* hp) {
  if (validate_ns(mats, n, hp) != MUON_OK) return 0;
  muon_plan_s* p = make_ns_plan(mats, n, hp);
  if (p == nullptr) return 0;
  const size_t s = p->ws_bytes;
  delete p;
  return s;
}

muon_status_t muon_newton_schulz_batched(const muon_ns_matrix_t* mats, int n,
                                         const muon_hparams_t* hp, void* workspace,
                                         size_t ws_bytes, void* stream) {
  muon_status_t st = validate_ns(mats, n, hp);
  if (st != MUON_OK || n == 0) return st;
  muon_plan_s* p = make_ns_plan(mats, n, hp);
  if (p == nullptr) return MUON_ERR_INVALID_ARG;
  st = run_plan(p, workspace, ws_bytes, nullptr, static_cast<cudaStream_t>(stream));
  delete p;
  return st;
}

muon_status_t muon_query_device_status(void* workspace, void* stream) {
  if (workspace == nullptr) return MUON_ERR_INVALID_ARG;
  // ordered on `stream` only: the read follows the work enqueued there, the clear
  // is enqueued behind it, and no other stream of the caller is waited for
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MUON_ERR_CUDA;
  if (word != 0 && (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess ||
                    cudaStreamSynchronize(s) != cudaSuccess))
    return MUON_ERR_CUDA;
  return word == 0 ? MUON_OK : static_cast<muon_status_t>(word);
}

}  // extern "C"
