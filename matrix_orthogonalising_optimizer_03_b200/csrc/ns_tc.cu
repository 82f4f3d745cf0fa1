// bf16 Newton-Schulz phases on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The three contractions of one iteration X <- aX + b(XX^T)X + c(XX^T)^2 X (the
// Newton-Schulz listing of "LLM Pretraining Loss Spike 진단과 처방", section "Muon
// head의 실체는 하이브리드 옵티마이저다"; section 2 of the "MUON IS SCALABLE FOR LLM
// TRAINING" review) as three grouped GEMM launches over every matrix of every
// shape class in the call:
//   GRAM   S  = alpha * X X^T        A = X (K-major), B = X (K-major), K = n
//   POLY   P  = b*S + c * S S        A = S (K-major), B = S (K-major, S = S^T), K = m
//   APPLY  X' = gamma * (a*X + P X)  A = P (K-major), B = X (MN-major), K = m
// GRAM and POLY have symmetric outputs: only tiles with ti <= tj are computed and
// each off-diagonal tile is stored twice (direct and mirrored).
// alpha = 1/(||U||+eps)^2, gamma = 1/(||U||+eps) on the first iteration (the
// slab holds the unnormalised U), 1 afterwards. X, S, P are stored in bf16,
// accumulation is fp32 in TMEM.
//
// Kernel structure (persistent, one CTA per SM, 192 threads):
//   warp 0   TMA producer: 128 x 64 A box and the B boxes into a STAGES-deep
//            ring of 128B-swizzled shared-memory stages (no multicast).
//   warp 1   TMEM allocator and MMA issuer: tcgen05.mma.cta_group::1.kind::f16,
//            M=128, N=BN, K=16 per instruction, into one of two TMEM accumulators.
//   warps 2-5 epilogue: tcgen05.ld 32 lanes x 32 columns, fused scale / axpy with
//            the bf16 C operand, bf16 stores (and mirrored stores).
// Slabs are [count][rows][ld] bf16 and are addressed by 3-D tensor maps
// (inner dim, rows, matrix), so out-of-range rows and columns of a matrix are
// zero-filled by TMA and never spill into the next matrix.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "muon_internal.h"
#include "ns_tc.h"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int BM = 128, BK = 64;
constexpr int kEpiWarps = 4;
constexpr int kThreadsTc = 192;

template <int BN>
struct TcCfg {
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
};

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
    while (rem >= k.tiles_i - ti) {
      rem -= k.tiles_i - ti;
      ++ti;
    }
    j.ti = ti;
    j.tj = ti + rem;
  } else {
    j.ti = rem / k.tiles_j;
    j.tj = rem - j.ti * k.tiles_j;
  }
  return j;
}

template <int BN, int PHASE>
__global__ void __launch_bounds__(kThreadsTc, 1) ns_tc_kernel(const __grid_constant__ TcParams P) {
  using C = TcCfg<BN>;
  constexpr bool SYM = PHASE != PH_APPLY;
  constexpr bool B_MN = PHASE == PH_APPLY;
  constexpr int S = C::kStages;
  static_assert(!SYM || BN == BM, "symmetric phases use square tiles");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const NsPhaseArgs& p = P.args;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.tile_base[p.num_classes];

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int c = 0; c < p.num_classes; ++c) {
        tma_prefetch(&P.ta[c]);
        tma_prefetch(&P.tb[c]);
      }
      long long q = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileJob j = decode(p, t, SYM);
        const int kb_n = p.cls[j.c].k_blocks;
        for (int kb = 0; kb < kb_n; ++kb) {
          const int s = static_cast<int>(q % S);
          const uint32_t par = static_cast<uint32_t>((q / S) & 1);
          if (!mbar_wait(&empty[s], par ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          mbar_expect_tx(&full[s], C::kStageBytes);
          tma_load_3d(sa, &P.ta[j.c], &full[s], kb * BK, j.ti * BM, j.mat);
          if (!B_MN) {
            tma_load_3d(sb, &P.tb[j.c], &full[s], kb * BK, j.tj * BN, j.mat);
          } else {
#pragma unroll
            for (int h = 0; h < BN / 64; ++h)
              tma_load_3d(sb + h * (64 * BK * 2), &P.tb[j.c], &full[s], j.tj * BN + h * 64,
                          kb * BK, j.mat);
          }
          ++q;
        }
      }
      if (!ok) {
        set_error(p.err, MUON_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      // Never leave the CTA with bulk copies still landing in its shared memory.
      for (long long r = (q > S ? q - S : 0); r < q; ++r)
        mbar_wait(&full[r % S], static_cast<uint32_t>((r / S) & 1), nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, B_MN);
      long long q = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const TileJob j = decode(p, t, SYM);
        const int kb_n = p.cls[j.c].k_blocks;
        const int ab = it & 1;
        const uint32_t apar = static_cast<uint32_t>((it >> 1) & 1);
        if (!mbar_wait(&tempty[ab], apar ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * BN);
        for (int kb = 0; kb < kb_n; ++kb) {
          const int s = static_cast<int>(q % S);
          const uint32_t par = static_cast<uint32_t>((q / S) & 1);
          if (!mbar_wait(&full[s], par, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::kStageBytes);
          const uint32_t sb = sa + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 64 * BK * 2, 1024)
                                     : smem_desc_sw128(sb + kk * 32, 16, 1024);
            umma_f16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);  // frees the stage once these MMAs have read it
          ++q;
        }
        if (!ok) break;
        umma_commit(&tfull[ab]);  // accumulator ready for the epilogue
      }
      if (!ok) {
        set_error(p.err, MUON_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      umma_commit(done);  // arrives once every MMA issued above has completed
      mbar_wait(done, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // the TMEM lane quarter this warp may access
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const TileJob j = decode(p, t, SYM);
      const NsClassArgs& k = p.cls[j.c];
      const int ab = it & 1;
      const uint32_t apar = static_cast<uint32_t>((it >> 1) & 1);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[ab], apar, abort_flag));
      if (!ok) {
        if (lane == 0) {
          set_error(p.err, MUON_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();

      const int m = k.m;
      const int ncols = PHASE == PH_APPLY ? k.n : m;
      const int row = j.ti * BM + quad * 32 + lane;
      float scale = 1.f;
      if (PHASE != PH_POLY && p.first_iter) {
        const double inv = 1.0 / (sqrt(p.scal[k.first + j.mat].u2) + (double)p.eps);
        scale = static_cast<float>(PHASE == PH_GRAM ? inv * inv : inv);
      }
      uint16_t* out;
      const uint16_t* cin = nullptr;
      int ldo;
      if (PHASE == PH_GRAM) {
        out = static_cast<uint16_t*>(k.s) + j.mat * k.sstride;
        ldo = k.lds;
      } else if (PHASE == PH_POLY) {
        out = static_cast<uint16_t*>(k.p) + j.mat * k.sstride;
        cin = static_cast<const uint16_t*>(k.s) + j.mat * k.sstride;
        ldo = k.lds;
      } else {
        out = static_cast<uint16_t*>(k.x_out) + j.mat * k.xstride;
        cin = static_cast<const uint16_t*>(k.x_in) + j.mat * k.xstride;
        ldo = k.ldx;
      }
      const bool row_ok = row < m;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                      static_cast<uint32_t>(ab * BN + ch * 32),
                  v);
        tmem_wait_ld();
        const int col0 = j.tj * BN + ch * 32;
        if (col0 >= ncols) continue;
        const int nv = min(32, ncols - col0);
        uint32_t packed[16];
        if (row_ok) {
          float cv[32];
          if (PHASE != PH_GRAM) {
            const uint16_t* cp = cin + (int64_t)row * ldo + col0;
            if (nv == 32) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const uint4 x = __ldg(reinterpret_cast<const uint4*>(cp) + q4);
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  cv[q4 * 8 + 2 * e] = __uint_as_float(w[e] << 16);
                  cv[q4 * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                }
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) cv[e] = e < nv ? bf16_to_f32(cp[e]) : 0.f;
            }
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float r0 = __uint_as_float(v[e]), r1 = __uint_as_float(v[e + 1]);
            if (PHASE == PH_GRAM) {
              r0 *= scale;
              r1 *= scale;
            } else if (PHASE == PH_POLY) {
              r0 = fmaf(p.b, cv[e], p.c * r0);
              r1 = fmaf(p.b, cv[e + 1], p.c * r1);
            } else {
              r0 = scale * fmaf(p.a, cv[e], r0);
              r1 = scale * fmaf(p.a, cv[e + 1], r1);
            }
            packed[e >> 1] = pack_bf16x2(r0, r1);
          }
          uint16_t* op = out + (int64_t)row * ldo + col0;
          if (nv == 32) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              reinterpret_cast<uint4*>(op)[q4] =
                  make_uint4(packed[4 * q4], packed[4 * q4 + 1], packed[4 * q4 + 2], packed[4 * q4 + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < nv) op[e] = static_cast<uint16_t>(packed[e >> 1] >> ((e & 1) * 16));
          }
          if (SYM && j.ti != j.tj) {
            // mirrored tile: element (col0+e, row); a warp writes 32 consecutive rows' column
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < nv)
                out[(int64_t)(col0 + e) * ldo + row] =
                    static_cast<uint16_t>(packed[e >> 1] >> ((e & 1) * 16));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int BN, int PHASE>
cudaError_t launch_one(const TcParams& P, int grid, cudaStream_t s) {
  using C = TcCfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(ns_tc_kernel<BN, PHASE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  ns_tc_kernel<BN, PHASE><<<grid, kThreadsTc, C::kSmemBytes, s>>>(P);
  return cudaGetLastError();
}

}  // namespace

int tc_block_n(int phase) { return phase == PH_APPLY ? 256 : 128; }
int tc_block_m() { return BM; }
int tc_block_k() { return BK; }

cudaError_t launch_ns_phase_tc(const TcParams& P, int num_sms, cudaStream_t s) {
  const int total = P.args.tile_base[P.args.num_classes];
  if (total <= 0) return cudaSuccess;
  const int grid = total < num_sms ? total : num_sms;
  switch (P.args.phase) {
    case PH_GRAM: return launch_one<128, PH_GRAM>(P, grid, s);
    case PH_POLY: return launch_one<128, PH_POLY>(P, grid, s);
    default: return launch_one<256, PH_APPLY>(P, grid, s);
  }
}

// Encodes a 3-D bf16 tensor map over a slab [count][rows][ld] with a
// box_inner x box_rows box (128B swizzle). Returns false on failure.
bool encode_slab_map_bf16(CUtensorMap* out, const void* base, int64_t inner, int64_t rows,
                          int64_t count, int64_t ld, int box_inner, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    cudaDriverEntryPointQueryResult qr;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess || fn == nullptr)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(count)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * 2),
                           static_cast<cuuint64_t>(rows * ld * 2)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace muon
