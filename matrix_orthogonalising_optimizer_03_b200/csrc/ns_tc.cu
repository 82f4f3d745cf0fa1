// bf16 Newton-Schulz phases on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The three contractions of one iteration X <- aX + b(XX^T)X + c(XX^T)^2 X (the
// Newton-Schulz listing of "LLM Pretraining Loss Spike 진단과 처방", section "Muon
// head의 실체는 하이브리드 옵티마이저다"; section 2 of the "MUON IS SCALABLE FOR LLM
// TRAINING" review) as three grouped GEMM launches over every matrix of every
// shape class in the call:
//   GRAM   S  = alpha * X X^T            A = X (K-major), B = X (K-major), K = n
//   POLY   P' = a*I + b*S + c * S S      A = S (K-major), B = S (K-major, S = S^T), K = m
//   APPLY  X' = gamma * P' X             A = P' (K-major), B = X (MN-major), K = m
// The a*X term of the recurrence is folded into P' (a*X + P X = (a I + P) X), so
// the apply epilogue needs no second read of X; P' is rounded to bf16 once, with
// its diagonal a + P_ii (about 0.7) in place of P_ii (about -2.7).
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

template <int BN, int PHASE>
struct TcCfg {
  static constexpr bool kHasC = PHASE == PH_POLY;       // epilogue reads a C tile (S)
  static constexpr bool kSym = PHASE != PH_APPLY;       // mirrored (transposed) store
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = BN == 256 ? 3 : 4;
  static constexpr int kTileBytes = BM * BN * 2;        // one bf16 output tile (C / D staging)
  static constexpr int kTBytes = kSym ? BN * BM * 2 : 0;  // transposed staging
  static constexpr int kOffD = kStages * kStageBytes;
  static constexpr int kOffT = kOffD + kTileBytes;
  static constexpr int kOffBar = kOffT + kTBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
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

// Byte offset of element (r, c) of a tile staged as 64-column boxes of 128 rows
// with the 128-byte swizzle (the layout TMA reads and writes for a 64 x 128 box).
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>((c >> 6) * (BM * 128) + r * 128 +
                               ((((c >> 3) & 7) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

template <int BN, int PHASE>
__global__ void __launch_bounds__(kThreadsTc, 1) ns_tc_kernel(const __grid_constant__ TcParams P) {
  using C = TcCfg<BN, PHASE>;
  constexpr bool SYM = C::kSym;
  constexpr bool HAS_C = C::kHasC;
  constexpr bool B_MN = PHASE == PH_APPLY;
  constexpr int S = C::kStages;
  static_assert(!SYM || BN == BM, "symmetric phases use square tiles");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* dtile = smem + C::kOffD;   // C tile in, D tile out (in place)
  uint8_t* ttile = smem + C::kOffT;   // transposed D (symmetric phases)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint64_t* cfull = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cfull + 1);
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
    mbar_init(cfull, 1);
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
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int quad = warp & 3;  // the TMEM lane quarter this warp may access
    const int r = quad * 32 + lane;  // tile row of this thread
    const bool leader = warp == 2 && lane == 0;
    bool c_pending = false;
    if (HAS_C && leader && static_cast<int>(blockIdx.x) < total) {
      const TileJob j = decode(p, blockIdx.x, SYM);
      mbar_expect_tx(cfull, C::kTileBytes);
#pragma unroll
      for (int h = 0; h < BN / 64; ++h)
        tma_load_3d(dtile + h * (BM * 128), &P.tc[j.c], cfull, j.tj * BN + h * 64, j.ti * BM, j.mat);
      c_pending = true;
    }
    // All four epilogue warps walk the same tiles and execute every named barrier,
    // also after a failed wait (they then skip the work), so no warp can be left
    // waiting at a barrier.
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const TileJob j = decode(p, t, SYM);
      const NsClassArgs& k = p.cls[j.c];
      const int ab = it & 1;
      const uint32_t apar = static_cast<uint32_t>((it >> 1) & 1);
      bool okw = ok && __all_sync(0xffffffffu, mbar_wait(&tfull[ab], apar, abort_flag));
      if (okw && HAS_C) okw = __all_sync(0xffffffffu, mbar_wait(cfull, it & 1, abort_flag));
      if (!okw && ok) {
        ok = false;
        if (lane == 0) {
          set_error(p.err, MUON_ERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      const bool mirror = SYM && j.ti != j.tj;
      if (ok) {
        if (leader) c_pending = false;
        tc_fence_after();
        float scale = 1.f;
        if (PHASE != PH_POLY && p.first_iter) {
          const double inv = 1.0 / (sqrt(p.scal[k.first + j.mat].u2) + (double)p.eps);
          scale = static_cast<float>(PHASE == PH_GRAM ? inv * inv : inv);
        }
#pragma unroll 1
        for (int ch = 0; ch < BN / 32; ++ch) {
          uint32_t v[32];
          tmem_ld32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                        static_cast<uint32_t>(ab * BN + ch * 32),
                    v);
          tmem_wait_ld();
          uint32_t packed[16];
          // the element of this row on the global diagonal, as a column of this chunk
          const int dcol = (j.ti * BM + r) - (j.tj * BN + ch * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint32_t off = sw128_off(r, ch * 32 + q4 * 8);
            uint4 cw = make_uint4(0, 0, 0, 0);
            if (HAS_C) cw = *reinterpret_cast<const uint4*>(dtile + off);
            const uint32_t cwv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i0 = q4 * 8 + 2 * e;
              float a0 = __uint_as_float(v[i0]), a1 = __uint_as_float(v[i0 + 1]);
              if (PHASE == PH_POLY) {
                a0 = fmaf(p.b, __uint_as_float(cwv[e] << 16), p.c * a0);
                a1 = fmaf(p.b, __uint_as_float(cwv[e] & 0xFFFF0000u), p.c * a1);
                if (i0 == dcol) a0 += p.a;
                if (i0 + 1 == dcol) a1 += p.a;
              } else {
                a0 *= scale;
                a1 *= scale;
              }
              packed[q4 * 4 + e] = pack_bf16x2(a0, a1);
            }
            *reinterpret_cast<uint4*>(dtile + off) = make_uint4(
                packed[q4 * 4], packed[q4 * 4 + 1], packed[q4 * 4 + 2], packed[q4 * 4 + 3]);
          }
          if (mirror) {
            // element (r, c) of D is element (c, r) of the mirrored tile
#pragma unroll
            for (int e = 0; e < 32; ++e)
              *reinterpret_cast<uint16_t*>(ttile + sw128_off(ch * 32 + e, r)) =
                  static_cast<uint16_t>(packed[e >> 1] >> ((e & 1) * 16));
          }
        }
        // the accumulator may be reused as soon as it has been read
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[ab]);
        fence_proxy_async_smem();
      }
      named_barrier(1, kEpiWarps * 32);
      if (leader && ok) {
        // boxes that start beyond the matrix edge hold nothing to store
        const int ncols = PHASE == PH_APPLY ? k.n : k.m;
#pragma unroll
        for (int h = 0; h < BN / 64; ++h)
          if (j.tj * BN + h * 64 < ncols)
            tma_store_3d(&P.td[j.c], dtile + h * (BM * 128), j.tj * BN + h * 64, j.ti * BM, j.mat);
        if (mirror) {
#pragma unroll
          for (int h = 0; h < BM / 64; ++h)
            if (j.ti * BM + h * 64 < k.m)
              tma_store_3d(&P.td[j.c], ttile + h * (BM * 128), j.ti * BM + h * 64, j.tj * BN, j.mat);
        }
        tma_store_commit();
        tma_store_wait_read();  // staging buffers are free again
        const int tn = t + static_cast<int>(gridDim.x);
        if (HAS_C && tn < total) {
          const TileJob jn = decode(p, tn, SYM);
          mbar_expect_tx(cfull, C::kTileBytes);
#pragma unroll
          for (int h = 0; h < BN / 64; ++h)
            tma_load_3d(dtile + h * (BM * 128), &P.tc[jn.c], cfull, jn.tj * BN + h * 64,
                        jn.ti * BM, jn.mat);
          c_pending = true;
        }
      }
      named_barrier(1, kEpiWarps * 32);
    }
    if (leader) {
      tma_store_wait_all();
      if (c_pending) mbar_wait(cfull, it & 1, nullptr);  // a C tile still landing
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ============================================================================
// CTA-pair variant: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256). CTA r of the pair loads rows
// [128r, 128r+128) of the A tile and half r of the B tile into its own shared
// memory (plain TMA loads whose bytes are counted on the first CTA's barrier),
// and owns rows [128r, 128r+128) of the accumulator in its TMEM. Per CTA this
// halves the operand bytes per flop of the 128 x 256 single-CTA tile.
// Symmetric phases: tile (ti, tj), tj >= ti, in 256-blocks; each CTA's two
// 128 x 128 sub-blocks (si = 2ti + r, sj = 2tj + h) are stored directly when
// sj >= si and also mirrored when sj > si (sub-blocks below the diagonal come
// from the mirror of another sub-block).
template <int PHASE>
struct PairCfg {
  static constexpr int kABytes = 128 * BK * 2;
  static constexpr int kBBytes = 128 * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;  // 32 KB per CTA
  static constexpr int kStages = PHASE == PH_APPLY ? 5 : 4;
  static constexpr int kCDBytes = 128 * 256 * 2;          // C tile in, D tile out
  static constexpr int kTBytes = PHASE == PH_APPLY ? 0 : 128 * 128 * 2;  // transposed sub-block
  static constexpr int kOffCD = kStages * kStageBytes;
  static constexpr int kOffT = kOffCD + kCDBytes;
  static constexpr int kOffBar = kOffT + kTBytes;
  static constexpr int kTmemCols = 512;                   // two 256-column accumulators
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
};

template <int PHASE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsTc, 1)
    ns_tc_pair_kernel(const __grid_constant__ TcParams P) {
  using C = PairCfg<PHASE>;
  constexpr bool SYM = PHASE != PH_APPLY;
  constexpr bool HAS_C = PHASE == PH_POLY;
  constexpr bool B_MN = PHASE == PH_APPLY;
  constexpr int S = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* cd = smem + C::kOffCD;
  uint8_t* tt = smem + C::kOffT;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint64_t* cfull = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const NsPhaseArgs& p = P.args;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.tile_base[p.num_classes];
  const uint32_t rank = cluster_cta_rank();
  const int cluster_id = static_cast<int>(blockIdx.x >> 1);
  const int nclusters = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);
    }
    mbar_init(done, 1);
    mbar_init(cfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      for (int c = 0; c < p.num_classes; ++c) {
        tma_prefetch(&P.ta[c]);
        tma_prefetch(&P.tb[c]);
      }
      long long q = 0;
      bool ok = true;
      for (int t = cluster_id; t < total && ok; t += nclusters) {
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
          if (rank == 0) mbar_expect_tx(&full[s], 2 * C::kStageBytes);
          tma_load_3d_pair(sa, &P.ta[j.c], &full[s], kb * BK, j.ti * 256 + static_cast<int>(rank) * 128,
                           j.mat);
          if (!B_MN) {
            tma_load_3d_pair(sb, &P.tb[j.c], &full[s], kb * BK,
                             j.tj * 256 + static_cast<int>(rank) * 128, j.mat);
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tma_load_3d_pair(sb + h * (64 * BK * 2), &P.tb[j.c], &full[s],
                               j.tj * 256 + static_cast<int>(rank) * 128 + h * 64, kb * BK, j.mat);
          }
          ++q;
        }
      }
      if (!ok) {
        set_error(p.err, MUON_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      // The first CTA's full barriers count both CTAs' bytes: waiting on them here
      // means no copy of either CTA is still landing when the pair exits.
      if (rank == 0)
        for (long long r = (q > S ? q - S : 0); r < q; ++r)
          mbar_wait(&full[r % S], static_cast<uint32_t>((r / S) & 1), nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (first CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256, B_MN);
      long long q = 0;
      int it = 0;
      bool ok = true;
      for (int t = cluster_id; t < total && ok; t += nclusters, ++it) {
        const TileJob j = decode(p, t, SYM);
        const int kb_n = p.cls[j.c].k_blocks;
        const int ab = it & 1;
        const uint32_t apar = static_cast<uint32_t>((it >> 1) & 1);
        if (!mbar_wait(&tempty[ab], apar ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * 256);
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
            umma_f16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          // the stage is free in both CTAs once these MMAs have read it
          umma_commit_pair(smem_u32(&empty[s]));
          umma_commit_pair(peer_addr(&empty[s], 1));
          ++q;
        }
        if (!ok) break;
        umma_commit_pair(smem_u32(&tfull[ab]));
        umma_commit_pair(peer_addr(&tfull[ab], 1));
      }
      if (!ok) {
        set_error(p.err, MUON_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      umma_commit_pair(smem_u32(done));
      mbar_wait(done, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5, both CTAs)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // row within this CTA's 128 rows
    const bool leader = warp == 2 && lane == 0;
    const int rk = static_cast<int>(rank);
    bool c_pending = false;
    if (HAS_C && leader && cluster_id < total) {
      const TileJob j = decode(p, cluster_id, SYM);
      mbar_expect_tx(cfull, C::kCDBytes);
#pragma unroll
      for (int h = 0; h < 4; ++h)
        tma_load_3d(cd + h * (128 * 128), &P.tc[j.c], cfull, j.tj * 256 + h * 64, j.ti * 256 + rk * 128,
                    j.mat);
      c_pending = true;
    }
    int it = 0;
    bool ok = true;
    for (int t = cluster_id; t < total; t += nclusters, ++it) {
      const TileJob j = decode(p, t, SYM);
      const NsClassArgs& k = p.cls[j.c];
      const int ab = it & 1;
      const uint32_t apar = static_cast<uint32_t>((it >> 1) & 1);
      bool okw = ok && __all_sync(0xffffffffu, mbar_wait(&tfull[ab], apar, abort_flag));
      if (okw && HAS_C) okw = __all_sync(0xffffffffu, mbar_wait(cfull, it & 1, abort_flag));
      if (!okw && ok) {
        ok = false;
        if (lane == 0) {
          set_error(p.err, MUON_ERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      const int m = k.m;
      const int ncols = PHASE == PH_APPLY ? k.n : m;
      const int row0 = j.ti * 256 + rk * 128;
      const int si = 2 * j.ti + rk;
      bool direct[2], mirror[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int sj = 2 * j.tj + h;
        direct[h] = (!SYM || sj >= si) && row0 < m && sj * 128 < ncols;
        mirror[h] = SYM && sj > si && row0 < m && sj * 128 < m;
      }
      float scale = 1.f;
      if (ok) {
        if (leader) c_pending = false;
        tc_fence_after();
        if (PHASE != PH_POLY && p.first_iter) {
          const double inv = 1.0 / (sqrt(p.scal[k.first + j.mat].u2) + (double)p.eps);
          scale = static_cast<float>(PHASE == PH_GRAM ? inv * inv : inv);
        }
      }
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        if (ok) {
#pragma unroll 1
          for (int ch = 4 * h; ch < 4 * h + 4; ++ch) {
            uint32_t v[32];
            tmem_ld32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                          static_cast<uint32_t>(ab * 256 + ch * 32),
                      v);
            tmem_wait_ld();
            uint32_t packed[16];
            const int dcol = (row0 + r) - (j.tj * 256 + ch * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const uint32_t off = sw128_off(r, ch * 32 + q4 * 8);
              uint4 cw = make_uint4(0, 0, 0, 0);
              if (HAS_C) cw = *reinterpret_cast<const uint4*>(cd + off);
              const uint32_t cwv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int i0 = q4 * 8 + 2 * e;
                float a0 = __uint_as_float(v[i0]), a1 = __uint_as_float(v[i0 + 1]);
                if (PHASE == PH_POLY) {
                  a0 = fmaf(p.b, __uint_as_float(cwv[e] << 16), p.c * a0);
                  a1 = fmaf(p.b, __uint_as_float(cwv[e] & 0xFFFF0000u), p.c * a1);
                  if (i0 == dcol) a0 += p.a;
                  if (i0 + 1 == dcol) a1 += p.a;
                } else {
                  a0 *= scale;
                  a1 *= scale;
                }
                packed[q4 * 4 + e] = pack_bf16x2(a0, a1);
              }
              *reinterpret_cast<uint4*>(cd + off) = make_uint4(
                  packed[q4 * 4], packed[q4 * 4 + 1], packed[q4 * 4 + 2], packed[q4 * 4 + 3]);
            }
            if (mirror[h]) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                *reinterpret_cast<uint16_t*>(tt + sw128_off((ch - 4 * h) * 32 + e, r)) =
                    static_cast<uint16_t>(packed[e >> 1] >> ((e & 1) * 16));
            }
          }
          if (h == 1) {
            // this CTA's accumulator rows have been read: free them for the MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (rk == 0) mbar_arrive(&tempty[ab]);
              else mbar_arrive_cluster(peer_addr(&tempty[ab], 0));
            }
          }
          fence_proxy_async_smem();
        }
        if (SYM || h == 1) {
          named_barrier(1, kEpiWarps * 32);
          if (leader && ok) {
            if (h == 1) {
#pragma unroll
              for (int b = 0; b < 4; ++b)
                if (direct[b >> 1] && j.tj * 256 + b * 64 < ncols)
                  tma_store_3d(&P.td[j.c], cd + b * (128 * 128), j.tj * 256 + b * 64, row0, j.mat);
            }
            if (mirror[h]) {
              const int sj = 2 * j.tj + h;
#pragma unroll
              for (int b = 0; b < 2; ++b)
                if (si * 128 + b * 64 < m)
                  tma_store_3d(&P.td[j.c], tt + b * (128 * 128), si * 128 + b * 64, sj * 128, j.mat);
            }
            tma_store_commit();
            tma_store_wait_read();  // staging buffers are free again
            const int tn = t + nclusters;
            if (h == 1 && HAS_C && tn < total) {
              const TileJob jn = decode(p, tn, SYM);
              mbar_expect_tx(cfull, C::kCDBytes);
#pragma unroll
              for (int b = 0; b < 4; ++b)
                tma_load_3d(cd + b * (128 * 128), &P.tc[jn.c], cfull, jn.tj * 256 + b * 64,
                            jn.ti * 256 + rk * 128, jn.mat);
              c_pending = true;
            }
          }
          named_barrier(1, kEpiWarps * 32);
        }
      }
    }
    if (leader) {
      tma_store_wait_all();
      if (c_pending) mbar_wait(cfull, it & 1, nullptr);
    }
  }

  __syncthreads();
  cluster_sync_all();  // no cross-CTA signal or TMEM access is outstanding past this point
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

template <int PHASE>
cudaError_t launch_pair(const TcParams& P, int grid, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(ns_tc_pair_kernel<PHASE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         PairCfg<PHASE>::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  ns_tc_pair_kernel<PHASE><<<grid, kThreadsTc, PairCfg<PHASE>::kSmemBytes, s>>>(P);
  return cudaGetLastError();
}

template <int BN, int PHASE>
cudaError_t launch_one(const TcParams& P, int grid, cudaStream_t s) {
  using C = TcCfg<BN, PHASE>;
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

cudaError_t launch_ns_phase_tc_pair(const TcParams& P, int num_sms, cudaStream_t s) {
  const int total = P.args.tile_base[P.args.num_classes];
  if (total <= 0) return cudaSuccess;
  const int pairs = total < num_sms / 2 ? total : num_sms / 2;
  switch (P.args.phase) {
    case PH_GRAM: return launch_pair<PH_GRAM>(P, 2 * pairs, s);
    case PH_POLY: return launch_pair<PH_POLY>(P, 2 * pairs, s);
    default: return launch_pair<PH_APPLY>(P, 2 * pairs, s);
  }
}

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
