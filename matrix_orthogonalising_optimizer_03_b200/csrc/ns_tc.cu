// bf16 Newton-Schulz phases on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The three contractions of one iteration X <- aX + b(XX^T)X + c(XX^T)^2 X (the
// Newton-Schulz listing of "LLM Pretraining Loss Spike 진단과 처방", section "Muon
// head의 실체는 하이브리드 옵티마이저다"; section 2 of the "MUON IS SCALABLE FOR LLM
// TRAINING" review) as three grouped GEMM launches over every matrix of every
// shape class in the call:
//   GRAM   S  = alpha * X X^T            A = X (K-major), B = X (K-major), K = n
//   POLY   P' = a*I + b*S + c * S S      A = S, B = S (S = S^T), K = m
//   APPLY  X' = gamma * P' X             A = P', B = X (MN-major), K = m
// alpha = 1/(||U||+eps)^2 and gamma = 1/(||U||+eps) on the first iteration (the
// slab then holds the unnormalised U), 1 afterwards. X, S, P' are stored in bf16,
// accumulation is fp32 in TMEM.
//
// The a*X term of the recurrence is folded into P' (a*X + P X = (a I + P) X), so the
// apply epilogue reads nothing but the accumulator; P' is rounded to bf16 once, with
// its diagonal a + P_ii (about 0.7) in place of P_ii (about -2.7).
//
// Symmetric storage: S and P' are symmetric, so only their 128 x 128 blocks on or
// above the block diagonal are computed and stored. A consumer that needs a block
// below the diagonal (rows in block i, columns in block k < i) loads its mirror
// block (k, i) and hands it to tcgen05.mma as an MN-major operand (the transpose is
// free in the instruction descriptor). MN-major blocks (these mirrors and APPLY's X)
// come in one TMA box of a 4-D view of the slab, [matrix][64-column chunk][row][64],
// which lands chunk after chunk in the MN-major layout.
//
// Kernel structure (persistent, one CTA per SM, 320 threads):
//   warp 0     TMA producer: a ring of 128B-swizzled shared-memory stages (as many as
//              fit 224 KB; single-CTA symmetric launches size their stages to their
//              largest tile); every load lands in one CTA's own shared memory. On the
//              block diagonal of GRAM and POLY it loads B only (A is B's first rows).
//   warp 1     TMEM allocator and MMA issuer (one thread), double-buffered fp32
//              accumulator in TMEM.
//   warps 2-9  epilogue: two warps per TMEM lane quarter, each taking every other
//              64-column chunk; tcgen05.ld, fused scale / polynomial, and per warp a
//              32 x 64 bf16 box staged in swizzled shared memory and written with the
//              warp's own TMA store (which clips ragged edges), with no barrier between
//              the warps. POLY's C tile (S) arrives by TMA one tile ahead (CTA pairs)
//              or is read from L2 into registers (single CTA).
// Two variants:
//   single CTA   APPLY tiles 128 x 256; GRAM / POLY tiles of one 128-row block and a
//                variable-width column piece (sym_piece), described stage by stage by
//                the producer to the MMA issuer; tcgen05.mma.cta_group::1, M = 128.
//   CTA pair     cluster of two CTAs, tile 256 x 256, tcgen05.mma.cta_group::2
//                (M = N = 256): each CTA loads its 128 rows of A and half of B into
//                its own shared memory (plain TMA loads whose bytes count on the first
//                CTA's barrier) and owns 128 accumulator rows in its TMEM. Per CTA this
//                halves the operand bytes per flop. Used for classes with m % 256 == 0.
// Slabs are [count][rows][ld] bf16 addressed by 3-D tensor maps (inner dim, rows,
// matrix), so out-of-range rows and columns of a matrix are zero-filled by TMA and
// never spill into the next matrix. Every wait is bounded (see ptx.cuh).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "muon_internal.h"
#include "ns_tc.h"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int BM = 128, BK = 64;
constexpr int kEpiWarps = 8;
constexpr int kThreadsTc = 64 + 32 * kEpiWarps;  // 320
constexpr int kWarpBoxBytes = 32 * 128;           // one 32-row x 64-column bf16 output box
constexpr int kMaxStages = 8;                     // barrier pairs reserved for the operand ring

template <int BN, int PHASE, bool PAIR>
struct TcCfg {
  static constexpr bool kSym = PHASE != PH_APPLY;         // symmetric (upper-block) output
  static constexpr bool kHasC = PHASE == PH_POLY;         // epilogue reads a C tile (S)
  // single-CTA symmetric phases: variable-width tiles (one row block, one column piece
  // of up to BN = 256 columns; see sym_piece), B loaded in 64-row units
  static constexpr bool kVarN = !PAIR && kSym;
  // POLY's C tile (S): staged through shared memory by TMA (CTA pairs), or, for the
  // short-K single-CTA tiles, read by each epilogue thread from global memory (L2)
  // into registers before it waits for the accumulator
  static constexpr bool kCStaged = kHasC && !kVarN;
  static constexpr bool kCRegs = kHasC && kVarN;
  static constexpr int kNCol = PAIR ? 256 : BN;            // accumulator columns per CTA
  static constexpr int kBRows = PAIR ? 128 : BN;           // B rows (or columns) per CTA
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = kBRows * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // epilogue: each warp stores 32 x 64 boxes; it takes every other 64-column chunk
  static constexpr int kChunksPerWarp = kNCol / 128;
  // one box buffer per warp: the epilogue has slack (it waits for the accumulator most of
  // the time), and the shared memory goes to the operand ring instead
  static constexpr int kEpiBufs = 1;
  static constexpr int kStagingBytes =
      kCStaged ? BM * kNCol * 2 : kEpiWarps * kEpiBufs * kWarpBoxBytes;  // C tile, or per-warp boxes
  static constexpr int kBudget = 224 * 1024;
  static constexpr int kFit = (kBudget - kStagingBytes) / kStageBytes;
  static constexpr int kStages = kFit > kMaxStages ? kMaxStages : kFit;
  static constexpr int kOffStg = kStages * kStageBytes;
  static constexpr int kOffBar = kOffStg + kStagingBytes;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kTmemCols = 2 * kNCol;
  // barrier region: full and empty per ring slot, tfull and tempty per accumulator, done,
  // cfull, the TMEM address, the abort flag and one stage_meta word per ring slot
  static_assert(8 * (2 * kMaxStages + 2 + 2 + 2) + 4 + 4 + 4 * kMaxStages <= 256,
                "barrier region overflow");
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  static constexpr int kMmaM = PAIR ? 256 : 128;
  static constexpr int kMmaN = PAIR ? 256 : BN;
  static constexpr int kTileM = PAIR ? 256 : 128;          // output tile (cluster) rows
  static constexpr int kTileN = PAIR ? 256 : BN;           // output tile columns
  static_assert(kStages >= 3, "pipeline too shallow");
  static_assert(!kVarN || BN == 256, "variable-width tiles are at most 256 columns");
};

struct TileJob {
  int c, mat, ti, tj;
  int col0, nt;  // first output column and width (columns) of the tile
};

// Tile t of the launch: its class, matrix and output block. Symmetric phases walk the
// upper block triangle: fixed square tiles (tile_n x tile_n, CTA pairs) or, with varn,
// the variable-width pieces of each 128-row block (sym_piece).
__device__ __forceinline__ TileJob decode(const NsPhaseArgs& p, int t, bool sym, bool varn,
                                          int tile_n) {
  int c = 0;
  while (c + 1 < p.num_classes && t >= p.tile_base[c + 1]) ++c;
  const NsClassArgs& k = p.cls[c];
  const int u = t - p.tile_base[c];
  TileJob j;
  j.c = c;
  if (varn) {
    // A matrix's tiles stay consecutive (they run at the same time and share its operand
    // rows in L2), but the order of its pieces is rotated by the matrix index: pieces
    // differ in width, and without the rotation a CTA of the round-robin would take the
    // same piece of every matrix whenever the CTA count is a multiple of the pieces
    j.mat = u / k.tiles_per_mat;
    int rem = (u - j.mat * k.tiles_per_mat + j.mat) % k.tiles_per_mat;
    int ti = 0;
    while (rem >= sym_pieces(k.m, ti)) {
      rem -= sym_pieces(k.m, ti);
      ++ti;
    }
    j.ti = ti;
    j.tj = rem;
    sym_piece(k.m, ti, rem, &j.col0, &j.nt);
    return j;
  }
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
  j.col0 = j.tj * tile_n;
  j.nt = tile_n;
  return j;
}

// The class of tile t (the first part of decode, for roles that need no more).
__device__ __forceinline__ int class_of(const NsPhaseArgs& p, int t) {
  int c = 0;
  while (c + 1 < p.num_classes && t >= p.tile_base[c + 1]) ++c;
  return c;
}

// Stage descriptor of a variable-width tile, written by the producer for the MMA issuer
// (which then decodes nothing): B's unit count, the first mirrored unit, A's layout, and
// whether A is B's first rows.
__device__ __forceinline__ uint32_t stage_meta(int nu, int split, bool a_t, bool shared_a) {
  return static_cast<uint32_t>(nu) | (static_cast<uint32_t>(split) << 3) |
         (a_t ? (1u << 6) : 0u) | (shared_a ? (1u << 7) : 0u);
}

// Whether B unit u (64 rows starting at output column col0 + 64 u) of k-block kb lies
// below the stored 128-block diagonal (variable-width symmetric tiles).
__device__ __forceinline__ bool unit_mirrored(bool sym_operand, int col0, int u, int kb) {
  return sym_operand && (kb * 64) / 128 < (col0 + 64 * u) / 128;
}

// Whether a tile's A operand is already in shared memory as the start of its B operand.
// In GRAM (A = B = X) and POLY (A = B = S) a tile on the block diagonal reads the same
// rows for both operands, with the same layout decision in every k-block (below_diag and
// unit_mirrored agree when the tile's first column is its first row): the tile then loads
// only B, and the MMA takes A from B's first 128 rows. A single-CTA piece needs at least
// two B units (128 rows); a CTA of a pair owns 128 rows of each.
__device__ __forceinline__ bool a_in_b(bool sym, bool varn, const TileJob& j, int tile_m) {
  if (!sym) return false;
  return varn ? (j.col0 == j.ti * tile_m && j.nt >= 128) : j.ti == j.tj;
}

// Stage size of a launch of variable-width symmetric tiles: the largest k-block of A and
// B that any of its tiles loads (B alone where a_in_b). The ring of fixed size then holds
// as many stages as fit (narrow pieces and diagonal tiles leave room for more).
__device__ __forceinline__ int varn_stage_bytes(const NsPhaseArgs& p, int a_bytes) {
  int most = 0;
  for (int c = 0; c < p.num_classes; ++c) {
    const int m = p.cls[c].m;
    for (int i = 0; i < sym_row_blocks(m); ++i)
      for (int jj = 0; jj < sym_pieces(m, i); ++jj) {
        int col0, width;
        sym_piece(m, i, jj, &col0, &width);
        const int bytes = (col0 == 128 * i && width >= 128 ? 0 : a_bytes) + width * (BK * 2);
        most = bytes > most ? bytes : most;
      }
  }
  return most;
}

// Byte offset of element (r, c) of a 128-row tile staged as 64-column boxes with
// the 128-byte swizzle (the layout TMA reads and writes for a 64 x 128 box).
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>((c >> 6) * (BM * 128) + r * 128 +
                               ((((c >> 3) & 7) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

// Whether k-block kb of the operand rows of a tile starting at row tile_row0 lies
// below the stored block diagonal (block size G) and must be read from its mirror.
// G is the class's tile height: 128 for single-CTA classes, 256 for CTA-pair
// classes (whose diagonal 256 x 256 tiles are stored whole, so that both CTAs of a
// pair always agree on the layout of a k-block).
__device__ __forceinline__ bool below_diag(bool sym_operand, int tile_row0, int kb, int G) {
  return sym_operand && (kb * BK) / G < tile_row0 / G;
}

// Loads the 128 x 64 block of a K-major operand, or, when it lies below the
// diagonal, its mirror as one box of the chunk view (two 64 x 64 chunks, 8 KB apart:
// the MN-major layout).
template <bool PAIR>
__device__ __forceinline__ void load_k_block(uint8_t* dst, const CUtensorMap* mk,
                                             const CUtensorMap* mt, uint64_t* bar, int row0,
                                             int kb, int mat, bool mirrored) {
  if (!mirrored) {
    if (PAIR) tma_load_3d_pair(dst, mk, bar, kb * BK, row0, mat);
    else tma_load_3d(dst, mk, bar, kb * BK, row0, mat);
  } else {
    if (PAIR) tma_load_4d_pair(dst, mt, bar, 0, kb * BK, row0 / 64, mat);
    else tma_load_4d(dst, mt, bar, 0, kb * BK, row0 / 64, mat);
  }
}

template <int BN, int PHASE, bool PAIR>
__global__ void __launch_bounds__(kThreadsTc, 1) ns_tc_kernel(const __grid_constant__ TcParams P) {
  using C = TcCfg<BN, PHASE, PAIR>;
  constexpr bool SYM = C::kSym;
  constexpr bool HAS_C = C::kCStaged;        // C tile staged in shared memory by TMA
  constexpr bool C_REGS = C::kCRegs;         // C read into registers from global memory
  constexpr bool A_SYM = PHASE != PH_GRAM;   // A is S (POLY) or P' (APPLY): upper blocks only
  constexpr bool B_SYM = PHASE == PH_POLY;   // B is S
  constexpr bool B_MN = PHASE == PH_APPLY;   // B is X read along its rows
  constexpr bool VARN = C::kVarN;            // variable-width symmetric tiles (single CTA)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stg = smem + C::kOffStg;  // output staging (POLY: the C tile, overwritten by D)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint64_t* cfull = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* meta = tmem_slot + 2;  // per ring slot: stage_meta (variable-width tiles)

  const NsPhaseArgs& p = P.args;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // operand ring: S stages of sbytes (variable-width tiles size them to the launch)
  int sbytes = C::kStageBytes;
  if (VARN) {
    sbytes = varn_stage_bytes(p, C::kABytes);
    sbytes = sbytes < 1024 ? 1024 : sbytes;
  }
  const int S_ = C::kRingBytes / sbytes;
  const int S = S_ > kMaxStages ? kMaxStages : S_;
  const int total = p.tile_base[p.num_classes];
  const int rank = PAIR ? static_cast<int>(cluster_cta_rank()) : 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int nunits = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], (PAIR ? 2 : 1) * kEpiWarps);
    }
    mbar_init(done, 1);
    mbar_init(cfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the prologue above overlaps the previous kernel's tail; its results are read below
  griddep_launch_dependents();
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int c = 0; c < p.num_classes; ++c) {
        tma_prefetch(&P.ta[c]);
        tma_prefetch(&P.tb[c]);
      }
      long long q = 0;        // stages loaded
      int s = 0;              // its slot, q mod S
      uint32_t par = 0;       // and the parity of the slot's use, (q / S) mod 2
      bool ok = true;
      for (int t = unit; t < total && ok; t += nunits) {
        const TileJob j = decode(p, t, SYM, VARN, C::kTileN);
        const int kb_n = p.cls[j.c].k_blocks;
        const int a_row0 = j.ti * C::kTileM + rank * 128;
        const int b_row0 = j.col0 + rank * (PAIR ? 128 : 0);
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&empty[s], par ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * sbytes;
          uint8_t* sb = sa + C::kABytes;
          if (VARN) {
            // A: the row block's 128 rows; B: the tile's nt rows in 64-row units, each
            // K-major (a 64 x 64 box) or, below the diagonal, its mirror (one chunk).
            // Without an A of its own the stage starts with B.
            const bool shared_a = a_in_b(SYM, true, j, C::kTileM);
            const bool a_t = below_diag(A_SYM, j.ti * C::kTileM, kb, C::kTileM);
            const int nu = j.nt / 64;
            int split = nu;  // first mirrored unit (unit_mirrored is monotone in u)
            for (int u = 0; u < nu; ++u)
              if (unit_mirrored(B_SYM, j.col0, u, kb)) { split = u; break; }
            // published to the MMA issuer by the arrive below (release, CTA scope)
            meta[s] = stage_meta(nu, split, a_t, shared_a);
            if (shared_a) sb = sa;
            mbar_expect_tx(&full[s], (shared_a ? 0 : C::kABytes) + j.nt * (BK * 2));
            if (!shared_a)
              load_k_block<false>(sa, &P.ta[j.c], &P.ta_t[j.c], &full[s], a_row0, kb, j.mat, a_t);
            // Two neighbouring units of the same layout come in one 128-row box through
            // A's maps (A and B are the same slab in GRAM and POLY): fewer, larger copies
            for (int u = 0; u < nu;) {
              uint8_t* dst = sb + u * (64 * BK * 2);
              const bool mir = u >= split;
              const bool two = u + 1 < nu && (u + 1 >= split) == mir;
              const CUtensorMap* km = two ? &P.ta[j.c] : &P.tb[j.c];
              const CUtensorMap* mm = two ? &P.ta_t[j.c] : &P.tb_t[j.c];
              if (mir) tma_load_4d(dst, mm, &full[s], 0, kb * BK, j.col0 / 64 + u, j.mat);
              else tma_load_3d(dst, km, &full[s], kb * BK, j.col0 + 64 * u, j.mat);
              u += two ? 2 : 1;
            }
            ++q;
            if (++s == S) s = 0, par ^= 1u;
            continue;
          }
          const bool shared_a = a_in_b(SYM, false, j, C::kTileM);
          if (!PAIR || rank == 0)
            mbar_expect_tx(&full[s], (PAIR ? 2 : 1) * (shared_a ? C::kABytes : C::kStageBytes));
          load_k_block<PAIR>(sa, &P.ta[j.c], &P.ta_t[j.c], &full[s], a_row0, kb, j.mat,
                             below_diag(A_SYM, j.ti * C::kTileM, kb, C::kTileM));
          if (shared_a) {
            // diagonal tile: B's rows are A's (the MMA reads both from the A stage)
          } else if (!B_MN) {
            load_k_block<PAIR>(sb, &P.tb[j.c], &P.tb_t[j.c], &full[s], b_row0, kb, j.mat,
                               below_diag(B_SYM, j.tj * C::kTileN, kb, C::kTileN));
          } else {  // X rows kb*BK.., columns b_row0.. in kBRows/64 chunks, one box
            if (PAIR) tma_load_4d_pair(sb, &P.tb[j.c], &full[s], 0, kb * BK, b_row0 / 64, j.mat);
            else tma_load_4d(sb, &P.tb[j.c], &full[s], 0, kb * BK, b_row0 / 64, j.mat);
          }
          ++q;
          if (++s == S) s = 0, par ^= 1u;
        }
      }
      if (!ok) {
        set_error(p.err, MUON_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      // Never leave with bulk copies still landing in shared memory (for a pair, the
      // first CTA's full barriers count both CTAs' bytes).
      if (!PAIR || rank == 0)
        for (long long r = (q > S ? q - S : 0); r < q; ++r)
          mbar_wait(&full[static_cast<int>(r % S)], static_cast<uint32_t>((r / S) & 1), nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && (!PAIR || rank == 0)) {
      const uint32_t idesc0 = idesc_bf16_f32(C::kMmaM, C::kMmaN, B_MN);
      // descriptors differ per k-slice only in the start-address field: build the
      // constant part once (K-major: LBO 16 B; MN-major: LBO 8 KB between 64-element
      // chunks; both SBO 1024 B) and add the address per slice
      const uint64_t kmaj_hi = smem_desc_sw128(0, 16, 1024);
      const uint64_t mnmaj_hi = smem_desc_sw128(0, 64 * BK * 2, 1024);
      int s = 0;              // slot of the next stage
      uint32_t par = 0;       // parity of that slot's use
      int it = 0;
      bool ok = true;
      for (int t = unit; t < total && ok; t += nunits, ++it) {
        // variable-width tiles: the producer describes each stage (meta); other tiles
        // are decoded here
        const TileJob j = VARN ? TileJob{class_of(p, t), 0, 0, 0, 0, 0}
                               : decode(p, t, SYM, VARN, C::kTileN);
        const int kb_n = p.cls[j.c].k_blocks;
        const int a_row0 = j.ti * C::kTileM;  // the first CTA's rows decide for both
        const int b_row0 = j.col0;
        const int ab = it & 1;
        const uint32_t apar = static_cast<uint32_t>((it >> 1) & 1);
        if (!mbar_wait(&tempty[ab], apar ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * C::kNCol);
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&full[s], par, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (VARN) {
            // B's 64-row units switch from K-major to mirrored (MN-major) at most once
            // along the tile (unit_mirrored is monotone in u): one MMA per run of units
            // of the same layout, each writing its own accumulator columns
            const uint32_t md = meta[s];
            const int nu = static_cast<int>(md & 7u), split = static_cast<int>((md >> 3) & 7u);
            const bool a_t = (md >> 6) & 1u, shared_a = (md >> 7) & 1u;
            const uint32_t sa = smem_u32(smem + s * sbytes);
            const uint32_t sb = shared_a ? sa : sa + C::kABytes;
            const uint64_t ad0 = (a_t ? mnmaj_hi : kmaj_hi) | static_cast<uint64_t>((sa >> 4) & 0x3FFFu);
            const uint64_t astep = a_t ? 128u : 2u;
#pragma unroll
            for (int run = 0; run < 2; ++run) {
              const int u0 = run == 0 ? 0 : split, u1 = run == 0 ? split : nu;
              if (u1 <= u0) continue;
              const bool b_t = run == 1;
              const uint32_t idesc = idesc_bf16_f32(128, 64 * (u1 - u0), b_t) |
                                     (a_t ? (1u << 15) : 0u);
              const uint32_t sbu = sb + static_cast<uint32_t>(u0 * (64 * BK * 2));
              const uint64_t bd0 = (b_t ? mnmaj_hi : kmaj_hi) | static_cast<uint64_t>((sbu >> 4) & 0x3FFFu);
              const uint64_t bstep = b_t ? 128u : 2u;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma_f16(d_tmem + static_cast<uint32_t>(u0 * 64), ad0 + astep * kk, bd0 + bstep * kk,
                         idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            umma_commit(&empty[s]);
            if (++s == S) s = 0, par ^= 1u;
            continue;
          }
          // one instruction serves both CTAs of a pair: the layout choice is made per
          // cluster tile (block size kTileM), identical for both halves
          const bool a_t = below_diag(A_SYM, a_row0, kb, C::kTileM);
          const bool b_t = B_MN || below_diag(B_SYM, b_row0, kb, C::kTileN);
          const uint32_t idesc = idesc0 | (a_t ? (1u << 15) : 0u) | (b_t ? (1u << 16) : 0u);
          const uint32_t sa = smem_u32(smem + s * sbytes);
          const uint32_t sb = a_in_b(SYM, false, j, C::kTileM) ? sa : sa + C::kABytes;
          // K-major slices advance 32 B (2 in the >>4 address field), MN-major 2 KB (128)
          const uint64_t ad0 = (a_t ? mnmaj_hi : kmaj_hi) | static_cast<uint64_t>((sa >> 4) & 0x3FFFu);
          const uint64_t bd0 = (b_t ? mnmaj_hi : kmaj_hi) | static_cast<uint64_t>((sb >> 4) & 0x3FFFu);
          const uint64_t astep = a_t ? 128u : 2u, bstep = b_t ? 128u : 2u;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = ad0 + astep * kk;
            const uint64_t bd = bd0 + bstep * kk;
            if (PAIR) umma_f16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            else umma_f16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          if (PAIR) {
            umma_commit_pair(smem_u32(&empty[s]));
            umma_commit_pair(peer_addr(&empty[s], 1));
          } else {
            umma_commit(&empty[s]);
          }
          if (++s == S) s = 0, par ^= 1u;
        }
        if (!ok) break;
        if (PAIR) {
          umma_commit_pair(smem_u32(&tfull[ab]));
          umma_commit_pair(peer_addr(&tfull[ab], 1));
        } else {
          umma_commit(&tfull[ab]);
        }
      }
      if (!ok) {
        set_error(p.err, MUON_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      if (PAIR) umma_commit_pair(smem_u32(done));
      else umma_commit(done);
      mbar_wait(done, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-9)
    // Each warp owns the 32 accumulator rows of its TMEM lane quarter and every other
    // 64-column chunk of the tile. It stages a chunk as a 32 x 64 bf16 box in its own
    // 128B-swizzled buffer (POLY: in place, over the C tile) and stores the box with
    // its own TMA store, so the warps never wait for one another inside a tile. POLY
    // synchronises the eight warps once per tile, before the next C tile may land.
    const int ew = warp - 2;
    const int quad = warp & 3;           // the TMEM lane quarter this warp may access
    const int grp = ew >> 2;             // chunks grp, grp + 2, ...
    const int r = quad * 32 + lane;      // tile row of this thread within the CTA
    const bool leader = ew == 0 && lane == 0;
    uint8_t* wbuf = stg + ew * (C::kEpiBufs * kWarpBoxBytes);  // GRAM / APPLY box buffers
    int nstore = 0;                                           // boxes this warp has staged
    bool c_pending = false;
    if (HAS_C && leader && unit < total) {
      const TileJob j = decode(p, unit, SYM, VARN, C::kTileN);
      mbar_expect_tx(cfull, static_cast<uint32_t>(j.nt * (BM * 2)));
      for (int h = 0; h < j.nt / 64; ++h)
        tma_load_3d(stg + h * (BM * 128), &P.tc[j.c], cfull, j.col0 + h * 64,
                    j.ti * C::kTileM + rank * 128, j.mat);
      c_pending = true;
    }
    // All epilogue warps walk the same tiles and, in POLY, execute every named
    // barrier, also after a failed wait (they then skip the work): no warp is ever
    // left waiting at a barrier.
    int it = 0;
    bool ok = true;
    for (int t = unit; t < total; t += nunits, ++it) {
      const TileJob j = decode(p, t, SYM, VARN, C::kTileN);
      const NsClassArgs& k = p.cls[j.c];
      const int ab = it & 1;
      const uint32_t apar = static_cast<uint32_t>((it >> 1) & 1);
      // C in registers: this thread's row of S for each of the warp's (at most two)
      // chunks, loaded before the accumulator wait so that the fetch overlaps the MMAs.
      // Columns past m inside the last chunk are the slab's padding: they only reach
      // output columns the store clips.
      uint4 creg[C_REGS ? 2 : 1][8];
      if (C_REGS && ok) {
        const int row = j.ti * C::kTileM + quad * 32 + lane;
        const uint16_t* srow = static_cast<const uint16_t*>(k.s) + j.mat * k.sstride +
                               static_cast<int64_t>(row) * k.lds + j.col0;
#pragma unroll
        for (int ci = 0; ci < (C_REGS ? 2 : 1); ++ci) {
          const int c64 = 2 * ci + grp;
          const bool have = row < k.m && c64 < j.nt / 64;
#pragma unroll
          for (int q8 = 0; q8 < 8; ++q8)
            creg[ci][q8] = have ? __ldg(reinterpret_cast<const uint4*>(srow + c64 * 64) + q8)
                                : make_uint4(0, 0, 0, 0);
        }
      }
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
      const int row0 = j.ti * C::kTileM + rank * 128;   // this CTA's first output row
      const int col0 = j.col0;                           // this CTA's first output column
      if (ok) {
        if (leader) c_pending = false;
        tc_fence_after();
        float scale = 1.f;
        if (PHASE != PH_POLY && p.first_iter) {
          const double inv = 1.0 / (sqrt(p.scal[k.first + j.mat].u2) + (double)p.eps);
          scale = static_cast<float>(PHASE == PH_GRAM ? inv * inv : inv);
        }
        // this warp's chunks of the tile: grp, grp + 2, ... below nt / 64
        const int nchw = VARN ? (j.nt / 64 - grp + 1) / 2 : C::kChunksPerWarp;
        if (nchw == 0) {  // nothing to read: release the accumulator at once
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[ab]);
        }
#pragma unroll 1
        for (int ci = 0; ci < nchw; ++ci) {
          const int c64 = 2 * ci + grp;  // 64-column chunk of the tile
          uint32_t v[2][32];
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                 static_cast<uint32_t>(ab * C::kNCol + c64 * 64);
          tmem_ld32(taddr, v[0]);
          tmem_ld32(taddr + 32, v[1]);
          tmem_wait_ld();
          if (ci == nchw - 1) {
            // this warp has read its share of the accumulator: free it for the MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (!PAIR || rank == 0) mbar_arrive(&tempty[ab]);
              else mbar_arrive_cluster(peer_addr(&tempty[ab], 0));
            }
          }
          uint8_t* box;
          if (HAS_C) {
            box = stg + c64 * (BM * 128) + quad * kWarpBoxBytes;  // this warp's rows of C
          } else {  // GRAM, APPLY, and POLY with C in registers
            box = wbuf + (nstore % C::kEpiBufs) * kWarpBoxBytes;
            if (nstore >= C::kEpiBufs) {  // the store that last read this buffer is done with it
              if (lane == 0) tma_store_wait_read_n<C::kEpiBufs - 1>();
              __syncwarp();
            }
          }
          // the element of this row on the global diagonal, as a column of this chunk
          const int dcol = (row0 + r) - (col0 + c64 * 64);
#pragma unroll
          for (int q8 = 0; q8 < 8; ++q8) {
            const uint32_t off = sw128_off(lane, q8 * 8);
            uint4 cw = make_uint4(0, 0, 0, 0);
            if (HAS_C) cw = *reinterpret_cast<const uint4*>(box + off);
            if (C_REGS) cw = ci == 0 ? creg[0][q8] : creg[C_REGS ? 1 : 0][q8];  // no dynamic index
            const uint32_t cwv[4] = {cw.x, cw.y, cw.z, cw.w};
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i0 = q8 * 8 + 2 * e;
              float a0 = __uint_as_float(v[i0 >> 5][i0 & 31]);
              float a1 = __uint_as_float(v[(i0 + 1) >> 5][(i0 + 1) & 31]);
              if (PHASE == PH_POLY) {
                a0 = fmaf(p.b, __uint_as_float(cwv[e] << 16), p.c * a0);
                a1 = fmaf(p.b, __uint_as_float(cwv[e] & 0xFFFF0000u), p.c * a1);
                if (i0 == dcol) a0 += p.a;
                if (i0 + 1 == dcol) a1 += p.a;
              } else {
                a0 *= scale;
                a1 *= scale;
              }
              pk[e] = pack_bf16x2(a0, a1);
            }
            *reinterpret_cast<uint4*>(box + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int x = col0 + c64 * 64, y = row0 + quad * 32;
            if (x < ncols && y < m) tma_store_3d(&P.td[j.c], box, x, y, j.mat);
            tma_store_commit();
          }
          ++nstore;
        }
      }
      if (HAS_C) {
        // every warp's boxes have been read out of the tile; then the next C lands
        if (lane == 0) tma_store_wait_read();
        named_barrier(1, kEpiWarps * 32);
        const int tn = t + nunits;
        if (leader && ok && tn < total) {
          const TileJob jn = decode(p, tn, SYM, VARN, C::kTileN);
          mbar_expect_tx(cfull, static_cast<uint32_t>(jn.nt * (BM * 2)));
          for (int b = 0; b < jn.nt / 64; ++b)
            tma_load_3d(stg + b * (BM * 128), &P.tc[jn.c], cfull, jn.col0 + b * 64,
                        jn.ti * C::kTileM + rank * 128, jn.mat);
          c_pending = true;
        }
      }
    }
    if (lane == 0) tma_store_wait_all();
    if (leader && c_pending) mbar_wait(cfull, it & 1, nullptr);  // a C tile still landing
  }

  __syncthreads();
  if (PAIR) cluster_sync_all();  // no cross-CTA signal or TMEM access outstanding
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int BN, int PHASE, bool PAIR>
cudaError_t launch_tc(const TcParams& P, int grid, cudaStream_t s) {
  using C = TcCfg<BN, PHASE, PAIR>;
  // the shared-memory opt-in is a per-device attribute: set it once on each device
  static std::atomic<uint64_t> attr_devices{0};
  auto kern = ns_tc_kernel<BN, PHASE, PAIR>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit == 0 || !(attr_devices.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_devices.fetch_or(bit, std::memory_order_acq_rel);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreadsTc, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PAIR ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

}  // namespace

int tc_block_n(int phase) { return phase == PH_APPLY ? 256 : 128; }  // symmetric: pieces, see sym_piece
int tc_block_m() { return BM; }
int tc_block_k() { return BK; }

cudaError_t launch_ns_phase_tc_pair(const TcParams& P, int num_sms, cudaStream_t s) {
  const int total = P.args.tile_base[P.args.num_classes];
  if (total <= 0) return cudaSuccess;
  const int pairs = total < num_sms / 2 ? total : num_sms / 2;
  switch (P.args.phase) {
    case PH_GRAM: return launch_tc<256, PH_GRAM, true>(P, 2 * pairs, s);
    case PH_POLY: return launch_tc<256, PH_POLY, true>(P, 2 * pairs, s);
    default: return launch_tc<256, PH_APPLY, true>(P, 2 * pairs, s);
  }
}

cudaError_t launch_ns_phase_tc(const TcParams& P, int num_sms, cudaStream_t s) {
  const int total = P.args.tile_base[P.args.num_classes];
  if (total <= 0) return cudaSuccess;
  const int grid = total < num_sms ? total : num_sms;
  switch (P.args.phase) {
    case PH_GRAM: return launch_tc<256, PH_GRAM, false>(P, grid, s);
    case PH_POLY: return launch_tc<256, PH_POLY, false>(P, grid, s);
    default: return launch_tc<256, PH_APPLY, false>(P, grid, s);
  }
}

// Encodes a 3-D bf16 tensor map over a slab [count][rows][ld] with a
// box_inner x box_rows box (128B swizzle). Returns false on failure.
// The driver's cuTensorMapEncodeTiled, looked up once (thread-safe static init);
// null when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    cudaDriverEntryPointQueryResult qr;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

bool encode_slab_map_bf16(CUtensorMap* out, const void* base, int64_t inner, int64_t rows,
                          int64_t count, int64_t ld, int box_inner, int box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return false;
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

bool encode_chunk_map_bf16(CUtensorMap* out, const void* base, int64_t inner, int64_t rows,
                           int64_t count, int64_t ld, int box_chunks) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return false;
  if (ld % 64 != 0) return false;  // every chunk lies inside a slab row
  cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>((inner + 63) / 64), static_cast<cuuint64_t>(count)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(ld * 2), 128,
                           static_cast<cuuint64_t>(rows * ld * 2)};
  cuuint32_t box[4] = {64, 64, static_cast<cuuint32_t>(box_chunks), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace muon
