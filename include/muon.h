/*
 * muon.h - C ABI of libmuon.so, the Muon / MuonGS optimizer step for a stack of
 * 2-D weight matrices on NVIDIA B200 (sm_100a).
 *
 * What one step computes, per matrix W (rows x cols, the storage shape; an
 * nn.Linear weight is (out, in)):
 *   a1  M_t = mu*M_{t-1} + G_t                       (SGD momentum)
 *   a2  U   = G_t + mu*M_t     (Nesterov; U = M_t without MUON_NESTEROV)
 *   a3  X_0 = U / (||U||_F + eps)
 *   a4  tall matrices (rows > cols) are iterated through X^T (exact identity)
 *   a5  ns_steps times: S = X X^T; P = b*S + c*S*S; X = a*X + P*X
 *   a6  optional row-or-column RMS equilibration          (MUON_EQUILIBRATE)
 *   a7  O = s*O, s = scale_k*sqrt(max(rows, cols))       (MUON_SCALE_MOONLIGHT)
 *   a8  MuonGS: O~ = O - (<W,O>_F / ||W||_F^2) W         (MUON_MODE_MUONGS)
 *   a9  W <- (1 - lr*weight_decay) W - lr*O~
 * Sources (page title, section):
 *   "LLM Pretraining Loss Spike 진단과 처방 ... 그리고 Muon 전환 판단", section
 *     "AdamW에서 Muon으로 갈아탈 것인가": the Newton-Schulz listing (a3, a5, the
 *     Keller shape correction), the defaults (lr 0.02, momentum 0.95, Nesterov,
 *     5 steps) and the Moonlight sub-section (decoupled weight decay, a7, a9).
 *   "MuonGS: Pretraining LLMs with Relaxed Weight-Norm Control", section
 *     "전제와 한계": the Gram-Schmidt projection a8 and the C_T statistics.
 *   "[논문 AI 리뷰] MUON IS SCALABLE FOR LLM TRAINING TECHNICAL REPORT", section 2:
 *     the Newton-Schulz recurrence (a5) and the Eq. 4 update scale (a7).
 *   "행과 열을 함께 정규화하는 사전학습 옵티마이저 MeqMuon 공개", section "핵심 내용":
 *     row or column normalisation of the orthogonalised update (a6).
 *   "[Deep Learning] Muon — 행렬 업데이트를 직교화하는 옵티마이저", sections 3 and 5:
 *     the step order and the API conventions (a list of 2-D params; lr,
 *     momentum, weight_decay; a non-2-D parameter is an error).
 *
 * Precision: G is bf16 or fp32, W and M are fp32 and are updated in place.
 * Default Newton-Schulz path: bf16 operands on the tcgen05 tensor cores with
 * fp32 accumulation; X, S and P are stored in bf16 between the GEMMs, as in the
 * printed listing. MUON_NS_FP32 runs the iteration in fp32 on the CUDA cores.
 *
 * Conventions common to every call:
 *   - All matrix pointers are DEVICE pointers owned by the caller. The library
 *     never allocates device memory: scratch space is the caller's workspace.
 *   - Matrices are row-major with a leading dimension (elements) >= cols.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream and never synchronise, except
 *     muon_query_device_status.
 *   - Host-side validation happens before anything is enqueued; on error the
 *     call returns the status and nothing runs.
 *   - A plan object is not thread-safe; distinct plans may be used concurrently
 *     on distinct streams with distinct workspaces.
 */
#ifndef MUON_H_
#define MUON_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUON_ABI_VERSION 1

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, n < 0, bad hyper-parameter */
  MUON_ERR_SHAPE = 2,        /* rows or cols < 1, ld < cols, rows*cols >= 2^31 */
  MUON_ERR_DTYPE = 3,        /* W must be F32; grad F32 or BF16 */
  MUON_ERR_ALIAS = 4,        /* a written buffer (W, momentum) overlaps another buffer */
  MUON_ERR_WORKSPACE = 5,    /* workspace null, misaligned (256 B) or too small */
  MUON_ERR_CUDA = 6,         /* a CUDA runtime/driver call or a launch failed */
  MUON_ERR_TIMEOUT = 7,      /* device side: a bounded wait inside a kernel gave up */
  MUON_ERR_UNSUPPORTED = 8   /* the current device is not sm_100 (B200) */
} muon_status_t;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1 } muon_dtype_t;

typedef enum {
  MUON_MODE_MUON = 0,    /* plain Muon (with decoupled weight decay when wd > 0) */
  MUON_MODE_MUONGS = 1,  /* MuonGS: radial (Gram-Schmidt) projection before the update */
  MUON_MODE_MUONH = 2,   /* MuonH: fixed radius, W_{t+1} = ||W_t|| W' / ||W'|| with W' the
                            plain Muon update ("MuonGS: Pretraining LLMs with Relaxed
                            Weight-Norm Control", section 무엇과 다른가, names fixed-norm
                            control; the retraction form is this library's reading) */
  MUON_MODE_TWOSIDED = 3 /* for 2-D parameters that are not orthogonalised ("행과 열을 함께
                            정규화하는 ... MeqMuon 공개", section 핵심 내용): no Newton-Schulz;
                            the Frobenius-normalised Nesterov direction X is normalised along
                            rows and columns at once, N_ij = X_ij rho / ((sqrt(r_i)+eps)
                            (sqrt(c_j)+eps)), r / c the row / column mean squares of X and rho
                            its RMS (this library's reading; no formula on the page). Use
                            scale MUON_SCALE_NONE for an update of RMS about 1. ns_steps and
                            MUON_EQUILIBRATE are ignored; stats report w_norm only (the
                            other fields are NaN). */
} muon_mode_t;

typedef enum {
  MUON_SCALE_MOONLIGHT = 0, /* s = scale_k * sqrt(max(rows, cols)), scale_k = 0.2 by default */
  MUON_SCALE_KELLER = 1,    /* s = sqrt(max(1, rows/cols)) */
  MUON_SCALE_NONE = 2       /* s = 1 */
} muon_scale_t;

enum {
  MUON_NESTEROV = 1u,      /* U = G + mu*M (else U = M) */
  MUON_EQUILIBRATE = 2u,   /* row-or-column RMS equilibration after orthogonalisation */
  MUON_NS_FP32 = 4u,       /* fp32 Newton-Schulz on CUDA cores (else bf16 tensor cores) */
  MUON_WANT_STATS = 8u     /* reserved; stats are written whenever stats_dev != NULL */
};

/* One weight matrix. W: F32, updated in place. grad: F32 or BF16, read only.
 * momentum: F32, updated in place (it holds M_t after the call; zero it before
 * the first step). Leading dimensions are in elements. */
typedef struct {
  void* W;
  const void* grad;
  void* momentum;
  int64_t rows, cols;
  int64_t ld_w, ld_g, ld_m;
  int32_t w_dtype;   /* muon_dtype_t, must be MUON_F32 */
  int32_t g_dtype;   /* muon_dtype_t */
} muon_matrix_t;

typedef struct {
  float lr;              /* eta, 0.02 by default */
  float momentum;        /* mu, 0.95 */
  float weight_decay;    /* lambda, 0 (decay multiplies lr: W <- (1 - lr*wd) W) */
  float ns_coeffs[3];    /* (a, b, c) = (3.4445, -4.7750, 2.0315) */
  int32_t ns_steps;      /* 5; 0 <= ns_steps <= 64 */
  float eps;             /* 1e-7, added to ||U||_F (and to row/col RMS in a6) */
  int32_t mode;          /* muon_mode_t */
  int32_t scale;         /* muon_scale_t */
  float scale_k;         /* 0.2 */
  uint32_t flags;        /* MUON_NESTEROV | ... ; default MUON_NESTEROV */
} muon_hparams_t;

/* Per-matrix statistics of the step just taken (device memory, one entry per
 * matrix in the caller's order). C_T of the MuonGS page accumulates lr/w_norm. */
typedef struct {
  float w_norm;       /* ||W_t||_F before the step */
  float w_dot_o;      /* <W_t, O>_F with O after equilibration and scale */
  float o_norm;       /* ||O~||_F, the applied direction */
  float update_rms;   /* ||O~||_F / sqrt(rows*cols) */
  int32_t equil_axis; /* 0 none, 1 rows, 2 columns */
  int32_t reserved;
} muon_stats_t;

/* Library ABI version (MUON_ABI_VERSION). */
MUON_API int muon_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
MUON_API const char* muon_status_string(muon_status_t status);

/* Fills *hp with the defaults listed in muon_hparams_t. */
MUON_API muon_status_t muon_hparams_default(muon_hparams_t* hp);

/* Host-only validation of a matrix list and hyper-parameters (no CUDA call). */
MUON_API muon_status_t muon_validate(const muon_matrix_t* mats, int n, const muon_hparams_t* hp);

/* Workspace bytes muon_step_batched needs for this list (0 if the list is
 * invalid). Host only. The workspace must be 256-byte aligned device memory. */
MUON_API size_t muon_workspace_size(const muon_matrix_t* mats, int n, const muon_hparams_t* hp);

/* One step over n matrices. Groups the matrices by shape on the host, copies a
 * descriptor table into the workspace and launches the kernels on `stream`.
 * stats_dev: device array of n muon_stats_t, or NULL. n == 0 is a no-op. */
MUON_API muon_status_t muon_step_batched(const muon_matrix_t* mats, int n, const muon_hparams_t* hp,
                                void* workspace, size_t ws_bytes, muon_stats_t* stats_dev,
                                void* stream);

/* ---- cached plan: grouping and descriptor table built once for a fixed list ---- */
typedef struct muon_plan_s* muon_plan_t;

/* Validates and groups the list (host only, no CUDA call). On success *out owns
 * a copy of the list; the pointers inside must stay valid while the plan is used. */
MUON_API muon_status_t muon_plan_create(const muon_matrix_t* mats, int n, const muon_hparams_t* hp,
                               muon_plan_t* out);
MUON_API size_t muon_plan_workspace_size(muon_plan_t plan);
/* Replaces the hyper-parameters (e.g. a learning-rate schedule). Flags that change
 * the workspace layout (MUON_NS_FP32, MUON_EQUILIBRATE) must not change. */
MUON_API muon_status_t muon_plan_set_hparams(muon_plan_t plan, const muon_hparams_t* hp);
/* One step. The descriptor table is uploaded into the workspace on the first call
 * with a given workspace pointer and reused afterwards. */
MUON_API muon_status_t muon_plan_step(muon_plan_t plan, void* workspace, size_t ws_bytes,
                             muon_stats_t* stats_dev, void* stream);
MUON_API void muon_plan_destroy(muon_plan_t plan);

/* ---- Newton-Schulz only: O = NS(X / (||X||_F + eps)), for tests and benchmarks ----
 * X and O are device matrices of the given dtype (X and O may not overlap).
 * Uses ns_coeffs, ns_steps, eps and MUON_NS_FP32 from hp; other fields ignored.
 * The workspace size is muon_ns_workspace_size for the same list. */
typedef struct {
  const void* X;
  void* O;
  int64_t rows, cols, ld_x, ld_o;
  int32_t dtype;     /* MUON_F32 or MUON_BF16, for both X and O */
  int32_t reserved;
} muon_ns_matrix_t;

MUON_API size_t muon_ns_workspace_size(const muon_ns_matrix_t* mats, int n, const muon_hparams_t* hp);
MUON_API muon_status_t muon_newton_schulz_batched(const muon_ns_matrix_t* mats, int n,
                                         const muon_hparams_t* hp, void* workspace,
                                         size_t ws_bytes, void* stream);

/* ---- per-kernel device timing of a plan (CUDA events around each launch) ----
 * Kernel kinds: "ingest", "ns_gram", "ns_poly", "ns_apply", "post_reduce",
 * "post_finalize", "post_apply", "ns_fused" (the fp32 path's single launch over all
 * iterations of small matrices), "post_stats" (the statistics of MUON_MODE_MUON and
 * MUON_MODE_TWOSIDED, after post_apply). flops / bytes are the algorithmic work of the
 * recorded launches: Newton-Schulz flops count the symmetric Gram and polynomial
 * once (m(m+1)n and m^2(m+1)) and the apply 2m^2n; bytes count each kernel's own
 * inputs and outputs once (ingest: G, M read, M and X_0 written; post_reduce: W and
 * O read, or O alone in MUON_MODE_MUON and MUON_MODE_TWOSIDED, whose update needs no
 * scalar of W; post_apply: W read and written, O read). */
typedef struct {
  char name[32];
  int32_t launches;   /* launches recorded since the last read */
  float total_ms;     /* their summed device time */
  double flops;       /* their algorithmic flops */
  double bytes;       /* their algorithmic bytes */
} muon_profile_entry_t;

/* Turns event recording on (1) or off (0) for later muon_plan_step calls. */
MUON_API muon_status_t muon_plan_profile_enable(muon_plan_t plan, int enable);
/* Waits for the recorded events, writes up to max_entries kinds (in the order
 * listed above) and clears the record. Returns the number of kinds written,
 * or -1 on a CUDA error. */
MUON_API int muon_plan_profile_read(muon_plan_t plan, muon_profile_entry_t* out, int max_entries);

/* ---- Newton-Schulz of one matrix without any caller workspace ----
 * The pages have no counterpart of this call: it exists for callers that cannot
 * call cudaMalloc. Examples: code that runs under a memory pool or framework
 * allocator owning all device memory, which must not be bypassed; code that
 * cannot afford the device-wide synchronisation cudaMalloc/cudaFree may imply.
 * Same result as muon_newton_schulz_batched for that one matrix (X in, O out,
 * device pointers, dtype F32 or BF16 for both): the arguments are validated by
 * the same host checks (so they get the same status) and the same kernels and tile
 * shapes run. Scratch is the library's own
 * 32 MiB static device array, which every GPU that loads the library keeps
 * until exit. A matrix whose scratch needs exceed it is rejected with
 * MUON_ERR_WORKSPACE before anything is enqueued. In bf16 that is 2*(m*ld_n +
 * m*ld_m)*2 bytes plus 2 KiB, with m <= n the sorted sides and ld_* rounded up
 * to 64, so 1024 x 4096 fits and 2048 x 2048 does not.
 * All calls share that array: calls that overlap on the GPU (two streams or
 * two host threads) race and must be serialised by the caller. The first call
 * on each device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current), so make it before any stream capture.
 * status_dev: optional uint32 in device memory of the current device (anything
 * else is rejected with MUON_ERR_INVALID_ARG) that receives MUON_ERR_TIMEOUT if a
 * bounded wait inside a kernel gives up; it is cleared to 0 at the start of the
 * call. With status_dev == NULL a timeout is not reported anywhere: the word it
 * lands in belongs to the shared scratch and the next call clears it, and O may
 * then hold garbage. Pass a status word whenever the result matters. */
MUON_API muon_status_t muon_newton_schulz_noalloc(const muon_ns_matrix_t* mat,
                                                  const muon_hparams_t* hp, uint32_t* status_dev,
                                                  void* stream);

/* ---- QK-Clip (MuonClip) ----
 * "LLM Pretraining Loss Spike 진단과 처방", section "Moonlight와 MuonClip이 추가한 것"
 * (QK-Clip listing): for attention head h whose largest pre-softmax logit S_max[h]
 * exceeds tau, gamma_h = tau / S_max[h] (else 1); the head's non-rotary query and key
 * projection rows are multiplied by gamma_h^0.5, its rotary query rows by gamma_h,
 * and the rotary key shared by all heads is not touched.
 * A slice names rows [row0, row0 + rows) of a row-major fp32 device matrix W (all
 * `cols` columns, leading dimension ld) that belong to head `head` and are scaled by
 * gamma_head^power (0.5 or 1.0 in the listing). s_max_dev: device array of n_heads
 * floats (the caller's forward pass measures them). Slices of one call may not
 * overlap (MUON_ERR_ALIAS; a slice of zero rows overlaps nothing). cols is at most
 * 2^26 (MUON_ERR_SHAPE). Asynchronous on `stream`; no workspace. */
typedef struct {
  void* W;
  int64_t row0, rows, cols, ld;
  int32_t head;
  float power;
} muon_qk_slice_t;

MUON_API muon_status_t muon_qk_clip(const muon_qk_slice_t* slices, int n, const float* s_max_dev,
                                    int n_heads, float tau, void* stream);

/* Self-test of the device-side timeout path: launches one thread that waits, with
 * the same bounded wait the pipelined kernels use, on an mbarrier nothing arrives
 * at, for limit_cycles SM clock cycles (1 .. 2e9), then records MUON_ERR_TIMEOUT
 * in the workspace's error word (read it with muon_query_device_status). The
 * workspace needs only its first 256 bytes. Nothing faults and nothing hangs. */
MUON_API muon_status_t muon_wait_probe(void* workspace, int64_t limit_cycles, void* stream);

/* Reads the sticky device-side error word of the workspace (MUON_OK or
 * MUON_ERR_TIMEOUT) behind the work already enqueued on `stream`, clears it on that
 * stream, and synchronises `stream` only (no other stream and no device-wide wait). The word is zeroed when
 * a plan first uses a workspace and on every muon_step_batched /
 * muon_newton_schulz_batched call, so after those it reflects that call only. */
MUON_API muon_status_t muon_query_device_status(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MUON_H_ */
