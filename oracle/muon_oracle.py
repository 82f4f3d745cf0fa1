"""Float64 CPU oracle of the Muon / MuonGS optimizer step.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module. The CUDA library never calls it and
shares no code with it.

It is plain NumPy in float64, written for a reader to check against the pages
by eye: one function per step of the method, in the pages' order and notation,
with `@` (a library matmul) and `numpy.linalg.svd` as the only primitives.

Sources (page title, then section):
  [P1] "LLM Pretraining Loss Spike 진단과 처방: 배치 사이즈, Gradient Accumulation,
       그리고 Muon 전환 판단", section "AdamW에서 Muon으로 갈아탈 것인가":
       sub-section "Muon head의 실체는 하이브리드 옵티마이저다" (the Newton-Schulz
       listing and the default hyper-parameters) and "Moonlight와 MuonClip이 추가한
       것" (decoupled weight decay, the max(A,B) update scale).
  [P2] "MuonGS: Pretraining LLMs with Relaxed Weight-Norm Control", sections
       "어떻게 동작하나" (C_T, Proposition 3.1), "무엇과 다른가" (MuonW bound) and
       "전제와 한계" (Gram-Schmidt projection, Theorem 4.1, Proposition 4.2).
  [P3] "[논문 AI 리뷰] MUON IS SCALABLE FOR LLM TRAINING TECHNICAL REPORT",
       section 2 "Key Methods and Approach" (Newton-Schulz recurrence, Eq. 4 scale).
  [P4] "행과 열을 함께 정규화하는 사전학습 옵티마이저 MeqMuon 공개", section
       "핵심 내용" (row or column normalisation picked automatically).
  [P5] "[Deep Learning] Muon — 행렬 업데이트를 직교화하는 옵티마이저", section
       "3. Muon의 업데이트 순서" (step order) and "5. PyTorch 2.13 적용 예시".

Readings where the pages are silent (each one also listed in the design notes):
  * momentum: M_t = mu*M_{t-1} + G_t; Nesterov look-ahead U = G_t + mu*M_t.
  * normaliser: Frobenius norm, eps added to the norm.
  * tall matrices (rows > cols) are orthogonalised through their transpose, an
    exact identity of the recurrence (pinned by a test).
  * decoupled weight decay: W <- (1 - lr*wd) W.
  * equilibration: stateless row-or-column RMS balancing (see `equilibrate`).
    PARITY UNPINNED beyond the invariants its tests check: the pages give no formula.
  * GS projection is skipped when ||W||_F = 0.
  * MuonH (fixed-radius control, named in [P2]): W_{t+1} = ||W_t|| W' / ||W'||,
    W' the plain Muon update; the radius carries over, so it stays ||W_0||.
  * two-sided normalisation ([P4], MeqMuon's treatment of the 2-D parameters that
    are not orthogonalised; no formula on the pages): see `two_sided_normalise`.
    PARITY UNPINNED beyond its rank-one closed form.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

# [P1] Newton-Schulz listing: quintic coefficients (a, b, c) and 5 iterations.
QUINTIC = (3.4445, -4.7750, 2.0315)
# Classical cubic Newton-Schulz for the polar factor (textbook special case).
CUBIC = (1.5, -0.5, 0.0)

AXIS_NONE, AXIS_ROWS, AXIS_COLS = 0, 1, 2


@dataclasses.dataclass
class HParams:
    """Step hyper-parameters. Defaults: [P1] Muon defaults (lr 0.02, momentum 0.95,
    Nesterov on, 5 NS steps); the 0.2 scale constant of [P3] Eq. 4."""
    lr: float = 0.02
    momentum: float = 0.95
    weight_decay: float = 0.0
    nesterov: bool = True
    ns_coeffs: Tuple[float, float, float] = QUINTIC
    ns_steps: int = 5
    eps: float = 1e-7
    mode: str = "muon"           # "muon" | "muongs" | "muonh" | "twosided"
    scale: str = "moonlight"     # "moonlight" | "keller" | "none"
    scale_k: float = 0.2
    equilibrate: bool = False
    exact_polar: bool = False    # replace the NS iteration by the SVD polar factor
    equil_axis: Optional[int] = None  # force the equilibration axis (tests of near-ties)


@dataclasses.dataclass
class StepResult:
    W: np.ndarray          # W_{t+1}
    M: np.ndarray          # M_t
    O: np.ndarray          # orthogonalised, equilibrated and scaled update before projection
    O_tilde: np.ndarray    # update actually applied (after the GS projection in MuonGS mode)
    w_norm: float          # ||W_t||_F
    w_dot_o: float         # <W_t, O>_F
    o_norm: float          # ||O_tilde||_F
    update_rms: float      # ||O_tilde||_F / sqrt(rows*cols)
    equil_axis: int
    imbalances: Tuple[float, float] = (float("nan"), float("nan"))  # (rows, cols) before a6


# ---------------------------------------------------------------- step a1-a2
def momentum(M_prev: np.ndarray, G: np.ndarray, mu: float, nesterov: bool = True
             ) -> Tuple[np.ndarray, np.ndarray]:
    """SGD momentum M_t = mu*M_{t-1} + G_t and the direction U fed to orthogonalisation.

    [P1] ("SGD-momentum update", momentum 0.95, nesterov True); [P5] step 2
    (accumulate momentum, Nesterov by default). The pages print no formula; the
    reading is the SGD form with the Nesterov look-ahead U = G_t + mu*M_t.
    """
    M = mu * M_prev + G
    U = G + mu * M if nesterov else M
    return M, U


# ---------------------------------------------------------------- step a3
def frobenius_normalise(U: np.ndarray, eps: float = 1e-7) -> np.ndarray:
    """X_0 = U / (||U||_F + eps): [P1] listing (norm over both matrix dims, + 1e-7),
    which bounds the spectral norm of X_0 by 1; [P5] step 3."""
    return U / (np.linalg.norm(U) + eps)


# ---------------------------------------------------------------- step a5
def newton_schulz(X: np.ndarray, coeffs: Sequence[float] = QUINTIC, steps: int = 5) -> np.ndarray:
    """The Newton-Schulz iteration exactly as printed, with no change of orientation.

    [P1] listing: A = X X^T; B = b*A + c*A A; X = a*X + B X, repeated `steps` times.
    [P3] section 2: X_k = a X + b (X X^T) X + c (X X^T)^2 X, N = 5.
    """
    a, b, c = coeffs
    for _ in range(steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X


def polar_factor(U: np.ndarray) -> np.ndarray:
    """U_svd V_svd^T, the orthogonal factor the iteration approximates ([P1]: keeping
    the product of left and right singular vectors; [P3]: (M M^T)^{-1/2} M)."""
    Us, _, Vt = np.linalg.svd(U, full_matrices=False)
    return Us @ Vt


def orthogonalise(U: np.ndarray, hp: HParams) -> np.ndarray:
    """Steps a3-a5: normalise, then Newton-Schulz (or the exact polar factor).

    A tall matrix (rows > cols) is iterated through its transpose and transposed
    back: (X X^T) X = X (X^T X), so the recurrence on X^T is the transpose of the
    recurrence on X; only the Gram size changes, to min(rows, cols)^2.
    """
    X = frobenius_normalise(U, hp.eps)
    if hp.exact_polar:
        if not np.any(X):
            return np.zeros_like(X)
        return polar_factor(X)
    tall = X.shape[0] > X.shape[1]
    if tall:
        X = X.T
    X = newton_schulz(X, hp.ns_coeffs, hp.ns_steps)
    return X.T if tall else X


# ---------------------------------------------------------------- step a6
def _imbalance(v: np.ndarray) -> float:
    mean = v.mean()
    return float(v.std() / mean) if mean > 0 else 0.0


def line_imbalances(O: np.ndarray) -> Tuple[float, float]:
    """(imbalance of the row RMS vector, imbalance of the column RMS vector) of O, the
    two numbers `equilibrate` compares; imbalance(v) = std(v) / mean(v)."""
    return (_imbalance(np.sqrt(np.mean(O * O, axis=1))),
            _imbalance(np.sqrt(np.mean(O * O, axis=0))))


def equilibrate(O: np.ndarray, eps: float = 1e-7, axis: Optional[int] = None
                ) -> Tuple[np.ndarray, int]:
    """Row-or-column RMS equilibration of the orthogonalised update.

    [P4] section 핵심 내용: NorMuon normalises per row; MeqMuon picks row or column
    normalisation per matrix to match its imbalance pattern. The pages give no
    formula. Reading: r_i = RMS of row i, c_j = RMS of column j, imbalance(v) =
    std(v)/mean(v); rows are balanced if imbalance(r) >= imbalance(c), else
    columns; each chosen line is rescaled to the global RMS rho = RMS(O):
    O_ij <- O_ij * rho / (r_i + eps) (columns likewise), which keeps ||O||_F.
    Closed form: a line-scaled sign matrix D_r Z (or Z D_c) picks rows (columns) and maps
    to RMS(O) * Z. PARITY UNPINNED beyond that closed form and the invariants.
    `axis` (AXIS_ROWS or AXIS_COLS) overrides the choice; the tests use it to follow the
    other valid result when the two imbalances are a floating-point tie.
    """
    r = np.sqrt(np.mean(O * O, axis=1))
    c = np.sqrt(np.mean(O * O, axis=0))
    rho = np.sqrt(np.mean(O * O))
    if axis is None:
        ir, ic = line_imbalances(O)
        axis = AXIS_ROWS if ir >= ic else AXIS_COLS
    if axis == AXIS_ROWS:
        return O * (rho / (r + eps))[:, None], AXIS_ROWS
    return O * (rho / (c + eps))[None, :], AXIS_COLS


def two_sided_normalise(X: np.ndarray, eps: float = 1e-7) -> np.ndarray:
    """Two-sided (row and column at once) normalisation of a momentum matrix, [P4]
    section 핵심 내용: MeqMuon normalises the momentum of the 2-D parameters it does not
    orthogonalise along both rows and columns, without storing a second moment. The
    pages give no formula. Reading: with r_i and c_j the mean squares of row i and
    column j and rho the RMS of X, N_ij = X_ij rho / ((sqrt(r_i) + eps)(sqrt(c_j) + eps)),
    the rank-one (row x column) estimate of the second moment a second-moment
    optimizer would divide by. Closed form: a scaled sign matrix X = D_r Z D_c (Z of
    +-1 entries, D_r, D_c positive diagonal) maps to Z; rank one, X = u v^T, maps to
    sign(u) sign(v)^T. PARITY UNPINNED beyond that closed form."""
    r = np.mean(X * X, axis=1)
    c = np.mean(X * X, axis=0)
    rho = np.sqrt(np.mean(X * X))
    return X * rho / ((np.sqrt(r) + eps)[:, None] * (np.sqrt(c) + eps)[None, :])


# ---------------------------------------------------------------- step a7
def update_scale(rows: int, cols: int, rule: str = "moonlight", k: float = 0.2) -> float:
    """Per-matrix update scale.

    moonlight: k*sqrt(max(A, B)), k = 0.2 ([P3] Eq. 4; [P1] Moonlight sub-section),
               bringing the update RMS from sqrt(1/max(A,B)) to k.
    keller:    sqrt(max(1, rows/cols)) ([P1] listing, last line, shape correction).
    none:      1.
    """
    if rule == "moonlight":
        return k * float(np.sqrt(max(rows, cols)))
    if rule == "keller":
        return float(np.sqrt(max(1.0, rows / cols)))
    if rule == "none":
        return 1.0
    raise ValueError(rule)


# ---------------------------------------------------------------- step a8
def gs_project(W: np.ndarray, O: np.ndarray) -> np.ndarray:
    """MuonGS radial projection O~ = O - (<W, O>_F / ||W||_F^2) W ([P2] 전제와 한계).
    Skipped when ||W||_F = 0 (reading: the radial direction is undefined)."""
    r2 = float(np.sum(W * W))
    if r2 == 0.0:
        return O.copy()
    return O - (float(np.sum(W * O)) / r2) * W


# ---------------------------------------------------------------- step a9
def apply_update(W: np.ndarray, O_tilde: np.ndarray, lr: float, wd: float) -> np.ndarray:
    """Decoupled weight decay and the update: W <- (1 - lr*wd) W - lr*O~.
    [P1] Moonlight sub-section (AdamW-style weight decay added to Muon); [P5] step 5."""
    return (1.0 - lr * wd) * W - lr * O_tilde


def retract_to_radius(W_new: np.ndarray, radius: float) -> np.ndarray:
    """MuonH's fixed-radius control ([P2] 무엇과 다른가: MuonH keeps the weight norm at a
    fixed radius R, so C_T = eta T / R). The pages print no retraction; reading: rescale
    the updated matrix back to the radius, W <- R W / ||W||, with R = ||W_t||."""
    n = float(np.linalg.norm(W_new))
    return W_new if n == 0.0 else (radius / n) * W_new


# ---------------------------------------------------------------- whole step
def muon_step(W: np.ndarray, G: np.ndarray, M_prev: np.ndarray, hp: HParams) -> StepResult:
    """One Muon / MuonGS step of one matrix, steps a1-a9 in the order of [P5] section 3:
    momentum (+Nesterov) -> normalise -> Newton-Schulz -> [equilibrate] -> scale ->
    [GS projection] -> decoupled weight decay and update."""
    W = np.asarray(W, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M_prev = np.asarray(M_prev, dtype=np.float64)
    if W.ndim != 2:
        raise ValueError("Muon takes 2-D matrices only")
    rows, cols = W.shape
    M, U = momentum(M_prev, G, hp.momentum, hp.nesterov)
    axis = AXIS_NONE
    imb = (float("nan"), float("nan"))
    if hp.mode == "twosided":
        O = two_sided_normalise(frobenius_normalise(U, hp.eps), hp.eps)
        axis = 3
    else:
        O = orthogonalise(U, hp)
        if hp.equilibrate:
            imb = line_imbalances(O)
            O, axis = equilibrate(O, hp.eps, hp.equil_axis)
    O = update_scale(rows, cols, hp.scale, hp.scale_k) * O
    w_norm = float(np.linalg.norm(W))
    w_dot_o = float(np.sum(W * O))
    O_tilde = gs_project(W, O) if hp.mode == "muongs" else O
    o_norm = float(np.linalg.norm(O_tilde))
    W_next = apply_update(W, O_tilde, hp.lr, hp.weight_decay)
    if hp.mode == "muonh":
        W_next = retract_to_radius(W_next, w_norm)
    return StepResult(W_next, M, O, O_tilde, w_norm, w_dot_o, o_norm,
                      o_norm / np.sqrt(rows * cols), axis, imb)


def muon_run(W0: np.ndarray, grads: Sequence[np.ndarray], hp: HParams,
             M0: Optional[np.ndarray] = None) -> List[StepResult]:
    """Consecutive steps from W0 and zero (or given) momentum, one gradient per step."""
    W = np.asarray(W0, dtype=np.float64)
    M = np.zeros_like(W) if M0 is None else np.asarray(M0, dtype=np.float64)
    out = []
    for G in grads:
        r = muon_step(W, G, M, hp)
        out.append(r)
        W, M = r.W, r.M
    return out


# ---------------------------------------------------------------- measurements
def accumulated_lr(lrs: Sequence[float], w_norms: Sequence[float]) -> float:
    """C_T = sum_t eta_t / ||W_t||_F over t = 0..T-1 with the pre-step W_t ([P2] 어떻게 동작하나)."""
    return float(sum(e / r for e, r in zip(lrs, w_norms)))


def muongs_ct_lower_bound(r0: float, p: float, eta: float, T: int) -> float:
    """[P2] Theorem 4.1: C_T >= (2/(p eta)) (sqrt(r0^2 + p eta^2 T) - r0)."""
    return 2.0 / (p * eta) * (np.sqrt(r0 * r0 + p * eta * eta * T) - r0)


def muongs_late_lower_bound(r0: float, p: float, eta: float, T: int) -> float:
    """[P2] Proposition 4.2: C_2T - C_T >= eta T / sqrt(r0^2 + 2 p eta^2 T)."""
    return eta * T / np.sqrt(r0 * r0 + 2.0 * p * eta * eta * T)


def muonw_radius(r0: float, p: float, lam: float) -> float:
    """[P2] 무엇과 다른가: R_lambda = max{r0, sqrt(p)/lambda}; MuonW keeps ||W_t|| <= R_lambda
    and C_T >= eta T / R_lambda."""
    return max(r0, np.sqrt(p) / lam)


# ---------------------------------------------------------------- QK-Clip
def qk_clip(weights: Sequence[np.ndarray], slices: Sequence[Tuple[int, int, int, int, float]],
            s_max: Sequence[float], tau: float = 100.0) -> List[np.ndarray]:
    """QK-Clip of [P1] (section "Moonlight와 MuonClip이 추가한 것", the QK-Clip listing):
    for each head h, gamma_h = min(1, tau / S_max[h]); the head's non-rotary query and
    key projections are multiplied by gamma^0.5, its rotary query projection by gamma,
    and the rotary key (shared by all heads) is left alone.

    `slices` lists (weight index, first row, row count, head, power): rows
    [first, first+count) of weights[index] belong to head `head` and are scaled by
    gamma_head ** power (0.5 for non-rotary q / k, 1.0 for rotary q). Returns new arrays.
    """
    out = [np.array(w, dtype=np.float64, copy=True) for w in weights]
    for wi, r0, nr, h, power in slices:
        gamma = min(1.0, tau / s_max[h])
        out[wi][r0:r0 + nr, :] *= gamma ** power
    return out
