"""Pins of the float64 oracle to facts that do not come from the oracle itself.

Each test ties one step of the oracle to a closed form, a textbook special case,
a hand-worked value, or an invariant/bound printed on the pages, so that a
dropped term, a wrong sign, a wrong index or a transposed operand fails.
"""
import numpy as np
import pytest

from oracle import muon_oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

# Coefficients as printed in the Newton-Schulz listing of "LLM Pretraining Loss Spike
# 진단과 처방" (section "Muon head의 실체는 하이브리드 옵티마이저다").
A_, B_, C_ = 3.4445, -4.7750, 2.0315


def _orthonormal(rng, n, k):
    q, _ = np.linalg.qr(rng.standard_normal((n, k)))
    return q


def _with_singular_values(rng, rows, cols, sigma):
    k = min(rows, cols)
    U = _orthonormal(rng, rows, k)
    V = _orthonormal(rng, cols, k)
    return U @ np.diag(sigma) @ V.T, U, V


def _scalar_quintic(x, steps):
    for _ in range(steps):
        x = A_ * x + B_ * x ** 3 + C_ * x ** 5
    return x


@pytest.mark.parametrize("rows,cols", [(6, 10), (10, 6), (8, 8), (1, 7), (7, 1), (1, 1)])
def test_ns_acts_on_each_singular_value(rows, cols):
    """Closed form: for X = U diag(s) V^T the recurrence maps each s_i through
    f(x) = a x + b x^3 + c x^5 independently, so NS_5(X) = U diag(f^5(s)) V^T."""
    rng = np.random.default_rng(1)
    k = min(rows, cols)
    sigma = np.linspace(0.05, 1.0, k)
    X, U, V = _with_singular_values(rng, rows, cols, sigma)
    want = U @ np.diag(_scalar_quintic(sigma, 5)) @ V.T
    hp = orc.HParams(eps=0.0)
    # orthogonalise() normalises first; undo that by feeding X scaled so that
    # ||X||_F = 1 and comparing with the same singular values.
    Xn = X / np.linalg.norm(X)
    want = U @ np.diag(_scalar_quintic(sigma / np.linalg.norm(sigma), 5)) @ V.T
    got = orc.orthogonalise(Xn * 3.7, hp)        # normalisation removes the 3.7
    assert np.linalg.norm(got - want) <= 1e-12 * max(1.0, np.linalg.norm(want))
    # the literal recurrence, no orientation change, gives the same matrix
    lit = orc.newton_schulz(Xn, orc.QUINTIC, 5)
    assert np.linalg.norm(lit - want) <= 1e-12 * max(1.0, np.linalg.norm(want))


@pytest.mark.parametrize("rows,cols", [(4, 6), (8, 8), (6, 4)])
def test_cubic_newton_schulz_converges_to_polar_factor(rows, cols):
    """Textbook special case: (a,b,c) = (1.5, -0.5, 0) is the classical Newton-Schulz
    polar iteration; on a well-conditioned matrix it reaches U V^T of the SVD."""
    rng = np.random.default_rng(2)
    k = min(rows, cols)
    sigma = np.linspace(0.1, 1.0, k)             # condition number 10
    X, _, _ = _with_singular_values(rng, rows, cols, sigma)
    hp = orc.HParams(ns_coeffs=orc.CUBIC, ns_steps=60, eps=0.0)
    got = orc.orthogonalise(X, hp)
    Us, _, Vt = np.linalg.svd(X, full_matrices=False)
    assert np.abs(got - Us @ Vt).max() <= 1e-12


@pytest.mark.parametrize("rows,cols", [(9, 5), (12, 3), (16, 15)])
def test_transposed_iteration_is_exact_for_tall_matrices(rows, cols):
    """(X X^T) X = X (X^T X): iterating on X^T and transposing back equals the
    literal recurrence on the tall X."""
    rng = np.random.default_rng(3)
    X = rng.standard_normal((rows, cols))
    X /= np.linalg.norm(X)
    lit = orc.newton_schulz(X, orc.QUINTIC, 5)
    via_t = orc.newton_schulz(X.T, orc.QUINTIC, 5).T
    assert np.abs(lit - via_t).max() <= 1e-12
    got = orc.orthogonalise(X, orc.HParams(eps=0.0))
    assert np.abs(got - lit).max() <= 1e-12


def test_frobenius_normalisation_bounds_spectral_norm():
    rng = np.random.default_rng(4)
    U = rng.standard_normal((20, 33)) * 1e-3
    X = orc.frobenius_normalise(U, 1e-7)
    nu = np.sqrt(np.sum(U * U))
    assert abs(np.sqrt(np.sum(X * X)) - nu / (nu + 1e-7)) < 1e-15
    assert np.linalg.norm(X, 2) <= 1.0
    # eps is added to the norm, not to its square: hand value for a 1x1 matrix
    assert orc.frobenius_normalise(np.array([[3.0]]), 1.0)[0, 0] == pytest.approx(0.75, abs=0)


def test_momentum_matches_geometric_sum():
    """M_T = sum_t mu^(T-t) G_t from zero momentum; Nesterov U = G_T + mu M_T."""
    rng = np.random.default_rng(5)
    mu, T = 0.95, 7
    Gs = rng.standard_normal((T, 3, 4))
    M = np.zeros((3, 4))
    for t in range(T):
        M, U = orc.momentum(M, Gs[t], mu, nesterov=True)
    weights = mu ** np.arange(T - 1, -1, -1)
    M_closed = np.tensordot(weights, Gs, axes=1)
    assert np.abs(M - M_closed).max() < 1e-14
    assert np.abs(U - (Gs[-1] + mu * M_closed)).max() < 1e-14
    _, U_plain = orc.momentum(np.zeros((3, 4)), Gs[0], mu, nesterov=False)
    assert np.array_equal(U_plain, Gs[0])


def test_two_step_update_through_the_svd():
    """Whole-step composition from an independent route: the Nesterov direction of
    step 2 is (1+mu) G2 + mu^2 G1, its NS image is U diag(f^5(s/||s||)) V^T."""
    rng = np.random.default_rng(6)
    rows, cols, mu, lr, wd = 5, 8, 0.95, 0.02, 0.1
    W0 = rng.standard_normal((rows, cols)) * 0.02
    G1 = rng.standard_normal((rows, cols)) * 1e-3
    G2 = rng.standard_normal((rows, cols)) * 1e-3
    hp = orc.HParams(lr=lr, momentum=mu, weight_decay=wd, mode="muongs", eps=0.0)
    r1, r2 = orc.muon_run(W0, [G1, G2], hp)
    U2 = (1 + mu) * G2 + mu * mu * G1
    Us, s, Vt = np.linalg.svd(U2, full_matrices=False)
    O = Us @ np.diag(_scalar_quintic(s / np.sqrt(np.sum(s * s)), 5)) @ Vt
    O *= 0.2 * np.sqrt(max(rows, cols))
    W1 = r1.W
    Ot = O - (np.sum(W1 * O) / np.sum(W1 * W1)) * W1
    W2 = (1 - lr * wd) * W1 - lr * Ot
    assert np.abs(r2.W - W2).max() < 1e-14
    assert np.abs(r2.M - (mu * G1 + G2)).max() < 1e-18


@pytest.mark.parametrize("rows,cols", [(16, 48), (48, 16), (32, 32)])
def test_moonlight_scale_gives_rms_0p2_for_exact_polar(rows, cols):
    """Eq. 4 of the Moonlight review: a full-rank orthogonal update has RMS
    sqrt(1/max(A,B)); scaling by 0.2 sqrt(max(A,B)) makes it exactly 0.2."""
    rng = np.random.default_rng(7)
    O = orc.polar_factor(rng.standard_normal((rows, cols)))
    assert np.sqrt(np.mean(O * O)) == pytest.approx(np.sqrt(1.0 / max(rows, cols)), rel=1e-13)
    s = orc.update_scale(rows, cols, "moonlight", 0.2)
    assert np.sqrt(np.mean((s * O) ** 2)) == pytest.approx(0.2, rel=1e-13)
    assert orc.update_scale(rows, cols, "keller") == pytest.approx(np.sqrt(max(1.0, rows / cols)))


def test_quintic_rms_is_close_to_0p2():
    """The quintic does not reach singular values 1 exactly; record the RMS on a
    random gradient (no page figure to assert against, only a sanity band)."""
    rng = np.random.default_rng(8)
    G = rng.standard_normal((128, 256)) * 1e-3
    O = orc.orthogonalise(G, orc.HParams()) * orc.update_scale(128, 256)
    rms = np.sqrt(np.mean(O * O))
    assert 0.1 < rms < 0.3


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_muongs_invariants(wd):
    """MuonGS (전제와 한계): <W, O~> = 0, ||O~|| <= ||O||, ||O~|| <= sqrt(p) at scale 1
    with the exact polar factor, and ||W_{t+1}||^2 = (1-lr wd)^2 ||W_t||^2 + lr^2 ||O~||^2
    (the wd = 0 case is the page's r_{t+1}^2 = r_t^2 + eta^2 ||O~||^2)."""
    rng = np.random.default_rng(9)
    rows, cols, lr = 12, 20, 0.02
    W = rng.standard_normal((rows, cols)) * 0.02
    p = min(rows, cols)
    for exact, scale in [(True, "none"), (False, "moonlight")]:
        hp = orc.HParams(mode="muongs", weight_decay=wd, exact_polar=exact, scale=scale)
        r = orc.muon_step(W, rng.standard_normal((rows, cols)) * 1e-3, np.zeros_like(W), hp)
        cos = np.sum(W * r.O_tilde) / (np.linalg.norm(W) * np.linalg.norm(r.O_tilde))
        assert abs(cos) <= 1e-12
        assert np.linalg.norm(r.O_tilde) <= np.linalg.norm(r.O) * (1 + 1e-15)
        if exact:
            assert np.linalg.norm(r.O_tilde) <= np.sqrt(p)
        lhs = np.sum(r.W * r.W)
        rhs = (1 - lr * wd) ** 2 * np.sum(W * W) + lr * lr * np.sum(r.O_tilde ** 2)
        assert lhs == pytest.approx(rhs, rel=1e-12)


def test_gs_projection_hand_value_and_zero_weight():
    W = np.array([[1.0, 0.0], [0.0, 0.0]])
    O = np.array([[2.0, 3.0], [4.0, 5.0]])
    # <W,O> = 2, ||W||^2 = 1 -> O~ = O - 2W
    assert np.array_equal(orc.gs_project(W, O), np.array([[0.0, 3.0], [4.0, 5.0]]))
    assert np.array_equal(orc.gs_project(np.zeros((2, 2)), O), O)


def test_accumulated_lr_meets_muongs_bounds():
    """Theorem 4.1 / Proposition 4.2 over a constant-lr run (64x128, scale 1, wd 0)."""
    rng = np.random.default_rng(10)
    rows, cols, eta, T = 64, 128, 0.02, 200
    p = min(rows, cols)
    W0 = rng.standard_normal((rows, cols)) * 0.02
    grads = [rng.standard_normal((rows, cols)) * 1e-3 for _ in range(2 * T)]
    for exact in (True, False):
        hp = orc.HParams(lr=eta, mode="muongs", scale="none", exact_polar=exact)
        res = orc.muon_run(W0, grads, hp)
        norms = [r.w_norm for r in res]
        r0 = norms[0]
        p_eff = p if exact else max(r.o_norm ** 2 for r in res)
        assert p_eff <= p * 1.5
        CT = orc.accumulated_lr([eta] * T, norms[:T])
        C2T = orc.accumulated_lr([eta] * (2 * T), norms)
        assert CT >= orc.muongs_ct_lower_bound(r0, p_eff, eta, T)
        assert C2T - CT >= orc.muongs_late_lower_bound(r0, p_eff, eta, T)
        # norm growth is only second order: r_T^2 <= r_0^2 + p eta^2 T
        assert norms[T] ** 2 <= r0 ** 2 + p_eff * eta ** 2 * T * (1 + 1e-12)


def test_muonw_radius_bound():
    """무엇과 다른가: with decoupled decay, ||W_t|| <= R = max(r0, sqrt(p)/lambda) and
    C_T >= eta T / R (exact polar update, scale 1)."""
    rng = np.random.default_rng(11)
    rows, cols, eta, lam, T = 8, 16, 0.05, 2.0, 300
    p = min(rows, cols)
    W0 = rng.standard_normal((rows, cols)) * 0.02
    hp = orc.HParams(lr=eta, weight_decay=lam, scale="none", exact_polar=True)
    res = orc.muon_run(W0, [rng.standard_normal((rows, cols)) for _ in range(T)], hp)
    R = orc.muonw_radius(np.linalg.norm(W0), p, lam)
    assert all(r.w_norm <= R * (1 + 1e-12) for r in res)
    assert orc.accumulated_lr([eta] * T, [r.w_norm for r in res]) >= eta * T / R


def test_bound_helpers_hand_values():
    """The three bound helpers of the MuonGS page at hand-computed points.
    Theorem 4.1: (2/(p eta)) (sqrt(r0^2 + p eta^2 T) - r0);
    Proposition 4.2: eta T / sqrt(r0^2 + 2 p eta^2 T);
    무엇과 다른가: R_lambda = max(r0, sqrt(p) / lambda)."""
    # r0 = 0, p = 4, eta = 1/2, T = 4: (2/2) * sqrt(4) = 2
    assert orc.muongs_ct_lower_bound(0.0, 4, 0.5, 4) == pytest.approx(2.0, rel=1e-15)
    # r0 = 3, p = 16, eta = 1/4, T = 7: p eta^2 T = 7, sqrt(16) - 3 = 1, 2/(16/4) = 1/2
    assert orc.muongs_ct_lower_bound(3.0, 16, 0.25, 7) == pytest.approx(0.5, rel=1e-15)
    # r0 = 2, p = 3, eta = 1, T = 2: 2 p eta^2 T = 12, sqrt(16) = 4, eta T / 4 = 1/2
    assert orc.muongs_late_lower_bound(2.0, 3, 1.0, 2) == pytest.approx(0.5, rel=1e-15)
    # r0 = 0, p = 8, eta = 1/2, T = 1: 2 p eta^2 T = 4 -> 1/2 / 2 = 1/4
    assert orc.muongs_late_lower_bound(0.0, 8, 0.5, 1) == pytest.approx(0.25, rel=1e-15)
    assert orc.muonw_radius(1.0, 16, 2.0) == pytest.approx(2.0, rel=1e-15)   # sqrt(16)/2
    assert orc.muonw_radius(5.0, 16, 2.0) == pytest.approx(5.0, rel=1e-15)   # r0 wins
    assert orc.muonw_radius(0.5, 9, 0.5) == pytest.approx(6.0, rel=1e-15)    # sqrt(9)/0.5


def test_muongs_bounds_are_tight_for_exact_polar_updates():
    """Sandwich of Theorem 4.1 and Proposition 4.2 on a MuonGS run with the exact polar
    factor (scale 1, wd 0, momentum 0 so that each update is independent of W_t). The
    projection makes O~ orthogonal to W_t, so the norm recursion r_{t+1}^2 = r_t^2 +
    eta^2 ||O~_t||^2 is exact and ||O~_t||^2 stays within a hair of p (independent random
    gradients are almost orthogonal to W). With p_lo / p_hi the
    smallest / largest ||O~_t||^2 of the run, for the decreasing 1/sqrt(.) sum:
        bound_41(p_hi) <= C_T <= eta / r0 + bound_41(p_lo)
    and the window C_2T - C_T lies between bound_42(p_hi) and 1.25 bound_42(p_lo)
    (the exact sum over the window is 2 (sqrt 2 - 1) / (1/sqrt 2) = 1.17 times the
    bound for large T). A loosened or mis-scaled bound (a factor 2, a dropped square
    root, a missing p) falls outside one side."""
    rng = np.random.default_rng(13)
    rows, cols, eta, T = 64, 128, 0.02, 200
    p = min(rows, cols)
    W0 = rng.standard_normal((rows, cols)) * 0.02
    grads = [rng.standard_normal((rows, cols)) * 1e-3 for _ in range(2 * T)]
    hp = orc.HParams(lr=eta, momentum=0.0, mode="muongs", scale="none", exact_polar=True)
    res = orc.muon_run(W0, grads, hp)
    norms = [r.w_norm for r in res]
    o2 = [r.o_norm ** 2 for r in res]
    p_lo, p_hi = min(o2), max(o2)
    assert p_hi <= p * (1 + 1e-12) and p_lo >= 0.99 * p
    r0 = norms[0]
    CT = orc.accumulated_lr([eta] * T, norms[:T])
    C2T = orc.accumulated_lr([eta] * (2 * T), norms)
    lo = orc.muongs_ct_lower_bound(r0, p_hi, eta, T)
    hi = eta / r0 + orc.muongs_ct_lower_bound(r0, p_lo, eta, T)
    assert lo <= CT <= hi
    assert hi - lo <= 0.02 * CT        # the sandwich is narrow: the bound is tight here
    assert orc.muongs_late_lower_bound(r0, p_hi, eta, T) <= C2T - CT
    assert C2T - CT <= 1.25 * orc.muongs_late_lower_bound(r0, p_lo, eta, T)


def test_muonw_radius_is_reached_by_an_aligned_update():
    """Tightness of R_lambda = max(r0, sqrt(p)/lambda): with W_t = a_t Q for a fixed
    semi-orthogonal Q (||Q||_F^2 = p) and the constant gradient -Q, the exact polar
    update is O = -Q, so a_{t+1} = (1 - eta lambda) a_t + eta converges to 1/lambda and
    ||W_t|| = a_t sqrt(p) rises to sqrt(p)/lambda from below, never above it."""
    rows, cols, eta, lam, T = 8, 16, 0.05, 2.0, 400
    p = min(rows, cols)
    Q = orc.polar_factor(np.random.default_rng(14).standard_normal((rows, cols)))
    W0 = 0.1 * Q
    hp = orc.HParams(lr=eta, weight_decay=lam, scale="none", exact_polar=True)
    res = orc.muon_run(W0, [-Q] * T, hp)
    R = orc.muonw_radius(np.linalg.norm(W0), p, lam)
    assert R == pytest.approx(np.sqrt(p) / lam, rel=1e-15)
    assert all(r.w_norm <= R * (1 + 1e-12) for r in res)
    assert np.linalg.norm(res[-1].W) == pytest.approx(R, rel=1e-9)


def test_equilibration_hand_worked():
    """Rows of O have equal RMS (sqrt 3 each) so the columns are balanced:
    c = (sqrt(1/2), sqrt 2, sqrt(13/2)), rho = sqrt 3, O_ij <- O_ij rho / c_j."""
    O = np.array([[1.0, 2.0, 2.0], [0.0, 0.0, 3.0]])
    got, axis = orc.equilibrate(O, eps=0.0)
    assert axis == orc.AXIS_COLS
    c = np.array([np.sqrt(0.5), np.sqrt(2.0), np.sqrt(6.5)])
    assert np.allclose(got, O * np.sqrt(3.0) / c[None, :], rtol=0, atol=1e-15)
    got_t, axis_t = orc.equilibrate(O.T, eps=0.0)
    assert axis_t == orc.AXIS_ROWS
    assert np.allclose(got_t, got.T, rtol=0, atol=1e-15)
    # row RMS (sqrt 3, sqrt 3): imbalance 0; column RMS above: imbalance > 0
    ir, ic = orc.line_imbalances(O)
    assert ir == 0.0 and ic > 0.3
    # forcing the other axis scales the rows to rho: here the identity (r_i = rho)
    forced, ax = orc.equilibrate(O, eps=0.0, axis=orc.AXIS_ROWS)
    assert ax == orc.AXIS_ROWS and np.allclose(forced, O, rtol=0, atol=1e-15)
    same, ax = orc.equilibrate(O, eps=0.0, axis=orc.AXIS_COLS)
    assert ax == orc.AXIS_COLS and np.array_equal(same, got)


@pytest.mark.parametrize("rows,cols", [(16, 16), (8, 24), (24, 8)])
def test_equilibration_invariants(rows, cols):
    rng = np.random.default_rng(12)
    O = orc.polar_factor(rng.standard_normal((rows, cols)))
    got, axis = orc.equilibrate(O, eps=1e-7)
    assert np.linalg.norm(got) == pytest.approx(np.linalg.norm(O), rel=1e-5)
    if rows == cols:
        assert np.abs(got - O).max() < 1e-5          # all lines already unit RMS
    elif rows < cols:
        assert axis == orc.AXIS_COLS                 # rows are orthonormal, hence balanced
    else:
        assert axis == orc.AXIS_ROWS
    rms = np.sqrt(np.mean(got * got, axis=1 if axis == orc.AXIS_ROWS else 0))
    assert np.ptp(rms) <= 1e-5 * rms.mean()


def test_degenerate_inputs():
    """Zero gradient and momentum: X_0 = 0, NS(0) = 0, only the decay acts.
    Zero weight in MuonGS mode: the projection is skipped."""
    W = np.ones((3, 5))
    hp = orc.HParams(weight_decay=0.1, mode="muongs")
    r = orc.muon_step(W, np.zeros((3, 5)), np.zeros((3, 5)), hp)
    assert np.array_equal(r.W, (1 - 0.02 * 0.1) * W)
    r0 = orc.muon_step(np.zeros((3, 5)), np.ones((3, 5)), np.zeros((3, 5)), hp)
    assert np.array_equal(r0.O_tilde, r0.O)
    with pytest.raises(ValueError):
        orc.muon_step(np.ones(4), np.ones(4), np.zeros(4), hp)


def test_rank_one_input_closed_form():
    """A rank-one U = u v^T has one singular value; after normalisation it is 1/(1+eps/||U||),
    so O = f^5(x) (u/|u|)(v/|v|)^T."""
    u = np.array([1.0, -2.0, 2.0])
    v = np.array([0.5, 0.5, -0.5, 0.5, 1.0])
    U = np.outer(u, v)
    nrm = np.linalg.norm(u) * np.linalg.norm(v)
    x = nrm / (nrm + 1e-7)
    want = _scalar_quintic(x, 5) * np.outer(u / np.linalg.norm(u), v / np.linalg.norm(v))
    got = orc.orthogonalise(U, orc.HParams())
    assert np.abs(got - want).max() < 1e-14


def test_muonh_keeps_the_radius_and_ct_is_linear():
    """Fixed-norm control (MuonGS page, 무엇과 다른가): ||W_t|| = R for all t and
    C_T = eta T / R exactly."""
    rng = np.random.default_rng(13)
    rows, cols, eta, T = 24, 40, 0.02, 50
    W0 = rng.standard_normal((rows, cols)) * 0.02
    R = np.linalg.norm(W0)
    hp = orc.HParams(lr=eta, mode="muonh", weight_decay=0.1)
    res = orc.muon_run(W0, [rng.standard_normal((rows, cols)) * 1e-3 for _ in range(T)], hp)
    assert all(abs(r.w_norm - R) <= 1e-12 * R for r in res)
    assert abs(np.linalg.norm(res[-1].W) - R) <= 1e-12 * R
    assert orc.accumulated_lr([eta] * T, [r.w_norm for r in res]) == pytest.approx(eta * T / R, rel=1e-12)
    # one step by hand: the plain Muon update rescaled to ||W_0||
    plain = orc.muon_step(W0, res[0].M, np.zeros_like(W0), orc.HParams(lr=eta, weight_decay=0.1))
    assert np.abs(res[0].W - plain.W * (R / np.linalg.norm(plain.W))).max() < 1e-15


def test_qk_clip_hand_values():
    """The QK-Clip listing with tau = 100: a head with S_max = 400 has gamma = 1/4, so its
    non-rotary q and k rows are halved and its rotary q rows quartered; a head with
    S_max = 50 is untouched, and so is the shared rotary key."""
    Wq = np.ones((8, 3))          # heads 0, 1: rows 0-3 / 4-7 (non-rotary q)
    Wqr = np.ones((4, 3))         # heads 0, 1: rows 0-1 / 2-3 (rotary q)
    Wk = np.ones((8, 3))          # non-rotary k
    Wkr = np.ones((2, 3))         # shared rotary k: not in any slice
    slices = [(0, 0, 4, 0, 0.5), (0, 4, 4, 1, 0.5), (1, 0, 2, 0, 1.0), (1, 2, 2, 1, 1.0),
              (2, 0, 4, 0, 0.5), (2, 4, 4, 1, 0.5)]
    q, qr, k, kr = orc.qk_clip([Wq, Wqr, Wk, Wkr], slices, s_max=[400.0, 50.0], tau=100.0)
    assert np.array_equal(q[:4], np.full((4, 3), 0.5)) and np.array_equal(q[4:], np.ones((4, 3)))
    assert np.array_equal(qr[:2], np.full((2, 3), 0.25)) and np.array_equal(qr[2:], np.ones((2, 3)))
    assert np.array_equal(k[:4], np.full((4, 3), 0.5)) and np.array_equal(k[4:], np.ones((4, 3)))
    assert np.array_equal(kr, Wkr)
    # after clipping, the head's largest logit q.k scales by gamma^(0.5+0.5) = tau/S_max
    assert (0.5 * 0.5) * 400.0 == 100.0


def test_two_sided_normalisation_rank_one_is_the_sign_pattern():
    """N(u v^T) = sign(u) sign(v)^T: the row and column factors of a rank-one matrix
    cancel exactly (eps = 0)."""
    u = np.array([0.5, -2.0, 3.0, -0.25])
    v = np.array([1.0, -1e-3, 7.0])
    got = orc.two_sided_normalise(np.outer(u, v), eps=0.0)
    assert np.allclose(got, np.outer(np.sign(u), np.sign(v)), rtol=1e-13, atol=0)
    # scale invariance of the whole step direction: normalisation removes any factor
    hp = orc.HParams(mode="twosided", scale="none", lr=1.0)
    W = np.zeros((4, 3))
    r1 = orc.muon_step(W, np.outer(u, v), np.zeros((4, 3)), hp)
    r2 = orc.muon_step(W, 1e3 * np.outer(u, v), np.zeros((4, 3)), hp)
    assert np.allclose(r1.O, r2.O, rtol=1e-5, atol=1e-9)
    # with eps = 1e-7 the small column (RMS ~7e-5 after normalisation) moves by ~0.14 %
    assert np.allclose(r1.O, np.outer(np.sign(u), np.sign(v)), rtol=2e-3, atol=0)


def test_two_sided_normalisation_of_a_scaled_sign_matrix_is_the_sign_matrix():
    """N(D_r Z D_c) = Z for any +-1 matrix Z (full rank in general) and positive row and
    column scalings D_r, D_c (eps = 0): the row mean square of X is d_ri^2 mean(d_c^2), the
    column one d_cj^2 mean(d_r^2), and the RMS sqrt(mean(d_r^2) mean(d_c^2)), so every
    factor cancels. The rank-one case is Z = sign(u) sign(v)^T."""
    rng = np.random.default_rng(21)
    for rows, cols in ((5, 7), (16, 3), (1, 9), (12, 12)):
        Z = rng.choice([-1.0, 1.0], size=(rows, cols))
        dr = np.exp(rng.normal(0.0, 1.5, rows))
        dc = np.exp(rng.normal(0.0, 1.5, cols))
        X = dr[:, None] * Z * dc[None, :]
        got = orc.two_sided_normalise(X, eps=0.0)
        assert np.allclose(got, Z, rtol=1e-12, atol=0), (rows, cols)
        if rows > 1 and cols > 1:
            assert np.linalg.matrix_rank(Z) > 1 or rows * cols <= 4


def test_equilibration_of_line_scaled_sign_matrices():
    """O = D_r Z (Z of +-1 entries, D_r positive and not constant): every column has the
    same RMS, sqrt(mean(d^2)), while the rows do not, so rows are chosen and
    O_ij <- d_i z_ij rho / d_i = rho z_ij with rho = RMS(O) (eps = 0). The column-scaled
    O = Z D_c maps to rho Z through the columns. ||O||_F is kept in both cases."""
    rng = np.random.default_rng(22)
    for rows, cols in ((6, 9), (9, 6), (10, 10)):
        Z = rng.choice([-1.0, 1.0], size=(rows, cols))
        d = np.exp(rng.normal(0.0, 1.0, max(rows, cols)))
        for O, axis in ((d[:rows, None] * Z, orc.AXIS_ROWS), (Z * d[None, :cols], orc.AXIS_COLS)):
            rho = np.sqrt(np.mean(O * O))
            got, ax = orc.equilibrate(O, eps=0.0)
            assert ax == axis, (rows, cols, axis)
            assert np.allclose(got, rho * Z, rtol=1e-12, atol=0)
            assert np.linalg.norm(got) == pytest.approx(np.linalg.norm(O), rel=1e-12)
