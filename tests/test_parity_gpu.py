"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle.

Tolerances (relative Frobenius error per matrix): 1e-4 for the fp32 Newton-Schulz
path, 3e-2 for the bf16 tensor-core path; checked on W_t, M_t and dW_t.
"""
import numpy as np
import pytest

from oracle import muon_oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(lib):
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    return B, torch


# ------------------------------------------------------------------ Newton-Schulz only
def _ns_gpu(B, torch, xs, hp, dtype):
    X = [torch.tensor(x, dtype=torch.float32, device="cuda").to(dtype) for x in xs]
    O = [torch.empty_like(x) for x in X]
    ws = B.newton_schulz(X, O, hp)
    torch.cuda.synchronize()
    assert B.load().muon_query_device_status(ws.data_ptr(), None) == 0
    return [o.double().cpu().numpy() for o in O]


SMALL = [(1, 1), (1, 40), (40, 1), (17, 33), (33, 17), (64, 64), (128, 256), (256, 128),
         (129, 130), (200, 700), (700, 200), (320, 512), (512, 320),
         # m a multiple of 256: the CTA-pair kernel (ragged n included)
         (256, 256), (512, 700), (768, 1000), (1000, 768)]


@pytest.mark.parametrize("coeffs,tol", [((1.0, 0.0, 0.0), 1e-2), ((0.0, 1.0, 0.0), 1e-2),
                                        ((0.0, 0.0, 1.0), 2e-2)])
def test_tensor_core_phases_isolated(env, coeffs, tol):
    """One iteration with (a,b,c) = e1, e2, e3 isolates a*X (APPLY epilogue), S X (GRAM
    then APPLY) and S^2 X (GRAM, POLY, APPLY): each against the literal recurrence."""
    B, torch = env
    shapes = [(17, 33), (128, 256), (129, 130), (320, 512), (512, 320), (200, 700),
              (256, 300), (512, 512), (768, 1000)]
    xs = [H.seeded_bf16(r, c, 10 + i, 1.0) for i, (r, c) in enumerate(shapes)]
    hp = B.hparams(ns_coeffs=coeffs, ns_steps=1)
    got = _ns_gpu(B, torch, xs, hp, torch.bfloat16)
    for x, g in zip(xs, got):
        want = orc.orthogonalise(x.astype(np.float64), orc.HParams(ns_coeffs=coeffs, ns_steps=1))
        assert H.rel(g, want) <= tol, (x.shape, H.rel(g, want))


@pytest.mark.parametrize("fp32", [True, False])
def test_newton_schulz_small_shapes(env, fp32):
    B, torch = env
    xs = [H.seeded(r, c, 100 + i, 1e-3) for i, (r, c) in enumerate(SMALL)]
    if not fp32:
        xs = [H.seeded_bf16(r, c, 100 + i, 1e-3) for i, (r, c) in enumerate(SMALL)]
    hp = B.hparams(ns_fp32=fp32)
    got = _ns_gpu(B, torch, xs, hp, torch.float32 if fp32 else torch.bfloat16)
    tol = H.TOL_FP32 if fp32 else H.TOL_BF16
    for x, g in zip(xs, got):
        want = orc.orthogonalise(x.astype(np.float64), orc.HParams())
        # a bf16 output adds its own rounding (2^-9 relative) on top of the path's error
        assert H.rel(g, want) <= tol, (x.shape, H.rel(g, want))


def test_newton_schulz_zero_steps_and_zero_input(env):
    B, torch = env
    xs = [H.seeded(48, 80, 7, 1.0), np.zeros((16, 24), np.float32)]
    got = _ns_gpu(B, torch, xs, B.hparams(ns_steps=0, ns_fp32=True), torch.float32)
    assert H.rel(got[0], orc.frobenius_normalise(xs[0].astype(np.float64))) <= 1e-6
    assert not np.any(got[1])
    got = _ns_gpu(B, torch, [xs[1]], B.hparams(), torch.bfloat16)
    assert not np.any(got[0])


# ------------------------------------------------------------------ whole step
@pytest.mark.parametrize("mode", ["muon", "muongs"])
def test_single_128x256_fp32_ten_steps(env, mode):
    """The single-matrix case: W 128x256 ~ N(0, 0.02^2), grads N(0, 1e-3^2) fp32, zero
    momentum, lr 0.02, wd 0.1, 0.2*sqrt(256) scale, 10 steps, fp32 path, 1e-4."""
    B, torch = env
    from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
    w = wl.WORKLOADS["single_128x256"]
    spec = w.matrices()[0]
    W0 = [wl.weight(w, spec)]
    grads = [[wl.grad(w, spec, t)] for t in range(10)]
    hp = H.gpu_hp(B, mode=mode, wd=0.1, ns_fp32=True)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.float32)
    worst = H.compare_runs(gpu, W0, grads, H.oracle_hp(mode=mode, wd=0.1), H.TOL_FP32)
    print(f"\nSINGLE {mode}: max rel err over 10 steps W {worst['W']:.2e} M {worst['M']:.2e} "
          f"dW {worst['dW']:.2e}")
    assert worst["dW"] <= H.TOL_FP32


STEP_SHAPES = [(17, 33), (33, 17), (128, 256), (256, 128), (200, 700), (320, 512), (512, 320),
               (384, 384), (512, 700), (768, 512)]


@pytest.mark.parametrize("mode,wd,eq", [("muongs", 0.0, False), ("muon", 0.1, False),
                                        ("muon", 0.1, True), ("muongs", 0.1, True),
                                        ("muonh", 0.0, False), ("muonh", 0.1, True)])
def test_bf16_step_mixed_shapes_ten_steps(env, mode, wd, eq):
    B, torch = env
    W0 = [H.seeded(r, c, 300 + i, 0.02) for i, (r, c) in enumerate(STEP_SHAPES)]
    grads = [[H.seeded_bf16(r, c, 1000 * (t + 1) + i, 1e-3) for i, (r, c) in enumerate(STEP_SHAPES)]
             for t in range(10)]
    hp = H.gpu_hp(B, mode=mode, wd=wd, equilibrate=eq)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.bfloat16)
    ohp = H.oracle_hp(mode=mode, wd=wd, equilibrate=eq)
    if eq:
        H.compare_runs_equilibrated(gpu, W0, grads, ohp, H.TOL_BF16)
    else:
        H.compare_runs(gpu, W0, grads, ohp, H.TOL_BF16)


# wide, tall, square and near-square shapes; ragged edges included
EQ_SHAPES = [(128, 384), (384, 128), (256, 256), (320, 336), (336, 320), (200, 700),
             (700, 200), (512, 512), (257, 255)]


@pytest.mark.parametrize("line_scale", ["rows", "cols", "none"])
def test_equilibration_axis_matches_oracle_ten_steps(env, line_scale):
    """The equilibration axis (section 핵심 내용 of the MeqMuon page: row or column
    normalisation picked per matrix) against the oracle's choice over 10 steps, with
    gradients whose rows (as in the 1.5B dense set) or columns carry log-normal scales.
    Where the oracle's two imbalances are clearly apart the GPU must pick the same
    axis; on a tie the oracle follows the GPU's axis and the result must match."""
    B, torch = env
    rng = np.random.default_rng(77)
    scales = [np.exp(rng.standard_normal(r if line_scale == "rows" else c))
              for (r, c) in EQ_SHAPES]
    W0 = [H.seeded(r, c, 1300 + i, 0.02) for i, (r, c) in enumerate(EQ_SHAPES)]

    def grad(i, t):
        r, c = EQ_SHAPES[i]
        g = H.seeded(r, c, 1400 + 16 * t + i, 1e-3).astype(np.float64)
        if line_scale == "rows":
            g = g * scales[i][:, None]
        elif line_scale == "cols":
            g = g * scales[i][None, :]
        from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
        return wl.bf16_round(g.astype(np.float32))

    grads = [[grad(i, t) for i in range(len(EQ_SHAPES))] for t in range(10)]
    hp = H.gpu_hp(B, mode="muon", wd=0.1, equilibrate=True)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.bfloat16)
    worst = H.compare_runs_equilibrated(gpu, W0, grads,
                                        H.oracle_hp(mode="muon", wd=0.1, equilibrate=True),
                                        H.TOL_BF16)
    print(f"\nEQ-AXIS {line_scale}: decided {worst['decided']} tied {worst['tied']}; max rel "
          f"err W {worst['W']:.2e} M {worst['M']:.2e} dW {worst['dW']:.2e}")
    assert worst["decided"] > 0


def test_fp32_step_mixed_shapes_one_shot_api(env):
    """muon_step_batched (no plan) with fp32 grads and the fp32 Newton-Schulz path."""
    B, torch = env
    shapes = [(5, 9), (64, 48), (100, 300)]
    W0 = [H.seeded(r, c, 50 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded(r, c, 60 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(3)]
    hp = H.gpu_hp(B, mode="muongs", wd=0.05, ns_fp32=True)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.float32, use_plan=False)
    H.compare_runs(gpu, W0, grads, H.oracle_hp(mode="muongs", wd=0.05), H.TOL_FP32)


@pytest.mark.parametrize("eq", [False, True])
def test_fp32_muon_step_statistics_from_post_apply(env, eq):
    """Muon on the fp32 Newton-Schulz path: with equilibration the reduction reads the
    fp32 slab alone (its row and column sums in the slab's frame, tall matrices
    included); without it no reduction runs and every statistic comes from post_apply.
    4 steps against the oracle at the fp32 tolerance."""
    B, torch = env
    shapes = [(5, 9), (64, 48), (100, 300), (300, 100), (257, 255)]
    W0 = [H.seeded(r, c, 70 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded(r, c, 80 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(4)]
    hp = H.gpu_hp(B, mode="muon", wd=0.1, ns_fp32=True, equilibrate=eq)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.float32)
    ohp = H.oracle_hp(mode="muon", wd=0.1, equilibrate=eq)
    if eq:
        H.compare_runs_equilibrated(gpu, W0, grads, ohp, H.TOL_FP32)
    else:
        H.compare_runs(gpu, W0, grads, ohp, H.TOL_FP32)


def test_muongs_invariants_on_gpu(env):
    """<W_t, O~> = 0 and ||W_{t+1}||^2 = ||W_t||^2 + lr^2 ||O~||^2 (wd = 0), at fp32 level."""
    B, torch = env
    W0 = [H.seeded(96, 160, 5, 0.02)]
    grads = [[H.seeded_bf16(96, 160, 70 + t, 1e-3)] for t in range(3)]
    gpu = H.run_steps(B, torch, W0, grads, H.gpu_hp(B, mode="muongs"), torch.bfloat16)
    W_prev = W0[0].astype(np.float64)
    for t in range(3):
        W = gpu[t][0][0]
        O_t = (W_prev - W) / 0.02
        assert abs(np.sum(W_prev * O_t)) <= 1e-4 * np.linalg.norm(W_prev) * np.linalg.norm(O_t)
        lhs, rhs = np.sum(W * W), np.sum(W_prev * W_prev) + 0.02 ** 2 * np.sum(O_t * O_t)
        assert abs(lhs - rhs) <= 1e-5 * rhs
        W_prev = W


def test_degenerate_step_inputs(env):
    """Zero gradient from zero momentum: only the decay acts. Zero weight in MuonGS
    mode: the projection is skipped. A 1x1 matrix."""
    B, torch = env
    W0 = [np.ones((8, 24), np.float32), np.zeros((16, 16), np.float32), np.full((1, 1), 0.5, np.float32)]
    grads = [[np.zeros((8, 24), np.float32), H.seeded_bf16(16, 16, 9, 1e-3),
              np.full((1, 1), -1e-3, np.float32)]]
    hp = H.gpu_hp(B, mode="muongs", wd=0.1)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.bfloat16)
    assert np.allclose(gpu[0][0][0], (1 - 0.02 * 0.1) * W0[0], rtol=0, atol=1e-7)
    H.compare_runs(gpu, W0, grads, H.oracle_hp(mode="muongs", wd=0.1), H.TOL_BF16)


def test_muonh_keeps_the_radius_on_gpu(env):
    """MuonH: ||W_t|| stays ||W_0|| step after step (fp32 level)."""
    B, torch = env
    shapes = [(96, 160), (768, 512)]
    W0 = [H.seeded(r, c, 40 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded_bf16(r, c, 80 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(4)]
    gpu = H.run_steps(B, torch, W0, grads, H.gpu_hp(B, mode="muonh", wd=0.1), torch.bfloat16)
    for i, w in enumerate(W0):
        R = np.linalg.norm(w.astype(np.float64))
        for t in range(4):
            assert abs(np.linalg.norm(gpu[t][0][i]) - R) <= 2e-6 * R


def test_two_sided_mode_ten_steps(env):
    """Two-sided normalisation (no Newton-Schulz, fp32 throughout): 1e-4 against the
    oracle over 10 steps, scale none, Adam-like learning rate."""
    B, torch = env
    shapes = [(17, 33), (128, 256), (300, 64), (512, 320)]
    W0 = [H.seeded(r, c, 500 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded_bf16(r, c, 600 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(10)]
    hp = B.hparams(lr=1e-3, weight_decay=0.01, mode="twosided", scale="none")
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.bfloat16)
    ohp = H.oracle_hp(mode="twosided", wd=0.01, lr=1e-3, scale="none")
    H.compare_runs(gpu, W0, grads, ohp, H.TOL_FP32, check_stats=False)
    for t in range(10):
        assert all(st["equil_axis"] == 3 for st in gpu[t][2])
        for i in range(len(shapes)):   # ||W_t|| of the GPU's own W_t (gathered by post_apply)
            wn = np.linalg.norm(W0[i].astype(np.float64) if t == 0 else gpu[t - 1][0][i])
            assert abs(gpu[t][2][i]["w_norm"] - wn) <= 1e-5 * wn


def test_strided_unaligned_views_ten_steps(env):
    """W, G and M as column slices of wider buffers at odd offsets: ld > cols, rows not
    16-byte aligned, so the elementwise kernels take their scalar paths. Parity against
    the oracle over 10 steps, and nothing outside the views is written."""
    B, torch = env
    cases = [((200, 300), 333, 1), ((300, 130), 141, 3), ((256, 300), 301, 1),
             ((300, 256), 259, 2), ((33, 17), 40, 5)]
    W0 = [H.seeded(r, c, 1100 + i, 0.02) for i, ((r, c), _, _) in enumerate(cases)]
    grads = [[H.seeded_bf16(r, c, 1200 + 10 * t + i, 1e-3) for i, ((r, c), _, _) in enumerate(cases)]
             for t in range(10)]
    bufs_w, bufs_m, bufs_g, Ws, Ms, Gs = [], [], [], [], [], []
    for i, ((r, c), ld, off) in enumerate(cases):
        bw = torch.full((r, ld), 7.0, dtype=torch.float32, device="cuda")
        bm = torch.full((r, ld), -3.0, dtype=torch.float32, device="cuda")
        bg = torch.zeros((r, ld + 2), dtype=torch.bfloat16, device="cuda")
        w = bw[:, off:off + c]
        w.copy_(torch.from_numpy(W0[i]))
        m = bm[:, off:off + c]
        m.zero_()
        bufs_w.append(bw), bufs_m.append(bm), bufs_g.append(bg)
        Ws.append(w), Ms.append(m), Gs.append(bg[:, off + 1:off + 1 + c])
    hp = H.gpu_hp(B, mode="muongs", wd=0.1)
    plan = B.Plan(Ws, Gs, Ms, hp)
    stats = B.new_stats(len(Ws))
    gpu = []
    for gl in grads:
        for g_dev, g in zip(Gs, gl):
            g_dev.copy_(torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)))
        plan.step(stats=stats)
        torch.cuda.synchronize()
        gpu.append(([w.double().cpu().numpy() for w in Ws], [m.double().cpu().numpy() for m in Ms],
                    B.decode_stats(stats)))
    assert plan.query_device_status() == 0
    plan.close()
    H.compare_runs(gpu, W0, grads, H.oracle_hp(mode="muongs", wd=0.1), H.TOL_BF16)
    for i, ((r, c), ld, off) in enumerate(cases):
        for buf, fill in ((bufs_w[i], 7.0), (bufs_m[i], -3.0)):
            outside = torch.cat([buf[:, :off], buf[:, off + c:]], dim=1)
            assert bool((outside == fill).all()), (i, fill)


@pytest.mark.parametrize("g_fp32,scale,nesterov,ns_steps", [(True, "keller", False, 5),
                                                            (False, "none", True, 3),
                                                            (True, "moonlight", True, 5)])
def test_bf16_path_option_combinations(env, g_fp32, scale, nesterov, ns_steps):
    """The bf16 tensor-core path with fp32 gradients, the Keller / no scale rules, plain
    momentum (U = M) and a non-default iteration count, against the oracle over 4 steps."""
    B, torch = env
    shapes = [(96, 160), (256, 384), (384, 256), (70, 70)]
    W0 = [H.seeded(r, c, 1300 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    gen = H.seeded if g_fp32 else H.seeded_bf16
    grads = [[gen(r, c, 1400 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(4)]
    hp = H.gpu_hp(B, mode="muongs", wd=0.05, scale=scale, nesterov=nesterov, ns_steps=ns_steps)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.float32 if g_fp32 else torch.bfloat16)
    ohp = H.oracle_hp(mode="muongs", wd=0.05, scale=scale, nesterov=nesterov, ns_steps=ns_steps)
    H.compare_runs(gpu, W0, grads, ohp, H.TOL_BF16)


def test_plan_hparams_change_between_steps(env):
    """muon_plan_set_hparams between steps: two Muon steps at lr 0.02, then two MuonGS
    steps at lr 0.01 with decay and 4 Newton-Schulz iterations (the result moves to the
    other slab), on the same plan, momenta carried over. W_t and dW_t per step."""
    B, torch = env
    shapes = [(128, 256), (512, 256)]
    W0 = [H.seeded(r, c, 1500 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded_bf16(r, c, 1600 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(4)]
    Ws = [torch.tensor(w, device="cuda") for w in W0]
    Ms = [torch.zeros_like(w) for w in Ws]
    Gs = [torch.empty(w.shape, dtype=torch.bfloat16, device="cuda") for w in Ws]
    plan = B.Plan(Ws, Gs, Ms, H.gpu_hp(B, mode="muon", lr=0.02))
    W_orc = [w.astype(np.float64) for w in W0]
    M_orc = [np.zeros_like(w) for w in W_orc]
    for t in range(4):
        if t == 2:
            plan.set_hparams(H.gpu_hp(B, mode="muongs", lr=0.01, wd=0.1, ns_steps=4))
        ohp = (H.oracle_hp(mode="muon", lr=0.02) if t < 2
               else H.oracle_hp(mode="muongs", lr=0.01, wd=0.1, ns_steps=4))
        W_prev_gpu = [w.double().cpu().numpy() for w in Ws]
        W_prev_orc = [w.copy() for w in W_orc]
        for g_dev, g in zip(Gs, grads[t]):
            g_dev.copy_(torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)))
        plan.step()
        torch.cuda.synchronize()
        for i in range(len(shapes)):
            r = orc.muon_step(W_orc[i], grads[t][i].astype(np.float64), M_orc[i], ohp)
            W_orc[i], M_orc[i] = r.W, r.M
            Wg = Ws[i].double().cpu().numpy()
            assert H.rel(Wg, W_orc[i]) <= H.TOL_BF16, (t, i)
            assert H.rel(W_prev_gpu[i] - Wg, W_prev_orc[i] - W_orc[i]) <= H.TOL_BF16, (t, i)
    assert plan.query_device_status() == 0
    plan.close()


def test_plan_learning_rate_schedule_updates_the_graph(env):
    """A new learning rate and decay before every step (muon_plan_set_hparams with the
    same launch sequence): from the third step on the captured graph is updated in place
    instead of re-instantiated. Every step against the oracle with that step's lr."""
    B, torch = env
    shapes = [(128, 256), (768, 512), (320, 512)]
    W0 = [H.seeded(r, c, 1700 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded_bf16(r, c, 1800 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(6)]
    lrs = [0.02, 0.015, 0.01, 0.03, 0.005, 0.02]
    wds = [0.0, 0.1, 0.0, 0.05, 0.1, 0.0]
    Ws = [torch.tensor(w, device="cuda") for w in W0]
    Ms = [torch.zeros_like(w) for w in Ws]
    Gs = [torch.empty(w.shape, dtype=torch.bfloat16, device="cuda") for w in Ws]
    plan = B.Plan(Ws, Gs, Ms, H.gpu_hp(B, mode="muongs", lr=lrs[0]))
    W_orc = [w.astype(np.float64) for w in W0]
    M_orc = [np.zeros_like(w) for w in W_orc]
    for t in range(6):
        plan.set_hparams(H.gpu_hp(B, mode="muongs", lr=lrs[t], wd=wds[t]))
        ohp = H.oracle_hp(mode="muongs", lr=lrs[t], wd=wds[t])
        W_prev_gpu = [w.double().cpu().numpy() for w in Ws]
        W_prev_orc = [w.copy() for w in W_orc]
        for g_dev, g in zip(Gs, grads[t]):
            g_dev.copy_(torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)))
        plan.step()
        torch.cuda.synchronize()
        for i in range(len(shapes)):
            r = orc.muon_step(W_orc[i], grads[t][i].astype(np.float64), M_orc[i], ohp)
            W_orc[i], M_orc[i] = r.W, r.M
            Wg = Ws[i].double().cpu().numpy()
            assert H.rel(Wg, W_orc[i]) <= H.TOL_BF16, (t, i)
            assert H.rel(W_prev_gpu[i] - Wg, W_prev_orc[i] - W_orc[i]) <= H.TOL_BF16, (t, i)
    assert plan.query_device_status() == 0
    plan.close()


def test_plan_graph_replay_matches_eager_steps(env):
    """A cached plan runs its first step eagerly, captures the second into a CUDA graph
    and replays it afterwards (re-capturing when the stats pointer changes). Four plan
    steps must equal four one-shot muon_step_batched calls (never graphed) up to the
    order of the atomic sums."""
    B, torch = env
    shapes = [(128, 256), (300, 130), (256, 256)]
    W0 = [H.seeded(r, c, 1700 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded_bf16(r, c, 1800 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(4)]
    hp = H.gpu_hp(B, mode="muongs", wd=0.05)
    runs = []
    for use_plan in (True, False):
        Ws = [torch.tensor(w, device="cuda") for w in W0]
        Ms = [torch.zeros_like(w) for w in Ws]
        Gs = [torch.empty(w.shape, dtype=torch.bfloat16, device="cuda") for w in Ws]
        stats = B.new_stats(len(Ws))
        plan = B.Plan(Ws, Gs, Ms, hp) if use_plan else None
        for t in range(4):
            for g_dev, g in zip(Gs, grads[t]):
                g_dev.copy_(torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)))
            st = stats if t != 2 else None          # step 3 has no stats: a new graph
            if use_plan:
                plan.step(stats=st)
            else:
                B.step_batched(Ws, Gs, Ms, hp, stats=st)
        torch.cuda.synchronize()
        if plan is not None:
            assert plan.query_device_status() == 0
            plan.close()
        runs.append(([w.double().cpu().numpy() for w in Ws], [m.double().cpu().numpy() for m in Ms],
                     B.decode_stats(stats)))
    for i in range(len(shapes)):
        assert H.rel(runs[0][0][i], runs[1][0][i]) <= 1e-5, i
        assert H.rel(runs[0][1][i], runs[1][1][i]) <= 1e-6, i
        for key in ("w_norm", "o_norm"):
            assert abs(runs[0][2][i][key] - runs[1][2][i][key]) <= 1e-5 * abs(runs[1][2][i][key]) + 1e-9


def test_fp32_fused_and_per_phase_classes_in_one_plan(env):
    """The fp32 path with six shape classes in one plan (classes are keyed by the oriented
    (m, n), so 64x200 and 200x64 share one): five small ones (n <= 256) run all iterations
    in the fused cluster kernel, in two launches of at most four classes; the 300x520 class
    takes one launch per phase. 10 steps, 1e-4 against the oracle."""
    B, torch = env
    shapes = [(9, 13), (64, 200), (256, 100), (128, 256), (200, 64), (300, 520), (520, 300),
              (1, 256)]
    W0 = [H.seeded(r, c, 1900 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded(r, c, 2000 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(10)]
    hp = H.gpu_hp(B, mode="muongs", wd=0.1, ns_fp32=True)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.float32)
    worst = H.compare_runs(gpu, W0, grads, H.oracle_hp(mode="muongs", wd=0.1), H.TOL_FP32)
    print(f"\nFP32 MIXED: max rel err W {worst['W']:.2e} M {worst['M']:.2e} dW {worst['dW']:.2e}")


@pytest.mark.parametrize("m", [64, 130, 192, 320, 448, 500, 640])
def test_single_cta_variable_width_tiles_ragged_m(env, m):
    """Single-CTA classes (m not a multiple of 256) cut every 128-row block of S and P'
    into variable-width column pieces; m values whose row blocks end ragged, whose pieces
    are 64, 128, 192 or 256 wide, and whose B units switch from K-major to mirrored inside
    a piece. 16 matrices per class (the piece order rotates per matrix), 3 steps."""
    B, torch = env
    shapes = [(m, m + 192)] * 8 + [(m + 320, m)] * 8
    W0 = [H.seeded(r, c, 2100 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded_bf16(r, c, 2200 + 20 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(3)]
    gpu = H.run_steps(B, torch, W0, grads, H.gpu_hp(B, mode="muongs"), torch.bfloat16)
    H.compare_runs(gpu, W0, grads, H.oracle_hp(mode="muongs"), H.TOL_BF16)


@pytest.mark.parametrize("mode,cols_tail,ns_steps,eq", [
    ("muongs", 8, 5, False), ("muongs", 4, 5, False), ("muongs", 3, 5, False),
    ("muongs", 8, 0, False), ("muongs", 8, 5, True), ("muongs", 8, 0, True),
    ("muon", 8, 5, False), ("muon", 8, 5, True), ("muon", 3, 5, True), ("muon", 8, 0, True)])
def test_large_ragged_step_staged_kernels(env, mode, cols_tail, ns_steps, eq):
    """A step above 4M elements. MuonGS needs <W,O>, ||W||^2 and ||O||^2 before the
    update; Muon needs no sum of W, so its reduction reads the slab alone (only with
    equilibration: ||O||^2 and the O^2 row / column sums, in the slab's frame) and
    post_apply gathers the statistics' sums of W. Every width a multiple of 8
    (cols_tail 8): ingest, the reduction and post_apply all stage their loads in shared
    memory; a width that is a multiple of 4 only (cols_tail 4, bf16 gradient rows not
    16-byte multiples): ingest keeps its register-staged kernel; an odd width
    (cols_tail 3): all three do. With equilibration the reduction also takes the per-row
    and per-column sums; with no Newton-Schulz iteration the slab holds U and every kernel
    applies 1/(||U||+eps) itself. The tiles end ragged in rows and columns, include a
    tall (transposed) matrix, and two matrices smaller than one 32 x 64 sub-tile. 2 steps
    against the oracle."""
    B, torch = env
    shapes = [(1000, 2048 + cols_tail), (2056, 1000), (516, 1288), (17, 24), (40, 8)]
    W0 = [H.seeded(r, c, 2300 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[H.seeded_bf16(r, c, 2400 + 10 * t + i, 1e-3) for i, (r, c) in enumerate(shapes)]
             for t in range(2)]
    hp = H.gpu_hp(B, mode=mode, wd=0.1, ns_steps=ns_steps, equilibrate=eq)
    gpu = H.run_steps(B, torch, W0, grads, hp, torch.bfloat16)
    ohp = H.oracle_hp(mode=mode, wd=0.1, ns_steps=ns_steps, equilibrate=eq)
    if eq:
        H.compare_runs_equilibrated(gpu, W0, grads, ohp, H.TOL_BF16)
    else:
        H.compare_runs(gpu, W0, grads, ohp, H.TOL_BF16)
