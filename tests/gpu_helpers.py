"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and
the float64 oracle on the same seeded inputs, and compare them."""
from __future__ import annotations

import numpy as np

from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
from oracle import muon_oracle as orc

TOL_FP32 = 1e-4   # relative Frobenius error, fp32 Newton-Schulz path
TOL_BF16 = 3e-2   # relative Frobenius error, bf16 tensor-core path


def rel(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))


def oracle_hp(mode="muon", wd=0.0, equilibrate=False, lr=0.02, ns_steps=5, coeffs=orc.QUINTIC,
              scale="moonlight", nesterov=True):
    return orc.HParams(lr=lr, momentum=0.95, weight_decay=wd, nesterov=nesterov, ns_coeffs=coeffs,
                       ns_steps=ns_steps, mode=mode, scale=scale, equilibrate=equilibrate)


def gpu_hp(B, mode="muon", wd=0.0, equilibrate=False, lr=0.02, ns_steps=5, coeffs=orc.QUINTIC,
           scale="moonlight", nesterov=True, ns_fp32=False):
    return B.hparams(lr=lr, momentum=0.95, weight_decay=wd, ns_coeffs=coeffs, ns_steps=ns_steps,
                     mode=mode, scale=scale, nesterov=nesterov, equilibrate=equilibrate,
                     ns_fp32=ns_fp32)


def run_steps(B, torch, W0s, grads_per_step, hp, g_dtype, use_plan=True):
    """Runs len(grads_per_step) steps on the GPU. Returns per step the lists of
    W, M (numpy float64) and the decoded stats."""
    dev = "cuda"
    Ws = [torch.tensor(w, dtype=torch.float32, device=dev) for w in W0s]
    Ms = [torch.zeros_like(w) for w in Ws]
    Gs = [torch.empty(w.shape, dtype=g_dtype, device=dev) for w in Ws]
    stats = B.new_stats(len(Ws))
    plan = B.Plan(Ws, Gs, Ms, hp) if use_plan else None
    out = []
    for gl in grads_per_step:
        for g_dev, g in zip(Gs, gl):
            g_dev.copy_(torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)))
        if use_plan:
            plan.step(stats=stats)
        else:
            B.step_batched(Ws, Gs, Ms, hp, stats=stats)
        torch.cuda.synchronize()
        out.append(([w.double().cpu().numpy() for w in Ws], [m.double().cpu().numpy() for m in Ms],
                    B.decode_stats(stats)))
    if plan is not None:
        assert plan.query_device_status() == 0
        plan.close()
    return out


def check_muon_stats_against_own_update(W_prev_gpu, Wg, st, ohp):
    """Muon mode has no projection, so the step applied O = ((1 - lr wd) W_t - W_{t+1}) / lr
    (float64 from the GPU's own fp32 W_t and W_{t+1}: about 1e-6 relative). The
    statistics <W_t, O> and ||O|| must describe that O; this pins the sums post_apply
    gathers for them, the scale included, far tighter than the oracle comparison can."""
    if ohp.mode != "muon":
        return
    O = ((1.0 - ohp.lr * ohp.weight_decay) * W_prev_gpu - Wg) / ohp.lr
    on, wn = np.linalg.norm(O), np.linalg.norm(W_prev_gpu)
    assert abs(st["o_norm"] - on) <= 1e-4 * on + 1e-9, (st["o_norm"], on)
    wo = float(np.sum(W_prev_gpu * O))
    assert abs(st["w_dot_o"] - wo) <= 1e-4 * wn * on + 1e-9, (st["w_dot_o"], wo, wn * on)


def compare_runs(gpu, W0s, grads_per_step, ohp, tol, check_stats=True):
    """Per matrix and per step: relative error of W_t, M_t and dW_t against the oracle."""
    worst = {"W": 0.0, "M": 0.0, "dW": 0.0}
    for i, W0 in enumerate(W0s):
        res = orc.muon_run(W0, [g[i] for g in grads_per_step], ohp)
        W_prev_gpu, W_prev_orc = np.asarray(W0, np.float64), np.asarray(W0, np.float64)
        for t, r in enumerate(res):
            Wg, Mg, st = gpu[t][0][i], gpu[t][1][i], gpu[t][2][i]
            eW, eM = rel(Wg, r.W), rel(Mg, r.M)
            edW = rel(W_prev_gpu - Wg, W_prev_orc - r.W)
            worst["W"] = max(worst["W"], eW)
            worst["M"] = max(worst["M"], eM)
            worst["dW"] = max(worst["dW"], edW)
            assert eW <= tol and eM <= tol and edW <= tol, (i, t, eW, eM, edW)
            if check_stats:
                wn = np.linalg.norm(W_prev_gpu)     # the stat describes the GPU's own W_t
                assert abs(st["w_norm"] - wn) <= 1e-5 * wn + 1e-12
                assert abs(st["o_norm"] - r.o_norm) <= 2 * tol * r.o_norm + 1e-6
                assert abs(st["update_rms"] - r.update_rms) <= 2 * tol * r.update_rms + 1e-6
                check_muon_stats_against_own_update(W_prev_gpu, Wg, st, ohp)
            W_prev_gpu, W_prev_orc = Wg, r.W
    return worst


# Equilibration picks the axis whose line-RMS imbalance is larger. The GPU takes that
# decision on its bf16-path O, which differs from the oracle's by about 1e-2 relative,
# so the two imbalances it compares move by up to about that much. Where the oracle's
# imbalances differ by more than this margin the axis is unique and must match; below
# it both results are valid, and the oracle is run with the GPU's axis (its result must
# then match within the path's tolerance).
EQ_AXIS_MARGIN_REL = 0.10
EQ_AXIS_MARGIN_ABS = 0.01


def axis_decided(ir: float, ic: float) -> bool:
    return abs(ir - ic) > EQ_AXIS_MARGIN_REL * max(ir, ic) + EQ_AXIS_MARGIN_ABS


def check_step(W, M, G, Wg, Mg, W_prev_gpu, st, ohp, tol, worst):
    """One oracle step of one matrix from the oracle's state (W, M) with gradient G,
    compared with the GPU's W_{t+1} (Wg), M_t (Mg) and dW_t = W_prev_gpu - Wg. With
    equilibration the axis is checked as described above (axis_decided) and the oracle
    follows the GPU's axis on a tie. Updates `worst`; returns the oracle's (W, M)."""
    import dataclasses
    if ohp.equilibrate:
        assert st["equil_axis"] in (orc.AXIS_ROWS, orc.AXIS_COLS)
        # the oracle's step with the GPU's axis; its pre-equilibration imbalances decide
        # whether that axis was the only correct one
        r = orc.muon_step(W, G, M, dataclasses.replace(ohp, equil_axis=st["equil_axis"]))
        ir, ic = r.imbalances
        natural = orc.AXIS_ROWS if ir >= ic else orc.AXIS_COLS
        if axis_decided(ir, ic):
            assert st["equil_axis"] == natural, (ir, ic, st["equil_axis"])
            worst["decided"] = worst.get("decided", 0) + 1
        else:
            worst["tied"] = worst.get("tied", 0) + 1
    else:
        r = orc.muon_step(W, G, M, ohp)
    eW, eM = rel(Wg, r.W), rel(Mg, r.M)
    edW = rel(W_prev_gpu - Wg, W - r.W)
    assert eW <= tol and eM <= tol and edW <= tol, (eW, eM, edW)
    wn = np.linalg.norm(W_prev_gpu)
    assert abs(st["w_norm"] - wn) <= 1e-5 * wn + 1e-12
    assert abs(st["o_norm"] - r.o_norm) <= 2 * tol * r.o_norm + 1e-6
    assert abs(st["update_rms"] - r.update_rms) <= 2 * tol * r.update_rms + 1e-6
    check_muon_stats_against_own_update(W_prev_gpu, Wg, st, ohp)
    for k, e in (("W", eW), ("M", eM), ("dW", edW)):
        worst[k] = max(worst.get(k, 0.0), e)
    return r.W, r.M


def compare_runs_equilibrated(gpu, W0s, grads_per_step, ohp, tol):
    """compare_runs for the equilibration mode: the oracle is stepped one step at a time
    from its own state (check_step); the GPU's axis must equal the oracle's where the
    choice is decided, and on a tie the oracle follows the GPU's axis. Returns the worst
    errors and the counts of decided / tied axis decisions."""
    worst = {"W": 0.0, "M": 0.0, "dW": 0.0, "decided": 0, "tied": 0}
    for i, W0 in enumerate(W0s):
        W = np.asarray(W0, np.float64)
        M = np.zeros_like(W)
        W_prev_gpu = W.copy()
        for t, gl in enumerate(grads_per_step):
            Wg, Mg, st = gpu[t][0][i], gpu[t][1][i], gpu[t][2][i]
            W, M = check_step(W, M, np.asarray(gl[i], np.float64), Wg, Mg, W_prev_gpu, st,
                              ohp, tol, worst)
            W_prev_gpu = Wg
    return worst


def seeded(rows, cols, seed, std):
    return wl.normal(rows, cols, seed, std)


def seeded_bf16(rows, cols, seed, std):
    return wl.normal(rows, cols, seed, std, bf16=True)
