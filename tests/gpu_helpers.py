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
            W_prev_gpu, W_prev_orc = Wg, r.W
    return worst


def seeded(rows, cols, seed, std):
    return wl.normal(rows, cols, seed, std)


def seeded_bf16(rows, cols, seed, std):
    return wl.normal(rows, cols, seed, std, bf16=True)
