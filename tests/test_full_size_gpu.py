"""Full-size parity: 10 consecutive steps over each whole shape set, in the launch
configuration bench.py times (one cached plan over all matrices, its CUDA graph
replayed from the third step on), checked matrix by matrix against the oracle on a
sample: one matrix per shape class plus two seeded picks. Matrices are independent,
so the sampled comparison is exact for those matrices. The oracle steps each sampled
matrix from its own state with the same gradients; W_t, M_t and dW_t must agree
within the bf16 path's 3e-2 at every step, and, with equilibration, the axis where it
is decided (see tests/gpu_helpers.py)."""
import numpy as np
import pytest

from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
from oracle import muon_oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

STEPS = 10


@pytest.fixture(scope="module")
def env(lib):
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    return B, torch


CASES = [("gpt160m", 0), ("gpt400m", 0), ("gpt400m", 1), ("moe_1b", 0), ("dense_1p5b", 0)]


@pytest.mark.parametrize("name,run_idx", CASES)
def test_full_shape_set_ten_steps(env, name, run_idx):
    B, torch = env
    w = wl.WORKLOADS[name]
    run = w.runs[run_idx]
    picks = wl.sample_indices(w, extra=2)
    specs = w.matrices()
    Ws, Gs = wl.device_inputs(w, "cuda", exact=picks)
    W_orc = {i: Ws[i].double().cpu().numpy() for i in picks}
    M_orc = {i: np.zeros_like(W_orc[i]) for i in picks}
    W_prev = dict(W_orc)
    Ms = [torch.zeros_like(x) for x in Ws]
    hp = B.hparams(lr=w.lr, momentum=w.momentum, weight_decay=run.weight_decay, mode=run.mode,
                   equilibrate=run.equilibrate)
    ohp = orc.HParams(lr=w.lr, momentum=w.momentum, weight_decay=run.weight_decay, mode=run.mode,
                      equilibrate=run.equilibrate)
    stats = B.new_stats(len(Ws))
    plan = B.Plan(Ws, Gs, Ms, hp)
    worst = {}
    for t in range(STEPS):
        if t > 0:   # fresh gradients in place (the plan holds the buffers' addresses)
            for g_dev, g_new in zip(Gs, wl.device_grads(w, "cuda", exact=picks, step=t)):
                g_dev.copy_(g_new)
        plan.step(stats=stats)
        torch.cuda.synchronize()
        assert plan.query_device_status() == 0
        st = B.decode_stats(stats)
        for i in picks:
            Wg = Ws[i].double().cpu().numpy()
            Mg = Ms[i].double().cpu().numpy()
            G = wl.grad(w, specs[i], t).astype(np.float64)
            W_orc[i], M_orc[i] = H.check_step(W_orc[i], M_orc[i], G, Wg, Mg, W_prev[i], st[i],
                                              ohp, H.TOL_BF16, worst)
            W_prev[i] = Wg
    print(f"\nFULLSIZE {name} run {run_idx}: {STEPS} steps, max rel err W {worst['W']:.2e} "
          f"M {worst['M']:.2e} dW {worst['dW']:.2e} over {len(picks)} sampled matrices"
          + (f"; axis decided {worst.get('decided', 0)} tied {worst.get('tied', 0)}"
             if run.equilibrate else ""))
    plan.close()
    del Ws, Gs, Ms
    torch.cuda.empty_cache()
