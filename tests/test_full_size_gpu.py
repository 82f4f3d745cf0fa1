"""Full-size parity: one step over each whole shape set, in the launch configuration
bench.py times (one plan over all matrices), checked matrix by matrix against the
oracle on a sample (one matrix per shape class plus seeded picks). Matrices are
independent, so the sampled comparison is exact for those matrices."""
import numpy as np
import pytest

from matrix_orthogonalising_optimizer_03_b200 import workloads as wl
from oracle import muon_oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(lib):
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    return B, torch


CASES = [("gpt160m", 0), ("gpt400m", 0), ("gpt400m", 1), ("moe_1b", 0), ("dense_1p5b", 0)]


@pytest.mark.parametrize("name,run_idx", CASES)
def test_full_shape_set_one_step(env, name, run_idx):
    B, torch = env
    w = wl.WORKLOADS[name]
    run = w.runs[run_idx]
    picks = wl.sample_indices(w)
    Ws, Gs = wl.device_inputs(w, "cuda", exact=picks)
    W0 = {i: Ws[i].double().cpu().numpy() for i in picks}
    Ms = [torch.zeros_like(x) for x in Ws]
    hp = B.hparams(lr=w.lr, momentum=w.momentum, weight_decay=run.weight_decay, mode=run.mode,
                   equilibrate=run.equilibrate)
    stats = B.new_stats(len(Ws))
    plan = B.Plan(Ws, Gs, Ms, hp)
    plan.step(stats=stats)
    torch.cuda.synchronize()
    assert plan.query_device_status() == 0
    st = B.decode_stats(stats)
    ohp = orc.HParams(lr=w.lr, momentum=w.momentum, weight_decay=run.weight_decay, mode=run.mode,
                      equilibrate=run.equilibrate)
    specs = w.matrices()
    worst = [0.0, 0.0, 0.0]
    for i in picks:
        G = wl.grad(w, specs[i], 0).astype(np.float64)
        r = orc.muon_step(W0[i], G, np.zeros_like(G), ohp)
        Wg = Ws[i].double().cpu().numpy()
        Mg = Ms[i].double().cpu().numpy()
        e_w, e_m = H.rel(Wg, r.W), H.rel(Mg, r.M)
        e_dw = H.rel(W0[i] - Wg, W0[i] - r.W)
        assert e_w <= H.TOL_BF16 and e_m <= H.TOL_BF16 and e_dw <= H.TOL_BF16, (i, e_w, e_m, e_dw)
        worst = [max(worst[0], e_w), max(worst[1], e_m), max(worst[2], e_dw)]
        assert abs(st[i]["w_norm"] - np.linalg.norm(W0[i])) <= 1e-5 * np.linalg.norm(W0[i])
        if run.equilibrate:
            assert st[i]["equil_axis"] in (1, 2)
    print(f"\nFULLSIZE {name} run {run_idx}: max rel err W {worst[0]:.2e} M {worst[1]:.2e} "
          f"dW {worst[2]:.2e} over {len(picks)} sampled matrices")
    plan.close()
    del Ws, Gs, Ms
    torch.cuda.empty_cache()
