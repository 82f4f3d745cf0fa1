"""The accumulated-learning-rate study on the GPU path: C_T = sum_t eta / ||W_t|| from
the per-step statistics of the plan, against the bounds of "MuonGS: Pretraining LLMs
with Relaxed Weight-Norm Control" (section 전제와 한계: Theorem 4.1, Proposition 4.2)
for MuonGS and the MuonW radius bound of its section "무엇과 다른가" for decoupled
weight decay.

The bounds are stated for an update of Frobenius norm at most sqrt(p); the quintic
Newton-Schulz iteration only approximates the polar factor, so p is replaced by the
largest ||O_t||^2 the run produced (p_eff), as in the oracle's own pin of the same
bounds with the Newton-Schulz update.
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


def _run_stats(B, torch, W0s, steps, hp, seed):
    """Runs `steps` plan steps with fresh seeded gradients; returns per step the decoded
    statistics (w_norm is the norm of the pre-step W_t) and the final weights."""
    Ws = [torch.tensor(w, dtype=torch.float32, device="cuda") for w in W0s]
    Ms = [torch.zeros_like(w) for w in Ws]
    Gs = [torch.empty(w.shape, dtype=torch.bfloat16, device="cuda") for w in Ws]
    stats = B.new_stats(len(Ws))
    plan = B.Plan(Ws, Gs, Ms, hp)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    out = []
    for _ in range(steps):
        for g in Gs:
            g.copy_(torch.randn(g.shape, generator=gen, device="cuda") * 1e-3)
        plan.step(stats=stats)
        out.append(B.decode_stats(stats))
    torch.cuda.synchronize()
    assert plan.query_device_status() == 0
    plan.close()
    return out, [w.double().cpu().numpy() for w in Ws]


def test_muongs_accumulated_lr_bounds_on_gpu(env):
    """MuonGS, wd 0, scale none, constant eta over 2T = 400 steps."""
    B, torch = env
    shapes = [(64, 128), (256, 512)]
    eta, T = 0.02, 200
    W0s = [H.seeded(r, c, 900 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    hp = B.hparams(lr=eta, momentum=0.95, mode="muongs", scale="none")
    st, _ = _run_stats(B, torch, W0s, 2 * T, hp, seed=7)
    for i, (r, c) in enumerate(shapes):
        norms = [s[i]["w_norm"] for s in st]
        r0 = norms[0]
        assert r0 == pytest.approx(np.linalg.norm(W0s[i].astype(np.float64)), rel=1e-5)
        p_eff = max(s[i]["o_norm"] ** 2 for s in st)
        assert p_eff <= 1.5 * min(r, c)
        CT = orc.accumulated_lr([eta] * T, norms[:T])
        C2T = orc.accumulated_lr([eta] * (2 * T), norms)
        assert CT >= orc.muongs_ct_lower_bound(r0, p_eff, eta, T) * (1 - 1e-5)
        assert C2T - CT >= orc.muongs_late_lower_bound(r0, p_eff, eta, T) * (1 - 1e-5)
        # the norm grows only at second order: r_T^2 <= r_0^2 + p eta^2 T
        assert norms[T] ** 2 <= (r0 ** 2 + p_eff * eta ** 2 * T) * (1 + 1e-5)


def test_muonw_radius_on_gpu(env):
    """Plain Muon with decoupled decay: ||W_t|| <= R = max(r0, sqrt(p_eff)/lambda) and
    C_T >= eta T / R."""
    B, torch = env
    shapes = [(32, 64), (256, 256)]
    eta, lam, T = 0.05, 2.0, 300
    W0s = [H.seeded(r, c, 950 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    hp = B.hparams(lr=eta, momentum=0.95, weight_decay=lam, mode="muon", scale="none")
    st, W_end = _run_stats(B, torch, W0s, T, hp, seed=8)
    for i, (r, c) in enumerate(shapes):
        norms = [s[i]["w_norm"] for s in st] + [float(np.linalg.norm(W_end[i]))]
        p_eff = max(s[i]["o_norm"] ** 2 for s in st)
        R = orc.muonw_radius(norms[0], p_eff, lam)
        assert max(norms) <= R * (1 + 1e-5)
        assert orc.accumulated_lr([eta] * T, norms[:T]) >= eta * T / R * (1 - 1e-5)
