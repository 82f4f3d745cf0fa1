"""ZeRO-1 sharded Muon: ownership partition (host) and the collective data movement
on two gloo ranks (CPU), checked against the oracle applied to the averaged gradient."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from matrix_orthogonalising_optimizer_03_b200 import distributed as D
from matrix_orthogonalising_optimizer_03_b200 import workloads as wl


def test_lpt_partition_balances_and_is_deterministic():
    w = wl.WORKLOADS["gpt160m"]
    costs = [wl.ns_flops(s.rows, s.cols) for s in w.matrices()]
    for world in (2, 3, 8):
        owner = D.lpt_partition(costs, world)
        assert owner == D.lpt_partition(costs, world)
        loads = [sum(c for c, o in zip(costs, owner) if o == r) for r in range(world)]
        assert max(loads) - min(loads) <= max(costs)
        assert sorted(set(owner)) == list(range(world))
    assert D.lpt_partition([5.0, 3.0, 3.0, 1.0], 2) == [0, 1, 1, 0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPES = [(12, 20), (20, 12), (16, 16), (8, 30), (30, 8)]


def _oracle_local_step(hp):
    from oracle import muon_oracle as orc
    import torch

    def step(Ws, Gs, Ms):
        for W, G, M in zip(Ws, Gs, Ms):
            r = orc.muon_step(W.double().numpy(), G.double().numpy(), M.double().numpy(), hp)
            W.copy_(torch.from_numpy(r.W))
            M.copy_(torch.from_numpy(r.M))
    return step


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    from oracle import muon_oracle as orc
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    hp = orc.HParams(mode="muongs", weight_decay=0.1)
    W0 = [wl.normal(r, c, 10 + i, 0.02) for i, (r, c) in enumerate(SHAPES)]
    opt = D.ShardedMuon(SHAPES, "cpu", init=[torch.from_numpy(w) for w in W0],
                        grad_dtype=torch.float32, local_step=_oracle_local_step(hp))
    for t in range(2):
        for i, (r, c) in enumerate(SHAPES):   # each rank has its own local gradient
            opt.grads[i].copy_(torch.from_numpy(wl.normal(r, c, 100 * t + 10 * rank + i, 1e-3)))
        opt.step()
    out[rank] = ([p.double().numpy().copy() for p in opt.params], sorted(opt.momenta),
                 list(opt.owner))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_sharded_step_matches_single_process_oracle():
    from oracle import muon_oracle as orc
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    hp = orc.HParams(mode="muongs", weight_decay=0.1)
    owner = res[0][2]
    assert res[1][2] == owner
    for rank in range(world):   # momentum only on the owner
        assert res[rank][1] == [i for i, o in enumerate(owner) if o == rank]
    for i, (r, c) in enumerate(SHAPES):
        W = wl.normal(r, c, 10 + i, 0.02).astype(np.float64)
        M = np.zeros_like(W)
        for t in range(2):
            G = np.mean([wl.normal(r, c, 100 * t + 10 * k + i, 1e-3) for k in range(world)],
                        axis=0, dtype=np.float64)
            step = orc.muon_step(W, G, M, hp)
            W, M = step.W, step.M
        for rank in range(world):   # every rank holds the same updated weights
            assert np.allclose(res[rank][0][i], W, rtol=1e-6, atol=1e-9)


@pytest.mark.gpu
def test_single_rank_sharded_step_runs_libmuon(lib):
    """World size 1 on the GPU: the owner's step is the libmuon plan step over views
    into the flat buffers; the result equals a plain plan step on the same inputs."""
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    shapes = [(256, 512), (768, 256), (100, 70)]
    W0 = [torch.tensor(wl.normal(r, c, 20 + i, 0.02)) for i, (r, c) in enumerate(shapes)]
    G = [torch.tensor(wl.normal(r, c, 30 + i, 1e-3, bf16=True)) for i, (r, c) in enumerate(shapes)]
    opt = D.ShardedMuon(shapes, "cuda", init=W0, mode="muongs")
    for g_view, g in zip(opt.grads, G):
        g_view.copy_(g)
    opt.step()
    Ws = [w.cuda() for w in W0]
    Gs = [g.cuda().to(torch.bfloat16) for g in G]
    Ms = [torch.zeros_like(w) for w in Ws]
    plan = B.Plan(Ws, Gs, Ms, B.hparams(mode="muongs"))
    plan.step()
    torch.cuda.synchronize()
    for a, b in zip(opt.params, Ws):
        assert torch.allclose(a, b, rtol=0, atol=1e-6)
    plan.close()


@pytest.mark.gpu
def test_single_rank_nccl_sharded_steps_match_oracle(lib):
    """The NCCL branch (in-place reduce_scatter_tensor and all_gather_into_tensor) on a
    one-rank NCCL process group, with the libmuon plan as the owner's step: three MuonGS
    steps, each weight against the float64 oracle at the bf16 path's tolerance."""
    import torch
    import torch.distributed as dist
    from oracle import muon_oracle as orc
    from tests import gpu_helpers as H
    shapes = [(256, 512), (768, 256), (100, 70), (512, 512)]
    W0 = [wl.normal(r, c, 40 + i, 0.02) for i, (r, c) in enumerate(shapes)]
    grads = [[wl.normal(r, c, 50 + 10 * t + i, 1e-3, bf16=True) for i, (r, c) in enumerate(shapes)]
             for t in range(3)]
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        opt = D.ShardedMuon(shapes, "cuda", init=[torch.from_numpy(w) for w in W0], mode="muongs")
        assert opt.grouped and opt.backend == "nccl"
        got = []
        for t in range(3):
            for g_view, g in zip(opt.grads, grads[t]):
                g_view.copy_(torch.from_numpy(g))
            opt.step()
            torch.cuda.synchronize()
            got.append([p.double().cpu().numpy() for p in opt.params])
        assert opt.plan.query_device_status() == 0
        opt.plan.close()
    finally:
        dist.destroy_process_group()
    hp = orc.HParams(mode="muongs")
    for i in range(len(shapes)):
        res = orc.muon_run(W0[i], [g[i] for g in grads], hp)
        W_prev_g = W_prev_o = W0[i].astype(np.float64)
        for t, r in enumerate(res):
            assert H.rel(got[t][i], r.W) <= H.TOL_BF16
            assert H.rel(W_prev_g - got[t][i], W_prev_o - r.W) <= H.TOL_BF16, (i, t)
            W_prev_g, W_prev_o = got[t][i], r.W
