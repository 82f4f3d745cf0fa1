"""Data-parallel Muon with sharded optimizer state (ZeRO-1 style).

The distributed variant of "[논문 AI 리뷰] MUON IS SCALABLE FOR LLM TRAINING TECHNICAL
REPORT", section 2 (distributed implementation): the momentum is partitioned over
the data-parallel ranks, the full gradient of a matrix is gathered on the rank that
owns it, the owner runs the Newton-Schulz step on the whole matrix and updates it,
and the updated weights are shared with every rank. Communication is about that of
a data-parallel all-reduce (reduce-scatter + all-gather), i.e. the "1.0-1.25x of
distributed AdamW" the pages quote.

Layout. Matrices are assigned to owners by longest-processing-time-first on their
Newton-Schulz flops. Gradients and weights live in flat buffers ordered by owner,
one equal-size segment per rank (zero padding at the end of short segments), so
one reduce-scatter and one all-gather move everything:

    grads  [rank 0 matrices | pad][rank 1 matrices | pad] ...  --reduce-scatter(avg)-->
    owned  [rank r matrices | pad]  --local Muon step (libmuon, in place on W)-->
    W      [rank 0 matrices | pad][rank 1 ...]   <--all-gather of each owner's segment

On NCCL the collectives are reduce_scatter_tensor / all_gather_into_tensor, both in
place (this rank's segment of the flat buffer is the reduce-scatter's output and the
all-gather's input, NCCL's in-place forms), so a step allocates and copies nothing
beyond the collectives themselves. They run whenever a process group exists, a
single-rank NCCL group included. On gloo (CPU tests) the same data movement is done
with all_reduce + slicing and all_gather. Without a process group the step is the
local step alone. The per-matrix parameter and gradient tensors handed out are views
into the flat buffers, so a training loop writes gradients in place and reads the
updated weights without copies.
"""
from __future__ import annotations

import heapq
from typing import Callable, List, Optional, Sequence, Tuple

from . import workloads as wl


def lpt_partition(costs: Sequence[float], world: int) -> List[int]:
    """Owner rank of each item: longest-processing-time-first onto the least loaded
    rank (ties to the lower rank), which keeps the largest load within one item of
    the mean. Deterministic, so every rank computes the same assignment."""
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    heap = [(0.0, r) for r in range(world)]
    owner = [0] * len(costs)
    for i in order:
        load, r = heapq.heappop(heap)
        owner[i] = r
        heapq.heappush(heap, (load + costs[i], r))
    return owner


class ShardedMuon:
    """ZeRO-1 Muon over the default process group (or a single process).

    shapes: (rows, cols) of every hidden matrix, identical on all ranks.
    init:   optional list of initial weights (torch tensors, any device) to copy in.
    hp:     keyword arguments of binding.hparams (lr, momentum, weight_decay, mode, ...).
    local_step: optional replacement of the owner's step, f(W_list, G_list, M_list),
            used by CPU tests; by default the libmuon plan step runs on the owner's GPU.
    """

    def __init__(self, shapes: Sequence[Tuple[int, int]], device, init=None,
                 grad_dtype=None, local_step: Optional[Callable] = None, **hp):
        import torch
        import torch.distributed as dist
        self.torch, self.dist = torch, dist
        self.grouped = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size() if self.grouped else 1
        self.rank = dist.get_rank() if self.grouped else 0
        self.backend = dist.get_backend() if self.grouped else None
        self.device = torch.device(device)
        self.shapes = [tuple(s) for s in shapes]
        self.owner = lpt_partition([wl.ns_flops(r, c) for r, c in self.shapes], self.world)
        gdt = grad_dtype or (torch.bfloat16 if self.device.type == "cuda" else torch.float32)

        # flat, owner-ordered layout with equal segments
        self.offsets = [0] * len(self.shapes)
        seg_len = [0] * self.world
        for i, (r, c) in enumerate(self.shapes):
            o = self.owner[i]
            self.offsets[i] = seg_len[o]
            seg_len[o] += r * c
        self.seg = max(seg_len) if seg_len else 0
        self.seg = (self.seg + 63) // 64 * 64  # keep every segment 256-byte aligned
        n = self.seg * self.world
        self.flat_w = torch.zeros(n, dtype=torch.float32, device=self.device)
        self.flat_g = torch.zeros(n, dtype=gdt, device=self.device)
        # this rank's segment: the in-place reduce-scatter leaves the averaged gradients
        # of the matrices it owns here
        self.my_g = self.flat_g[self.rank * self.seg:(self.rank + 1) * self.seg]
        self.my_w = self.flat_w[self.rank * self.seg:(self.rank + 1) * self.seg]
        self.params, self.grads = [], []
        for i, (r, c) in enumerate(self.shapes):
            base = self.owner[i] * self.seg + self.offsets[i]
            self.params.append(self.flat_w[base:base + r * c].view(r, c))
            self.grads.append(self.flat_g[base:base + r * c].view(r, c))
            if init is not None:
                self.params[i].copy_(init[i])
        # momentum only for the matrices this rank owns (the ZeRO-1 saving)
        self.mine = [i for i in range(len(self.shapes)) if self.owner[i] == self.rank]
        self.momenta = {i: torch.zeros(self.shapes[i], dtype=torch.float32, device=self.device)
                        for i in self.mine}
        self._my_w = [self.params[i] for i in self.mine]
        self._my_g = [self.my_g[self.offsets[i]:self.offsets[i] + r * c].view(r, c)
                      for i, (r, c) in ((i, self.shapes[i]) for i in self.mine)]
        self._my_m = [self.momenta[i] for i in self.mine]
        self.local_step = local_step
        self.plan = None
        if local_step is None and self.mine:
            from . import binding as B
            self.plan = B.Plan(self._my_w, self._my_g, self._my_m, B.hparams(**hp))

    # -- collectives ------------------------------------------------------------
    def _reduce_scatter_grads(self):
        dist = self.dist
        if not self.grouped:
            return                          # one process: my_g is the whole buffer
        if self.backend == "nccl":
            dist.reduce_scatter_tensor(self.my_g, self.flat_g, op=dist.ReduceOp.AVG)
            return
        buf = self.flat_g.clone()
        dist.all_reduce(buf, op=dist.ReduceOp.SUM)
        self.my_g.copy_(buf[self.rank * self.seg:(self.rank + 1) * self.seg] / self.world)

    def _all_gather_weights(self):
        dist = self.dist
        if not self.grouped:
            return
        if self.backend == "nccl":
            dist.all_gather_into_tensor(self.flat_w, self.my_w)
            return
        parts = list(self.flat_w.split(self.seg))
        dist.all_gather(parts, self.my_w.clone())

    # -- one optimizer step -----------------------------------------------------
    def step(self, stats=None):
        """Averages the gradients onto their owners, runs the owners' Muon step and
        shares the updated weights. The gradient views must hold this rank's local
        gradients on entry."""
        self._reduce_scatter_grads()
        if self.mine:
            if self.local_step is not None:
                self.local_step(self._my_w, self._my_g, self._my_m)
            else:
                self.plan.step(stats=stats)
        self._all_gather_weights()
