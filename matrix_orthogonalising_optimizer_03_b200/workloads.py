"""Seeded synthetic workloads for the Muon step: matrix shapes, weights and gradients.

This module holds no step arithmetic. It only describes the shape sets and draws
their inputs, so the CPU oracle and the CUDA path can be fed the same values.

Shape sets follow the model shapes named on the pages:
  * GPT-160M (12 layers, hidden 768) and GPT-400M (24 layers, hidden 1024) and the
    MoE model (32 layers, hidden 512, 64 routed + 1 shared expert) of
    "MuonGS: Pretraining LLMs with Relaxed Weight-Norm Control", section 전제와 한계
    (experiment description).
  * the 399M-1.5B dense models of the "MUON IS SCALABLE FOR LLM TRAINING" review,
    section 2 (Key Methods and Approach, experiment design).
The FFN / expert widths (3072, 4096, 320, 5632) are the stated benchmark
configuration, not a page figure.

Random numbers: every tensor is drawn from NumPy's Philox generator keyed by
(base seed, workload id, matrix index, step, tensor kind). Values are drawn in
float32 and, for bf16 tensors, rounded to bfloat16 with round-to-nearest-even so
that both sides see identical bf16 values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import numpy as np

BASE_SEED = 0
KIND_W, KIND_G, KIND_ROWSCALE = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class MatrixSpec:
    index: int
    rows: int
    cols: int
    role: str


@dataclasses.dataclass(frozen=True)
class Run:
    """One hyper-parameter setting the workload is run with."""
    mode: str            # "muon" or "muongs"
    weight_decay: float
    equilibrate: bool = False


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    wid: int                                  # id used in the generator key
    layout: Tuple[Tuple[int, int, int, str], ...]  # (rows, cols, count, role)
    grad_dtype: str                           # "f32" or "bf16"
    grad_dist: str                            # "normal" | "student_t3" | "rowscaled"
    runs: Tuple[Run, ...]
    ns_fp32: bool = False
    lr: float = 0.02
    momentum: float = 0.95
    w_std: float = 0.02
    g_std: float = 1e-3
    steps: int = 1

    def matrices(self) -> List[MatrixSpec]:
        out, i = [], 0
        for rows, cols, count, role in self.layout:
            for _ in range(count):
                out.append(MatrixSpec(i, rows, cols, role))
                i += 1
        return out

    @property
    def n_matrices(self) -> int:
        return sum(c for _, _, c, _ in self.layout)

    @property
    def n_params(self) -> int:
        return sum(r * c * k for r, c, k, _ in self.layout)


WORKLOADS: Dict[str, Workload] = {
    "single_128x256": Workload(
        "single_128x256", 1, ((128, 256, 1, "single"),), "f32", "normal",
        (Run("muon", 0.1), Run("muongs", 0.1)), ns_fp32=True, steps=10),
    "gpt160m": Workload(
        "gpt160m", 2,
        ((768, 768, 48, "attn_qkvo"), (3072, 768, 12, "mlp_fc"), (768, 3072, 12, "mlp_proj")),
        "bf16", "normal", (Run("muongs", 0.0),)),
    "gpt400m": Workload(
        "gpt400m", 3,
        ((1024, 1024, 96, "attn_qkvo"), (4096, 1024, 24, "mlp_fc"), (1024, 4096, 24, "mlp_proj")),
        "bf16", "normal", (Run("muongs", 0.0), Run("muon", 0.1))),
    "moe_1b": Workload(
        "moe_1b", 4,
        ((320, 512, 4160, "expert_gate_up"), (512, 320, 2080, "expert_down"), (512, 512, 128, "attn_qkvo")),
        "bf16", "student_t3", (Run("muongs", 0.0),)),
    "dense_1p5b": Workload(
        "dense_1p5b", 5,
        ((5632, 2048, 48, "mlp_gate_up"), (2048, 5632, 24, "mlp_down"), (2048, 2048, 96, "attn_qkvo")),
        "bf16", "rowscaled", (Run("muon", 0.1, equilibrate=True),)),
}


def _rng(wid: int, index: int, step: int, kind: int) -> np.random.Generator:
    ss = np.random.SeedSequence([BASE_SEED, wid, index, step, kind])
    return np.random.Generator(np.random.Philox(ss))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The uint16 bit patterns of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def weight(w: Workload, spec: MatrixSpec) -> np.ndarray:
    """W_0 ~ N(0, w_std^2), float32, row-major rows x cols."""
    g = _rng(w.wid, spec.index, 0, KIND_W)
    return g.standard_normal((spec.rows, spec.cols), dtype=np.float32) * np.float32(w.w_std)


def grad(w: Workload, spec: MatrixSpec, step: int) -> np.ndarray:
    """G_step as float32 values (bf16-representable when the workload's grads are bf16)."""
    g = _rng(w.wid, spec.index, step, KIND_G)
    shape = (spec.rows, spec.cols)
    if w.grad_dist == "normal":
        x = g.standard_normal(shape, dtype=np.float32) * np.float32(w.g_std)
    elif w.grad_dist == "student_t3":
        x = (g.standard_t(3.0, shape) * w.g_std).astype(np.float32)
    elif w.grad_dist == "rowscaled":
        rs = np.exp(_rng(w.wid, spec.index, step, KIND_ROWSCALE).standard_normal(spec.rows))
        x = g.standard_normal(shape, dtype=np.float32) * np.float32(w.g_std)
        x *= rs.astype(np.float32)[:, None]
    else:
        raise ValueError(w.grad_dist)
    if w.grad_dtype == "bf16":
        x = bf16_round(x)
    return x


def ns_flops(rows: int, cols: int, steps: int = 5) -> int:
    """Algorithmic NS flops of one matrix (symmetric Gram and polynomial counted once).

    m = min, n = max. Per iteration: Gram m(m+1)n, polynomial m^2(m+1), apply 2 m^2 n.
    """
    m, n = min(rows, cols), max(rows, cols)
    return steps * (m * (m + 1) * n + m * m * (m + 1) + 2 * m * m * n)


def workload_ns_flops(w: Workload, steps: int = 5) -> int:
    return sum(ns_flops(r, c, steps) * k for r, c, k, _ in w.layout)


def normal(rows: int, cols: int, seed: int, std: float, bf16: bool = False) -> np.ndarray:
    """A seeded N(0, std^2) float32 matrix outside the named shape sets (test cases)."""
    g = np.random.Generator(np.random.Philox(np.random.SeedSequence([BASE_SEED, 1000, seed])))
    x = g.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    return bf16_round(x) if bf16 else x


def device_inputs(w: Workload, device, seed: int = 0, exact=(), step: int = 0, only=None):
    """W_0 and G_step for every matrix of a shape set, drawn on `device` with torch's
    seeded generator from the same distributions as `weight` / `grad`:
    N(0, w_std^2) weights; N(0, g_std^2), g_std * Student-t(3) (a normal over the root
    mean square of three normals), or exp(N(0,1)) row scales times N(0, g_std^2)
    gradients, rounded to bf16 when the set's gradients are bf16. Matrices whose
    index is in `exact` get the host generator's values instead, so that the oracle
    can be run on them with identical inputs. With `only` (a set of indices) just those
    matrices are drawn, in order (a subset for profiling; its values differ from the
    full set's). Returns (Ws fp32, Gs) as lists."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([BASE_SEED, w.wid, seed, step]).generate_state(1)[0]))
    gdt = torch.bfloat16 if w.grad_dtype == "bf16" else torch.float32
    exact = set(exact)
    Ws, Gs = [], []
    for spec in w.matrices():
        if only is not None and spec.index not in only:
            continue
        shape = (spec.rows, spec.cols)
        if spec.index in exact:
            Ws.append(torch.from_numpy(weight(w, spec)).to(device))
            Gs.append(torch.from_numpy(grad(w, spec, step)).to(device=device, dtype=gdt))
            continue
        Ws.append(torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * w.w_std)
        z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        if w.grad_dist == "student_t3":
            v = torch.randn((3,) + shape, generator=gen, device=device, dtype=torch.float32)
            z = z / torch.sqrt((v * v).mean(0))
        elif w.grad_dist == "rowscaled":
            z = z * torch.exp(torch.randn((spec.rows, 1), generator=gen, device=device))
        Gs.append((z * w.g_std).to(gdt))
    return Ws, Gs


def device_grads(w: Workload, device, seed: int = 0, exact=(), step: int = 0):
    """G_step for every matrix of a shape set, drawn on `device` from the distributions
    `device_inputs` uses, with a generator of their own keyed by (seed, step) (the
    weights are not drawn again). Matrices whose index is in `exact` get the host
    generator's `grad(w, spec, step)` values, so that the oracle can follow them."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([BASE_SEED, w.wid, seed, step, KIND_G])
                        .generate_state(1)[0]))
    gdt = torch.bfloat16 if w.grad_dtype == "bf16" else torch.float32
    exact = set(exact)
    Gs = []
    for spec in w.matrices():
        shape = (spec.rows, spec.cols)
        if spec.index in exact:
            Gs.append(torch.from_numpy(grad(w, spec, step)).to(device=device, dtype=gdt))
            continue
        z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        if w.grad_dist == "student_t3":
            v = torch.randn((3,) + shape, generator=gen, device=device, dtype=torch.float32)
            z = z / torch.sqrt((v * v).mean(0))
        elif w.grad_dist == "rowscaled":
            z = z * torch.exp(torch.randn((spec.rows, 1), generator=gen, device=device))
        Gs.append((z * w.g_std).to(gdt))
    return Gs


def sample_indices(w: Workload, extra: int = 8, seed: int = 7) -> List[int]:
    """One matrix per shape class (its first) plus `extra` seeded picks: the matrices a
    full-size parity check compares with the oracle one by one."""
    first = {}
    for s in w.matrices():
        first.setdefault((s.rows, s.cols), s.index)
    picks = sorted(first.values())
    rng = np.random.default_rng(seed)
    rest = [i for i in range(w.n_matrices) if i not in picks]
    picks += sorted(rng.choice(rest, size=min(extra, len(rest)), replace=False).tolist())
    return picks
