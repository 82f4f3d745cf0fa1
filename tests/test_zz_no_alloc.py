"""The workspace-free Newton-Schulz entry point (muon_newton_schulz_noalloc).

It serves callers that cannot call cudaMalloc, for example code running under a
memory pool that owns all device memory, or code that cannot take the device-wide
synchronisation an allocation may cause. Its scratch is the library's static
32 MiB device array instead of a caller workspace.

These tests call it through the C ABI twice in a row and check each result
  * against muon_newton_schulz_batched (caller workspace) on the same input: the two
    run the same kernels and tile shapes, so they agree to the summation-order noise
    of the fp64 norm atomics (relative 1e-5 here, far below the bf16 path's 3e-2,
    so a stale scratch or a wrong slab offset cannot pass);
  * against the float64 oracle, at the path's own tolerance (3e-2 bf16, 1e-4 fp32).
The second call of each pair is smaller than the first, so stale scratch contents
would show. A matrix too large for the static array, and a status word outside
device memory, are rejected on the host.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from oracle import muon_oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

TOL_SAME_KERNELS = 1e-5


@pytest.fixture(scope="module")
def env(lib):
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    return B, torch


def _pair(B, torch, x_np, dtype, hp):
    x = torch.tensor(x_np, device="cuda").to(dtype)
    o_ref = torch.empty_like(x)
    B.newton_schulz([x], [o_ref], hp)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    o_new = torch.empty_like(x)
    B.newton_schulz_noalloc(x, o_new, hp, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return (o_new.double().cpu().numpy(), o_ref.double().cpu().numpy(),
            x.double().cpu().numpy())


@pytest.mark.parametrize("fp32", [False, True])
def test_noalloc_matches_workspace_entry_point_twice(env, fp32):
    B, torch = env
    hp = B.hparams(ns_fp32=fp32)
    dtype = torch.float32 if fp32 else torch.bfloat16
    tol = H.TOL_FP32 if fp32 else H.TOL_BF16
    # bf16: a CTA-pair shape (m = 768) then a single-CTA ragged tall shape
    shapes = [(768, 3072), (517, 300)] if not fp32 else [(300, 517), (64, 40)]
    for i, (r, c) in enumerate(shapes):
        x = H.seeded(r, c, 900 + i, 1e-3)
        got, ref, x_used = _pair(B, torch, x, dtype, hp)
        assert got.shape == (r, c)
        assert np.linalg.norm(got) > 0
        assert H.rel(got, ref) <= TOL_SAME_KERNELS, (r, c, H.rel(got, ref))
        want = orc.orthogonalise(x_used, orc.HParams())
        assert H.rel(got, want) <= tol, (r, c, H.rel(got, want))


def test_noalloc_rejects_matrices_beyond_the_static_scratch(env):
    B, torch = env
    hp = B.hparams()
    x = torch.zeros(2048, 2048, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(x)
    with pytest.raises(B.MuonError) as e:
        B.newton_schulz_noalloc(x, o, hp)
    assert e.value.status == 5   # MUON_ERR_WORKSPACE
    m = B.MuonNSMatrix(x.data_ptr(), x.data_ptr(), 64, 64, 64, 64, 1, 0)
    assert B.load().muon_newton_schulz_noalloc(ctypes.byref(m), ctypes.byref(hp), None, None) == 4


def test_noalloc_rejects_a_status_word_in_host_memory(env):
    """The C entry point checks that status_dev is device memory of the current device
    (a kernel stores to it) and returns MUON_ERR_INVALID_ARG before enqueueing."""
    B, torch = env
    hp = B.hparams()
    x = torch.zeros(64, 96, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(x)
    m = B.MuonNSMatrix(x.data_ptr(), o.data_ptr(), 64, 96, 96, 96, 1, 0)
    host_word = ctypes.c_uint32(0)
    st = B.load().muon_newton_schulz_noalloc(ctypes.byref(m), ctypes.byref(hp),
                                             ctypes.addressof(host_word), None)
    assert st == 1
