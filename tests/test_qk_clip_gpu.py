"""QK-Clip on the GPU against the oracle (exact up to fp32 rounding of gamma^power)."""
import numpy as np
import pytest

from oracle import muon_oracle as orc
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def test_qk_clip_matches_oracle(lib):
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    n_heads, dh, dr, d = 8, 64, 32, 512
    Wq = H.seeded(n_heads * dh, d, 1, 0.02)       # non-rotary q, head-major rows
    Wqr = H.seeded(n_heads * dr, d, 2, 0.02)      # rotary q
    Wk = H.seeded(n_heads * dh, 333, 3, 0.02)     # non-rotary k (odd width: scalar path)
    Wkr = H.seeded(dr, d, 4, 0.02)                # shared rotary k
    s_max = np.array([50, 100, 100.5, 250, 1e4, 99, 400, 101], np.float32)
    slices = []
    for h in range(n_heads):
        slices += [(0, h * dh, dh, h, 0.5), (1, h * dr, dr, h, 1.0), (2, h * dh, dh, h, 0.5)]
    want = orc.qk_clip([Wq, Wqr, Wk, Wkr], slices, s_max.astype(np.float64), tau=100.0)
    dev = [torch.tensor(x, device="cuda") for x in (Wq, Wqr, Wk, Wkr)]
    B.qk_clip([(dev[i], r0, nr, h, pw) for i, r0, nr, h, pw in slices],
              torch.tensor(s_max, device="cuda"), tau=100.0)
    torch.cuda.synchronize()
    for g, w in zip(dev, want):
        assert np.allclose(g.double().cpu().numpy(), w, rtol=2e-7, atol=0)
    assert np.array_equal(dev[3].cpu().numpy(), Wkr)   # shared rotary key untouched


def test_qk_clip_rejects_overlap_and_bad_head(lib):
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    W = torch.zeros(16, 8, device="cuda")
    s = torch.ones(2, device="cuda")
    with pytest.raises(B.MuonError) as e:
        B.qk_clip([(W, 0, 8, 0, 0.5), (W, 4, 8, 1, 0.5)], s)
    assert e.value.status == 4
    with pytest.raises(B.MuonError) as e:
        B.qk_clip([(W, 0, 8, 5, 0.5)], s)
    assert e.value.status == 1


def test_qk_clip_many_slices_in_several_launches(lib):
    """More slices than one launch carries (448), given out of row order, in heads of 24
    rows (blocks of 16 rows end ragged), on aligned and odd-width matrices; against the
    oracle."""
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    n_heads, dh = 40, 24
    widths = [256, 130, 512, 77]
    Ws = [H.seeded(n_heads * dh, wd, 30 + i, 0.02) for i, wd in enumerate(widths)]
    rng = np.random.default_rng(5)
    s_max = np.where(rng.random(n_heads) < 0.5, 150.0, 60.0).astype(np.float32)
    slices = []
    for i in range(len(Ws)):
        for h in range(n_heads):
            for part in range(3):  # three slices of 8 rows per head
                slices.append((i, h * dh + 8 * part, 8, h, 0.5 if i % 2 == 0 else 1.0))
    order = rng.permutation(len(slices))
    slices = [slices[k] for k in order]
    assert len(slices) > 448
    want = orc.qk_clip(Ws, slices, s_max.astype(np.float64), tau=100.0)
    dev = [torch.tensor(x, device="cuda") for x in Ws]
    B.qk_clip([(dev[i], r0, nr, h, pw) for i, r0, nr, h, pw in slices],
              torch.tensor(s_max, device="cuda"), tau=100.0)
    torch.cuda.synchronize()
    for g, w in zip(dev, want):
        assert np.allclose(g.double().cpu().numpy(), w, rtol=2e-7, atol=0)


def test_qk_clip_overlap_found_in_any_order(lib):
    """An overlap with a slice that is not the next one in row order (an empty slice
    between them, input unsorted) is rejected before any launch; touching slices are not
    an overlap."""
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    W = torch.ones(32, 8, device="cuda")
    s = torch.full((2,), 50.0, device="cuda")
    with pytest.raises(B.MuonError) as e:
        B.qk_clip([(W, 20, 4, 0, 0.5), (W, 6, 2, 1, 0.5), (W, 4, 0, 0, 0.5), (W, 0, 8, 0, 0.5)], s)
    assert e.value.status == 4
    B.qk_clip([(W, 8, 8, 0, 0.5), (W, 0, 8, 1, 0.5)], s)  # touching: accepted
    torch.cuda.synchronize()
