"""Failure detection without a GPU fault: a bounded wait that runs out is reported
as MUON_ERR_TIMEOUT through the workspace error word, the context stays usable,
and the word is cleared by reading it."""
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(lib):
    import torch
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    ws = B.new_workspace(256)
    ws.zero_()
    assert lib.muon_wait_probe(ws.data_ptr(), 200_000, None) == 0   # ~0.1 ms of SM clock
    assert lib.muon_query_device_status(ws.data_ptr(), None) == 7    # MUON_ERR_TIMEOUT
    assert lib.muon_query_device_status(ws.data_ptr(), None) == 0    # cleared by the read
    # the context still runs work normally
    x = torch.randn(64, 96, device="cuda").to(torch.bfloat16)
    o = torch.empty_like(x)
    B.newton_schulz([x], [o], B.hparams())
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert lib.muon_wait_probe(ws.data_ptr(), 0, None) == 1           # limit out of range
