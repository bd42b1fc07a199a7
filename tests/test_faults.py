"""Failure detection without faulting the GPU: a bounded device-side wait on a flag that
nothing sets gives up after its limit, records GSPN_ERR_DEVICE_TIMEOUT in the workspace status
word, and the context stays usable for the next call."""
import pytest
import torch

import linear_spatial_propagation_gspn_b200 as g

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert g.debug_wait_timeout(ws, 2_000_000) == g.GSPN_OK          # 2 ms limit
    assert g.device_status(ws) == g.GSPN_ERR_DEVICE_TIMEOUT
    assert g.device_status(ws) == g.GSPN_OK                          # status was cleared
    x = torch.randn(1, 1, 8, 8, device="cuda")
    a = torch.randn(1, 1, 1, 3, 8, 8, device="cuda")
    y = g.forward(x, a, torch.ones_like(x), torch.ones_like(x), 0, 1)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()


def test_forward_status_ok():
    x = torch.randn(1, 2, 16, 16, device="cuda")
    a = torch.randn(4, 1, 2, 3, 16, 16, device="cuda")
    d = g.desc_for(x, 0, 15)
    ws = g.alloc_workspace(d, False, x.device)
    g.forward(x, a, torch.rand_like(x), torch.randn_like(x), 0, 15, ws=ws)
    assert g.device_status(ws) == g.GSPN_OK


def test_copy_ceiling_copies():
    src = torch.randn(1 << 20, device="cuda")
    dst = torch.empty_like(src)
    g.copy_ceiling(src, dst)
    torch.cuda.synchronize()
    assert torch.equal(src, dst)
