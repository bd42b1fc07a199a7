"""gspn_forward_noalloc: the forward with its workspace taken from a fixed device array inside
the library, for callers that cannot allocate device memory when they call (for example code
running under another component's allocator, or on a path where cudaMalloc / cudaFree would
synchronise the device). The GPU test calls it through the C ABI twice in a row and compares
each result with gspn_forward's on the same inputs. This file is collected last on purpose."""
import ctypes

import pytest
import torch

import linear_spatial_propagation_gspn_b200 as g

SCRATCH_BYTES = 64 << 20


def _call(desc, x, a, lam, u, y):
    return g.lib().gspn_forward_noalloc(ctypes.byref(desc), x.data_ptr(), a.data_ptr(), lam.data_ptr(),
                                        u.data_ptr(), y.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_rejects_problems_larger_than_the_scratch():
    d = g.make_desc(16, 8, 1024, 1024, g.SHARED, 15, g.F32, g.ALGO_GENERIC)
    assert g.workspace_size(d) > SCRATCH_BYTES
    fake = 0x10000
    s = g.lib().gspn_forward_noalloc(ctypes.byref(d), fake, fake, fake, fake, fake, None)
    assert s == g.GSPN_ERR_WORKSPACE
    assert g.lib().gspn_forward_noalloc(None, fake, fake, fake, fake, fake, None) == g.GSPN_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("shape,wmode,dtype", [((2, 3, 256, 256), g.SHARED, torch.float32),
                                               ((1, 4, 96, 128), g.PER_CHANNEL, torch.bfloat16)])
def test_noalloc_matches_forward_on_two_calls(shape, wmode, dtype):
    gen = torch.Generator(device="cuda").manual_seed(77)
    N, C, H, W = shape
    Cw = 1 if wmode == g.SHARED else C
    x = torch.randn(shape, device="cuda", generator=gen).to(dtype)
    lam = torch.rand(shape, device="cuda", generator=gen).to(dtype)
    u = torch.randn(shape, device="cuda", generator=gen).to(dtype)
    a = torch.randn(4, N, Cw, 3, H, W, device="cuda", generator=gen).to(dtype)
    desc = g.desc_for(x, wmode, 15)
    assert g.workspace_size(desc) <= SCRATCH_BYTES
    ref = g.forward(x, a, lam, u, wmode, 15)
    tol = (1e-5 if dtype == torch.float32 else 2e-2) * max(1.0, ref.float().abs().max().item())
    for call in range(2):
        y = torch.full_like(x, float("nan"))
        assert _call(desc, x, a, lam, u, y) == g.GSPN_OK
        torch.cuda.synchronize()
        err = (y.float() - ref.float()).abs().max().item()
        assert err <= tol, f"call {call}: max|d| {err} > {tol}"
        # second call on different data must not see the first call's scratch contents
        x = x.flip(-1).contiguous()
        ref = g.forward(x, a, lam, u, wmode, 15)
