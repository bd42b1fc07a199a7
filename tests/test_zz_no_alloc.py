"""gspn_forward_noalloc: the forward with its workspace taken from a fixed device array inside
the library, for callers that cannot allocate device memory when they call (for example code
running under another component's allocator, or on a path where cudaMalloc / cudaFree would
synchronise the device). The GPU test calls it through the C ABI twice in a row and compares
each result with gspn_forward's on the same inputs and with the float64 oracle. This file is
collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import linear_spatial_propagation_gspn_b200 as g
import oracle

SCRATCH_BYTES = 64 << 20


def _call(desc, x, a, lam, u, y):
    return g.lib().gspn_forward_noalloc(ctypes.byref(desc), x.data_ptr(), a.data_ptr(), lam.data_ptr(),
                                        u.data_ptr(), y.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_rejects_before_touching_the_device():
    """Every rejection is decided on the host; null pointers are passed so that a regression in
    the order of the checks would stop at the null check instead of launching a kernel."""
    L = g.lib()
    big = g.make_desc(16, 8, 1024, 1024, g.SHARED, 15, g.F32, g.ALGO_GENERIC)
    assert g.workspace_size(big) > SCRATCH_BYTES
    assert L.gspn_forward_noalloc(ctypes.byref(big), None, None, None, None, None, None) == g.GSPN_ERR_WORKSPACE
    assert L.gspn_forward_noalloc(None, None, None, None, None, None, None) == g.GSPN_ERR_INVALID_ARG
    bad = g.make_desc(1, 1, 0, 8)                                   # malformed: H = 0
    assert L.gspn_forward_noalloc(ctypes.byref(bad), None, None, None, None, None, None) == g.GSPN_ERR_INVALID_ARG
    # well formed, but the forced sweep family does not run per-direction lambda / u
    unsup = g.make_desc(1, 1, 64, 64, g.PER_CHANNEL, 15, g.F32, g.ALGO_SWEEP, per_dir=1)
    assert g.selected_algo(unsup) == -1
    assert L.gspn_forward_noalloc(ctypes.byref(unsup), None, None, None, None, None, None) == g.GSPN_ERR_UNSUPPORTED
    small = g.make_desc(1, 2, 32, 32)
    assert L.gspn_forward_noalloc(ctypes.byref(small), None, None, None, None, None, None) == g.GSPN_ERR_INVALID_ARG


def _f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


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
    for call in range(2):
        ref = g.forward(x, a, lam, u, wmode, 15)
        ref_o = oracle.forward(_f64(x), _f64(a), _f64(lam), _f64(u), wmode, 15)
        m = float(np.abs(ref_o).max())
        tol = 1e-5 * max(1.0, m) if dtype == torch.float32 else 2e-2 * m
        y = torch.full_like(x, float("nan"))
        assert _call(desc, x, a, lam, u, y) == g.GSPN_OK
        torch.cuda.synchronize()
        err = (y.float() - ref.float()).abs().max().item()
        assert err <= tol, f"call {call}: max|d| against gspn_forward {err} > {tol}"
        err_o = float(np.abs(_f64(y) - ref_o).max())
        assert err_o <= tol, f"call {call}: max|d| against the oracle {err_o} > {tol}"
        # the second call runs on different data and must not see the first call's scratch
        x = x.flip(-1).contiguous()
