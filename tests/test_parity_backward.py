"""Backward (reverse scans) against the float64 oracle's backward.

Small forced-plane cases (per-channel) cover odd sizes, masks and both dtypes. Each named
workload then runs its backward at full size in the library's own configuration: per-plane
gradients (dx, dlambda, du and, per-channel, da) are checked on seeded sample planes; in the
channel-shared mode da is a sum over channels, so it is checked over every channel of one batch
item (highres), or, for 1152 channels, on a channel subset plus additivity over channel groups."""
import numpy as np
import pytest
import torch

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
import oracle
from gspn_inputs import small_case

from _cases import assert_close, check_backward, f64, grad_tol

pytestmark = pytest.mark.gpu

SHAPES = [(1, 4, 16, 16), (2, 3, 17, 33), (1, 2, 1, 5), (1, 2, 5, 1), (2, 2, 31, 7), (1, 1, 64, 40), (2, 1, 56, 56)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mask", [15, 1, 6, 9])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_plane_backward_small(shape, mask, dtype):
    wl = small_case(*shape, mask=mask, wmode=0, dtype=dtype, seed=11 * sum(shape) + mask)
    d = g.make_desc(*shape, 0, mask, 0 if dtype == "f32" else 1, g.ALGO_PLANE)
    assert g.selected_algo(d, True) == g.ALGO_PLANE
    check_backward(wl, g.ALGO_PLANE)


def _sample(wl, k, seed):
    rng = np.random.default_rng(seed)
    idx = rng.choice(wl.N * wl.C, size=min(k, wl.N * wl.C), replace=False)
    return [(int(i) // wl.C, int(i) % wl.C) for i in idx]


def _plane_grads(t, n, c, wl, cs=None):
    cs = slice(c, c + 1) if cs is None else cs
    cw = slice(0, 1) if wl.wmode else cs
    return oracle.backward(f64(t["x"][n:n + 1, cs]), f64(t["a"][:, n:n + 1, cw]), f64(t["lam"][n:n + 1, cs]),
                           f64(t["u"][n:n + 1, cs]), f64(t["dy"][n:n + 1, cs]), wl.wmode, wl.mask)


def _check_plane(got, ref, n, c, wl, name, check_da):
    dx, da, dlam, du = got
    sl = (slice(n, n + 1), slice(c, c + 1))
    assert_close(f64(dx[sl]), ref[0], grad_tol(wl.dtype, ref[0]), f"{name} dx ({n},{c})")
    assert_close(f64(dlam[sl]), ref[2], grad_tol(wl.dtype, ref[2]), f"{name} dlam ({n},{c})")
    assert_close(f64(du[sl]), ref[3], grad_tol(wl.dtype, ref[3]), f"{name} du ({n},{c})")
    if check_da:
        assert_close(f64(da[:, n:n + 1, c:c + 1]), ref[1], grad_tol(wl.dtype, ref[1]), f"{name} da ({n},{c})")


@pytest.mark.parametrize("name", ["tiny", "classifier", "train"])
def test_full_size_per_channel(name):
    wl = gspn_inputs.WORKLOADS[name]
    t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True)
    got = g.backward(t["x"], t["a"], t["lam"], t["u"], t["dy"], wl.wmode, wl.mask)
    got2 = g.backward(t["x"], t["a"], t["lam"], t["u"], t["dy"], wl.wmode, wl.mask)
    torch.cuda.synchronize()
    for a_, b_ in zip(got, got2):
        assert torch.equal(a_, b_), "two runs differ"
    for (n, c) in _sample(wl, 6, 3):
        _check_plane(got, _plane_grads(t, n, c, wl), n, c, wl, name, True)


def test_full_size_highres_shared():
    wl = gspn_inputs.WORKLOADS["highres"]
    t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True)
    got = g.backward(t["x"], t["a"], t["lam"], t["u"], t["dy"], wl.wmode, wl.mask)
    got2 = g.backward(t["x"], t["a"], t["lam"], t["u"], t["dy"], wl.wmode, wl.mask)
    torch.cuda.synchronize()
    # the channel-summed logit gradient is a fixed-point integer sum: bitwise repeatable
    for a_, b_ in zip(got, got2):
        assert torch.equal(a_, b_), "two runs differ"
    n = 3
    ref = _plane_grads(t, n, None, wl, cs=slice(0, wl.C))     # every channel of batch item n
    dx, da, dlam, du = got
    for k, (gg, rr) in enumerate(zip((dx[n:n + 1], da[:, n:n + 1], dlam[n:n + 1], du[n:n + 1]), ref)):
        assert_close(f64(gg), rr, grad_tol(wl.dtype, rr), f"highres grad {k} of n={n}")


def test_full_size_wide_shared():
    wl = gspn_inputs.WORKLOADS["wide"]
    t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True)
    got = g.backward(t["x"], t["a"], t["lam"], t["u"], t["dy"], wl.wmode, wl.mask)
    got2 = g.backward(t["x"], t["a"], t["lam"], t["u"], t["dy"], wl.wmode, wl.mask)
    torch.cuda.synchronize()
    for a_, b_ in zip(got, got2):
        assert torch.equal(a_, b_), "two runs differ"
    del got2
    for (n, c) in _sample(wl, 3, 5):
        _check_plane(got, _plane_grads(t, n, c, wl), n, c, wl, "wide", False)
    # da: the library on a channel subset matches the oracle on that subset ...
    sub = slice(0, 4)
    ts = {k: (v[:, sub].contiguous() if k != "a" else v) for k, v in t.items()}
    gs = g.backward(ts["x"], ts["a"], ts["lam"], ts["u"], ts["dy"], wl.wmode, wl.mask)
    torch.cuda.synchronize()
    ref = _plane_grads(t, 0, None, wl, cs=sub)
    assert_close(f64(gs[1]), ref[1], grad_tol(wl.dtype, ref[1]), "wide da on 4 channels")
    # ... and the full-size da is the sum of the da of disjoint channel groups
    parts = None
    for lo in range(0, wl.C, 288):
        s2 = slice(lo, lo + 288)
        tp = {k: (v[:, s2].contiguous() if k != "a" else v) for k, v in t.items()}
        dap = g.backward(tp["x"], tp["a"], tp["lam"], tp["u"], tp["dy"], wl.wmode, wl.mask)[1].float()
        parts = dap if parts is None else parts + dap
    torch.cuda.synchronize()
    full = got[1].float()
    err = (full - parts).abs().max().item()
    assert err <= 2e-2 * full.abs().max().item(), f"da additivity {err}"
