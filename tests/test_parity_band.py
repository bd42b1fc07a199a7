"""The band family (GSPN_ALGO_BAND: 1024 x 1024 maps, all four directions): checkpointed
top->bottom and left->right scans, then bottom->top and right->left scans that recompute the
opposite direction band by band from the checkpoints. Compared with the float64 oracle plane by
plane, and with the direction-by-direction sweeps on the same inputs; both storage dtypes and
weight modes, more planes than resident CTAs, and extreme logits."""

import numpy as np
import pytest
import torch

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
import oracle

from _cases import assert_close, f64, fwd_tol

pytestmark = pytest.mark.gpu


def _oracle_planes(t, planes, wmode, mask=15):
    out = []
    for (n, c) in planes:
        cw = 0 if wmode else c
        out.append(oracle.forward(f64(t["x"][n:n + 1, c:c + 1]), f64(t["a"][:, n:n + 1, cw:cw + 1]),
                                  f64(t["lam"][n:n + 1, c:c + 1]), f64(t["u"][n:n + 1, c:c + 1]), wmode, mask))
    return out


def _sweep(t, wmode):
    y = g.forward(t["x"], t["a"], t["lam"], t["u"], wmode, 15, algo=g.ALGO_SWEEP)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_band_every_plane(wmode, dtype):
    wl = gspn_inputs.small_case(1, 3, 1024, 1024, mask=15, wmode=wmode, dtype=dtype, a_std=1.5, seed=41 + wmode)
    t = gspn_inputs.make_inputs(wl, device="cuda")
    y = g.forward(t["x"], t["a"], t["lam"], t["u"], wmode, 15, algo=g.ALGO_BAND)
    torch.cuda.synchronize()
    planes = [(0, c) for c in range(3)]
    for (n, c), ref in zip(planes, _oracle_planes(t, planes, wmode)):
        assert_close(f64(y[n:n + 1, c:c + 1]), ref, fwd_tol(dtype, ref), f"band plane ({n},{c})")
    ys = _sweep(t, wmode)
    m = ys.float().abs().max().item()
    tol = (1e-5 * max(1.0, m)) if dtype == "f32" else 2e-2 * m
    assert (y.float() - ys.float()).abs().max().item() <= tol


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_band_many_planes_per_cta(dtype):
    """More planes than resident CTAs: every CTA carries its cursors, staging blocks and
    checkpoint buffers from plane to plane."""
    wl = gspn_inputs.small_case(3, 110, 1024, 1024, mask=15, wmode=1, dtype=dtype, seed=8)
    t = gspn_inputs.make_inputs(wl, device="cuda")
    y = g.forward(t["x"], t["a"], t["lam"], t["u"], 1, 15, algo=g.ALGO_BAND)
    y2 = g.forward(t["x"], t["a"], t["lam"], t["u"], 1, 15, algo=g.ALGO_BAND)
    torch.cuda.synchronize()
    assert torch.equal(y, y2), "two runs differ"
    rng = np.random.default_rng(3)
    idx = rng.choice(3 * 110, size=6, replace=False)
    idx = sorted(set(int(i) for i in idx) | {0, 3 * 110 - 1, 148, 149})
    planes = [(i // 110, i % 110) for i in idx]
    for (n, c), ref in zip(planes, _oracle_planes(t, planes, 1)):
        assert_close(f64(y[n:n + 1, c:c + 1]), ref, fwd_tol(dtype, ref), f"band plane ({n},{c})")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("lo,hi", [(-60.0, 60.0), (-60.0, -41.0)])
def test_band_extreme_logits(dtype, lo, hi):
    gen = torch.Generator(device="cuda").manual_seed(13)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    shape = (1, 2, 1024, 1024)
    x = torch.randn(shape, device="cuda", generator=gen).to(dt)
    a = (torch.rand(4, 1, 2, 3, 1024, 1024, device="cuda", generator=gen) * (hi - lo) + lo).to(dt)
    lam = torch.rand(shape, device="cuda", generator=gen).to(dt)
    u = torch.randn(shape, device="cuda", generator=gen).to(dt)
    y = g.forward(x, a, lam, u, 0, 15, algo=g.ALGO_BAND)
    torch.cuda.synchronize()
    ref = oracle.forward(f64(x), f64(a), f64(lam), f64(u), 0, 15)
    assert_close(f64(y), ref, fwd_tol(dtype, ref), f"band extreme logits [{lo}, {hi}]")


def test_band_declines_what_it_does_not_run():
    assert g.selected_algo(g.make_desc(1, 2, 1024, 1024, 1, 15, g.F32, g.ALGO_BAND)) == g.ALGO_BAND
    assert g.selected_algo(g.make_desc(1, 2, 1024, 1024, 1, 15, g.F32, g.ALGO_BAND), True) == -1   # forward only
    assert g.selected_algo(g.make_desc(1, 2, 512, 1024, 1, 15, g.F32, g.ALGO_BAND)) == -1
    assert g.selected_algo(g.make_desc(1, 2, 1024, 1024, 1, 7, g.F32, g.ALGO_BAND)) == -1
    assert g.selected_algo(g.make_desc(1, 2, 1024, 1024, 1, 15, g.F32, g.ALGO_BAND, chunk=8)) == -1
    assert g.selected_algo(g.make_desc(1, 2, 1024, 1024, 1, 15, g.F32)) == g.ALGO_SWEEP   # AUTO
