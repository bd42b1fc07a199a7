"""Extreme logits in the fast kernel families, against the float64 oracle.

The plane and sweep families form weights with the MUFU exponential and reciprocal on logits
clamped at -40; a row whose in-range logits fall below that is redone with the max-shifted
log-sigmoid form (behind a warp vote in the plane kernels, per element in the weight-table
kernel). Logits drawn uniformly in [-60, 60] mix both paths within a warp; logits all in
[-60, -41] send every row through the shifted form. Both storage dtypes, both weight modes and
every single direction plus all four are compared element by element at the contract
tolerances, on maps that span several warps and tiles (the 1024-lane fixed-width sweep and a
56 x 56 plane)."""
import pytest
import torch

import linear_spatial_propagation_gspn_b200 as g
import oracle

from _cases import assert_close, f64, fwd_tol

pytestmark = pytest.mark.gpu


def _inputs(shape, wmode, mask, dtype, lo, hi, seed):
    N, C, H, W = shape
    D = bin(mask).count("1")
    Cw = 1 if wmode == g.SHARED else C
    gen = torch.Generator(device="cuda").manual_seed(seed)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    x = torch.randn(shape, device="cuda", generator=gen).to(dt)
    a = (torch.rand(D, N, Cw, 3, H, W, device="cuda", generator=gen) * (hi - lo) + lo).to(dt)
    lam = torch.rand(shape, device="cuda", generator=gen).to(dt)
    u = torch.randn(shape, device="cuda", generator=gen).to(dt)
    return x, a, lam, u


CASES = [((2, 3, 64, 1024), g.ALGO_SWEEP), ((2, 3, 1024, 64), g.ALGO_SWEEP), ((2, 3, 56, 56), g.ALGO_PLANE),
         ((2, 3, 64, 64), g.ALGO_PLANE)]


@pytest.mark.parametrize("shape,algo", CASES)
@pytest.mark.parametrize("mask", [15, 1, 2, 4, 8])
@pytest.mark.parametrize("wmode", [g.PER_CHANNEL, g.SHARED])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("lo,hi", [(-60.0, 60.0), (-60.0, -41.0)])
def test_extreme_logits(shape, algo, mask, wmode, dtype, lo, hi):
    x, a, lam, u = _inputs(shape, wmode, mask, dtype, lo, hi, seed=int(hi) + 7 * mask + 3 * wmode)
    desc = g.desc_for(x, wmode, mask, algo)
    assert g.selected_algo(desc) == algo
    y = g.forward(x, a, lam, u, wmode, mask, algo=algo)
    torch.cuda.synchronize()
    ref = oracle.forward(f64(x), f64(a), f64(lam), f64(u), wmode, mask)
    assert_close(f64(y), ref, fwd_tol(dtype, ref), f"extreme logits [{lo}, {hi}] algo={algo} mask={mask}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("wmode", [g.PER_CHANNEL, g.SHARED])
def test_extreme_logits_backward(dtype, wmode):
    """The plane backward's gradient pass (MUFU sigmoid, argument clamped) and the generic
    backward on logits in [-60, 60]."""
    shape = (1, 2, 24, 40)
    x, a, lam, u = _inputs(shape, wmode, 15, dtype, -60.0, 60.0, seed=91 + wmode)
    gen = torch.Generator(device="cuda").manual_seed(5)
    dy = torch.randn(shape, device="cuda", generator=gen).to(x.dtype)
    got = g.backward(x, a, lam, u, dy, wmode, 15)
    torch.cuda.synchronize()
    ref = oracle.backward(f64(x), f64(a), f64(lam), f64(u), f64(dy), wmode, 15)
    from _cases import grad_tol
    for name, gg, rr in zip(("dx", "da", "dlam", "du"), got, ref):
        assert_close(f64(gg), rr, grad_tol(dtype, rr), f"extreme backward {name}")
