"""Per-direction lambda and u (y = sum_d u_d * h^d(lam_d x)) against the float64 oracle: the
generic family forward and backward, the plane family forward, both weight modes and dtypes,
with and without local chunks; the sweep family declines the mode and AUTO falls back."""
import pytest
import torch

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
import oracle
from gspn_inputs import small_case

from _cases import assert_close, f64, fwd_tol, grad_tol

pytestmark = pytest.mark.gpu


def _inputs(wl, seed):
    t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True, seed=seed, per_dir=True)
    return t["x"], t["a"], t["lam"], t["u"], t["dy"]


@pytest.mark.parametrize("algo", [g.ALGO_GENERIC, g.ALGO_PLANE])
@pytest.mark.parametrize("shape", [(2, 3, 24, 40), (1, 2, 17, 33)])
@pytest.mark.parametrize("mask", [15, 6, 1])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("chunk", [0, 5])
def test_per_direction_forward(algo, shape, mask, wmode, dtype, chunk):
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=sum(shape) + mask)
    x, a, lam, u, _ = _inputs(wl, seed=mask + chunk)
    y = g.forward(x, a, lam, u, wmode, mask, algo=algo, chunk=chunk, per_dir=1)
    torch.cuda.synchronize()
    ref = oracle.forward(f64(x), f64(a), f64(lam), f64(u), wmode, mask, chunk=chunk, per_dir=1)
    assert_close(f64(y), ref, fwd_tol(dtype, ref), f"per-direction forward algo={algo}")


@pytest.mark.parametrize("shape", [(1, 2, 19, 21), (2, 1, 8, 33)])
@pytest.mark.parametrize("mask", [15, 5])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("chunk", [0, 4])
def test_per_direction_backward(shape, mask, wmode, chunk):
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype="f32", seed=7 * sum(shape) + mask)
    x, a, lam, u, dy = _inputs(wl, seed=3 + mask + chunk)
    got = g.backward(x, a, lam, u, dy, wmode, mask, chunk=chunk, per_dir=1)
    torch.cuda.synchronize()
    ref = oracle.backward(f64(x), f64(a), f64(lam), f64(u), f64(dy), wmode, mask, chunk=chunk, per_dir=1)
    for name, gg, rr in zip(("dx", "da", "dlam", "du"), got, ref):
        assert_close(f64(gg), rr, grad_tol("f32", rr), f"per-direction backward {name}")


def test_per_direction_selection():
    """The sweep family declines per-direction lambda / u; AUTO runs large maps on the generic
    family, small maps on the plane family (forward) and the generic one (backward)."""
    big = g.make_desc(1, 2, 256, 256, 1, 15, g.F32, per_dir=1)
    assert g.selected_algo(big) == g.ALGO_GENERIC
    assert g.selected_algo(g.make_desc(1, 2, 256, 256, 1, 15, g.F32, g.ALGO_SWEEP, per_dir=1)) == -1
    small = g.make_desc(1, 2, 32, 32, 0, 15, g.F32, per_dir=1)
    assert g.selected_algo(small) == g.ALGO_PLANE
    assert g.selected_algo(small, True) == g.ALGO_GENERIC


def test_per_direction_large_map_forward():
    wl = small_case(1, 2, 256, 128, mask=15, wmode=1, dtype="f32", seed=11)
    x, a, lam, u, _ = _inputs(wl, seed=12)
    y = g.forward(x, a, lam, u, 1, 15, per_dir=1)
    torch.cuda.synchronize()
    ref = oracle.forward(f64(x), f64(a), f64(lam), f64(u), 1, 15, per_dir=1)
    assert_close(f64(y), ref, fwd_tol("f32", ref), "per-direction large map")


@pytest.mark.parametrize("shape,mask,wmode,dtype", [((1, 2, 1024, 1024), 15, 1, "f32"),
                                                    ((2, 1, 96, 1024), 9, 0, "f32"),
                                                    ((1, 2, 128, 264), 15, 0, "bf16")])
def test_per_direction_large_map_backward(shape, mask, wmode, dtype):
    """The large-map backward (all directions at once, horizontal directions on transposed copies
    of x, dy and each direction's lam / u) with per-direction lam / u, against the oracle's
    backward: a full 1024 x 1024 map, a map wider than tall with a subset of directions, bf16."""
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=sum(shape) + mask)
    x, a, lam, u, dy = _inputs(wl, seed=5 + mask)
    got = g.backward(x, a, lam, u, dy, wmode, mask, per_dir=1)
    again = g.backward(x, a, lam, u, dy, wmode, mask, per_dir=1)
    torch.cuda.synchronize()
    ref = oracle.backward(f64(x), f64(a), f64(lam), f64(u), f64(dy), wmode, mask, per_dir=1)
    for name, gg, g2, rr in zip(("dx", "da", "dlam", "du"), got, again, ref):
        assert torch.equal(gg, g2), f"per-direction large-map backward {name}: two runs differ"
        assert_close(f64(gg), rr, grad_tol(dtype, rr), f"per-direction large-map backward {name}")
