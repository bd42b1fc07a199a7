"""libgspn's line-sweep kernels (large maps) against the float64 oracle.

Small forced-sweep cases cover both horizontal schemes (lane-major hand-over when both axes give
16-byte rows, column tiles otherwise), ragged staging blocks (scan lengths that are not a
multiple of the staging block), single-step scans, several planes per CTA, every direction mask
and both weight modes and dtypes. The two 1024x1024
workloads run at full size in the launch configuration the benchmark times; the oracle checks
seeded sample planes one by one (each output plane depends only on its own x, lambda, u and its
logits)."""
import numpy as np
import pytest
import torch

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
import oracle
from gspn_inputs import small_case

from _cases import assert_close, check_forward, f64, fwd_tol

pytestmark = pytest.mark.gpu

SHAPES = [(2, 3, 64, 64), (1, 2, 37, 40), (1, 1, 300, 16), (1, 2, 5, 8), (2, 1, 1, 8), (1, 1, 257, 24), (1, 2, 8, 1024),
          (1, 2, 40, 24), (2, 1, 72, 2048)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mask", [15, 1, 2, 4, 8, 5, 10, 6, 9, 12, 3])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sweep_forward_small(shape, mask, wmode, dtype):
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=3 * sum(shape) + mask)
    d = g.make_desc(*shape, wmode, mask, 0 if dtype == "f32" else 1, g.ALGO_SWEEP)
    assert g.selected_algo(d) == g.ALGO_SWEEP
    check_forward(wl, g.ALGO_SWEEP)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sweep_many_planes_per_cta(dtype):
    """More planes than resident CTAs: every CTA runs several planes through the same staging
    buffers and hand-off barriers."""
    wl = small_case(40, 40, 16, 16, mask=15, wmode=0, dtype=dtype, seed=17)
    check_forward(wl, g.ALGO_SWEEP)


@pytest.mark.parametrize("shape", [(1, 3, 64, 1024), (1, 2, 1024, 64), (3, 40, 32, 1024)])
@pytest.mark.parametrize("mask", [15, 1, 2, 5, 10, 12, 3])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sweep_fixed_width_lines(shape, mask, wmode, dtype):
    """1024-lane lines (the fixed-width kernel): vertical scans of 1024-wide maps, horizontal
    scans of 1024-high maps, and more planes than resident CTAs."""
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=5 * sum(shape) + mask)
    check_forward(wl, g.ALGO_SWEEP)


def test_sweep_matches_generic_bitwise_close():
    wl = small_case(2, 2, 96, 128, mask=15, wmode=1, dtype="f32", seed=9)
    t = gspn_inputs.make_inputs(wl, device="cuda")
    ys = g.forward(t["x"], t["a"], t["lam"], t["u"], 1, 15, algo=g.ALGO_SWEEP)
    yg = g.forward(t["x"], t["a"], t["lam"], t["u"], 1, 15, algo=g.ALGO_GENERIC)
    torch.cuda.synchronize()
    assert (ys - yg).abs().max().item() <= 1e-5 * max(1.0, yg.abs().max().item())


def _sample_planes(wl, k, seed):
    rng = np.random.default_rng(seed)
    idx = rng.choice(wl.N * wl.C, size=min(k, wl.N * wl.C), replace=False)
    return [(int(i) // wl.C, int(i) % wl.C) for i in idx]


@pytest.mark.parametrize("name", ["highres", "wide"])
def test_full_size_sampled_planes(name):
    wl = gspn_inputs.WORKLOADS[name]
    d = g.make_desc(wl.N, wl.C, wl.H, wl.W, wl.wmode, wl.mask, 0 if wl.dtype == "f32" else 1)
    assert g.selected_algo(d) == g.ALGO_SWEEP
    t = gspn_inputs.make_inputs(wl, device="cuda")
    y = g.forward(t["x"], t["a"], t["lam"], t["u"], wl.wmode, wl.mask)
    y2 = g.forward(t["x"], t["a"], t["lam"], t["u"], wl.wmode, wl.mask)
    torch.cuda.synchronize()
    assert torch.equal(y, y2), "two runs differ"
    for (n, c) in _sample_planes(wl, 8, 123):
        cw = 0 if wl.wmode else c
        ref = oracle.forward(f64(t["x"][n:n + 1, c:c + 1]), f64(t["a"][:, n:n + 1, cw:cw + 1]),
                             f64(t["lam"][n:n + 1, c:c + 1]), f64(t["u"][n:n + 1, c:c + 1]), wl.wmode, wl.mask)
        assert_close(f64(y[n:n + 1, c:c + 1]), ref, fwd_tol(wl.dtype, ref), f"{name} plane ({n},{c})")
