"""libgspn's small-map (plane) kernels against the float64 oracle.

Forced-plane cases cover odd sizes, single rows/columns, every direction mask, both weight modes
and both storage dtypes. The classifier-stage (56x56, bf16), training (64x64, fp32) and tiny
(16x16, TB only) workloads run at full size in the launch configuration the benchmark uses;
the oracle checks seeded sample planes (every output plane depends only on its own inputs)."""
import numpy as np
import pytest
import torch

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
import oracle
from gspn_inputs import small_case

from _cases import assert_close, check_forward, f64, fwd_tol

pytestmark = pytest.mark.gpu

# fp32 maps whose rows are a multiple of 4 run the concurrent-direction forward (17 lines are not a
# whole number of 4-line strips; 1 x 8 and 3 x 8 are single-lane and single-line scans; 100 x 16
# and 60 x 96 use 4 lanes per thread); bf16 maps and the other shapes run the direction-serial one
SHAPES = [(1, 4, 16, 16), (2, 3, 17, 33), (1, 2, 1, 5), (1, 2, 5, 1), (2, 2, 31, 7), (1, 1, 64, 40), (1, 1, 1, 1),
          (2, 2, 56, 56), (1, 1, 128, 3), (3, 1, 33, 128), (2, 3, 17, 40), (2, 3, 17, 36), (1, 2, 1, 8),
          (1, 1, 3, 8), (1, 2, 100, 16), (2, 1, 60, 96)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mask", [15, 1, 2, 4, 8, 6, 9])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_plane_forward_small(shape, mask, wmode, dtype):
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=5 * sum(shape) + mask)
    d = g.make_desc(*shape, wmode, mask, 0 if dtype == "f32" else 1, g.ALGO_PLANE)
    assert g.selected_algo(d) == g.ALGO_PLANE
    check_forward(wl, g.ALGO_PLANE)


@pytest.mark.parametrize("name", ["tiny", "classifier", "train"])
def test_full_size_sampled_planes(name):
    wl = gspn_inputs.WORKLOADS[name]
    d = g.make_desc(wl.N, wl.C, wl.H, wl.W, wl.wmode, wl.mask, 0 if wl.dtype == "f32" else 1)
    assert g.selected_algo(d) == g.ALGO_PLANE
    t = gspn_inputs.make_inputs(wl, device="cuda")
    y = g.forward(t["x"], t["a"], t["lam"], t["u"], wl.wmode, wl.mask)
    y2 = g.forward(t["x"], t["a"], t["lam"], t["u"], wl.wmode, wl.mask)
    torch.cuda.synchronize()
    assert torch.equal(y, y2), "two runs differ"
    rng = np.random.default_rng(7)
    idx = rng.choice(wl.N * wl.C, size=min(12, wl.N * wl.C), replace=False)
    for i in idx:
        n, c = int(i) // wl.C, int(i) % wl.C
        cw = 0 if wl.wmode else c
        ref = oracle.forward(f64(t["x"][n:n + 1, c:c + 1]), f64(t["a"][:, n:n + 1, cw:cw + 1]),
                             f64(t["lam"][n:n + 1, c:c + 1]), f64(t["u"][n:n + 1, c:c + 1]), wl.wmode, wl.mask)
        assert_close(f64(y[n:n + 1, c:c + 1]), ref, fwd_tol(wl.dtype, ref), f"{name} plane ({n},{c})")


def test_plane_matches_generic():
    wl = small_case(4, 5, 48, 40, mask=15, wmode=0, dtype="f32", seed=12)
    t = gspn_inputs.make_inputs(wl, device="cuda")
    yp = g.forward(t["x"], t["a"], t["lam"], t["u"], 0, 15, algo=g.ALGO_PLANE)
    yg = g.forward(t["x"], t["a"], t["lam"], t["u"], 0, 15, algo=g.ALGO_GENERIC)
    torch.cuda.synchronize()
    assert (yp - yg).abs().max().item() <= 1e-5 * max(1.0, yg.abs().max().item())
