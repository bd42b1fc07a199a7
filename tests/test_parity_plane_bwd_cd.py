"""The plane backward with the four directions scanned concurrently (fp32 storage, per-channel
weights, rows a multiple of 4): each direction's warp recomputes its h plane and runs its reverse
scan into a delta plane of its own; the logit gradients and dx, dlambda, du are then formed from
those planes. Compared element by element with the float64 oracle's backward over odd heights,
single lines and lanes, 2 and 4 lanes per thread, every direction mask, local chunks and extreme
logits; two runs must agree bit for bit (the per-direction planes are summed in a fixed order)."""
import pytest
import torch

import linear_spatial_propagation_gspn_b200 as g
import oracle
from gspn_inputs import make_inputs, small_case

from _cases import assert_close, check_backward, f64, grad_tol

pytestmark = pytest.mark.gpu

SHAPES = [(2, 3, 17, 36), (1, 2, 1, 8), (1, 1, 3, 8), (1, 2, 100, 16), (2, 1, 60, 96), (3, 2, 64, 64),
          (1, 4, 16, 16), (2, 2, 33, 12)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mask", [15, 1, 2, 4, 8, 3, 12, 5, 10, 6, 9, 14])
def test_plane_backward_concurrent(shape, mask):
    wl = small_case(*shape, mask=mask, wmode=0, dtype="f32", seed=13 * sum(shape) + mask)
    d = g.make_desc(*shape, 0, mask, g.F32, g.ALGO_PLANE)
    assert g.selected_algo(d, True) == g.ALGO_PLANE
    check_backward(wl, g.ALGO_PLANE)


@pytest.mark.parametrize("chunk", [1, 3, 8, 17])
@pytest.mark.parametrize("mask", [15, 2, 8])
def test_plane_backward_concurrent_chunked(chunk, mask):
    wl = small_case(2, 2, 24, 40, mask=mask, wmode=0, dtype="f32", seed=chunk + mask)
    check_backward(wl, g.ALGO_PLANE, chunk=chunk)


def test_plane_backward_concurrent_extreme_logits_and_repeatable():
    shape = (2, 3, 48, 64)
    gen = torch.Generator(device="cuda").manual_seed(29)
    x = torch.randn(shape, device="cuda", generator=gen)
    a = torch.rand(4, 2, 3, 3, 48, 64, device="cuda", generator=gen) * 120 - 60
    lam = torch.rand(shape, device="cuda", generator=gen)
    u = torch.randn(shape, device="cuda", generator=gen)
    dy = torch.randn(shape, device="cuda", generator=gen)
    got = g.backward(x, a, lam, u, dy, 0, 15, algo=g.ALGO_PLANE)
    again = g.backward(x, a, lam, u, dy, 0, 15, algo=g.ALGO_PLANE)
    torch.cuda.synchronize()
    ref = oracle.backward(f64(x), f64(a), f64(lam), f64(u), f64(dy), 0, 15)
    for name, gg, g2, rr in zip(("dx", "da", "dlam", "du"), got, again, ref):
        assert torch.equal(gg, g2), f"{name}: two runs differ"
        assert_close(f64(gg), rr, grad_tol("f32", rr), f"extreme logits {name}")
