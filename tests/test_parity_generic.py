"""libgspn's any-shape (generic) kernels against the float64 oracle on small seeded cases
spanning odd sizes, single lanes/steps, every weight mode, several direction masks and both
storage dtypes."""
import pytest

from gspn_inputs import small_case
import linear_spatial_propagation_gspn_b200 as g

from _cases import check_backward, check_forward

pytestmark = pytest.mark.gpu

SHAPES = [(1, 4, 16, 16), (2, 3, 17, 33), (1, 2, 1, 5), (1, 2, 5, 1), (2, 2, 31, 7), (1, 1, 64, 40), (1, 1, 1, 1)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mask", [1, 15, 6, 9])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_generic_forward(shape, mask, wmode, dtype):
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=sum(shape) + mask)
    check_forward(wl, g.ALGO_GENERIC)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mask", [1, 15, 10])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_generic_backward(shape, mask, wmode, dtype):
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=7 * sum(shape) + mask)
    check_backward(wl, g.ALGO_GENERIC)


def test_generic_extreme_logits():
    """Logits in [-60, 60] take the max-shifted weight path: finite and within tolerance."""
    import torch
    import numpy as np
    import oracle
    from _cases import f64, assert_close, fwd_tol
    wl = small_case(1, 2, 12, 12, mask=15, wmode=0, dtype="f32", seed=5)
    gen = torch.Generator(device="cuda").manual_seed(11)
    x = torch.randn(1, 2, 12, 12, device="cuda", generator=gen)
    a = (torch.rand(4, 1, 2, 3, 12, 12, device="cuda", generator=gen) * 120 - 60)
    lam = torch.rand(1, 2, 12, 12, device="cuda", generator=gen)
    u = torch.randn(1, 2, 12, 12, device="cuda", generator=gen)
    y = g.forward(x, a, lam, u, 0, 15, algo=g.ALGO_GENERIC)
    ref = oracle.forward(f64(x), f64(a), f64(lam), f64(u), 0, 15)
    assert_close(f64(y), ref, fwd_tol("f32", ref), "extreme logits")
