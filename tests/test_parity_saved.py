"""The training pair: gspn_forward_save keeps each direction's h and gspn_backward_saved reads it
instead of recomputing the forward scans. The forward's y is the plain forward's, bit for bit; the
gradients match the float64 oracle's backward at the gradient tolerance; the pair declines what it
does not run; the autograd function uses it."""
import pytest
import torch

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
import oracle
from gspn_inputs import small_case

from _cases import assert_close, f64, fwd_tol, grad_tol

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(2, 3, 64, 64), (1, 2, 24, 40), (2, 2, 56, 56), (1, 3, 32, 96)])
@pytest.mark.parametrize("mask", [15, 6, 9, 1])
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("chunk", [0, 5])
def test_saved_pair(shape, mask, wmode, dtype, chunk):
    if dtype == "bf16" and shape[3] % 8:
        pytest.skip("bf16 rows of the concurrent forward are whole 16-byte chunks")
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=sum(shape) + mask + wmode)
    t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True, seed=mask + 7 * wmode)
    desc = g.desc_for(t["x"], wmode, mask, chunk=chunk)
    assert g.hsave_size(desc) == 4 * bin(mask).count("1") * t["x"].numel()
    y_plain = g.forward(t["x"], t["a"], t["lam"], t["u"], wmode, mask, chunk=chunk)
    y, hsave = g.forward_save(t["x"], t["a"], t["lam"], t["u"], wmode, mask, chunk=chunk)
    got = g.backward_saved(t["x"], t["a"], t["lam"], t["u"], t["dy"], hsave, wmode, mask, chunk=chunk)
    got2 = g.backward_saved(t["x"], t["a"], t["lam"], t["u"], t["dy"], hsave, wmode, mask, chunk=chunk)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain), "forward_save changed y"
    ref_y = oracle.forward(f64(t["x"]), f64(t["a"]), f64(t["lam"]), f64(t["u"]), wmode, mask, chunk=chunk)
    assert_close(f64(y), ref_y, fwd_tol(dtype, ref_y), "forward_save y")
    ref = oracle.backward(f64(t["x"]), f64(t["a"]), f64(t["lam"]), f64(t["u"]), f64(t["dy"]), wmode, mask,
                          chunk=chunk)
    for name, gg, g2, rr in zip(("dx", "da", "dlam", "du"), got, got2, ref):
        assert torch.equal(gg, g2), f"backward_saved {name}: two runs differ"
        assert_close(f64(gg), rr, grad_tol(dtype, rr), f"backward_saved {name}")


def test_saved_pair_declines():
    """Per-direction lambda / u, rows the concurrent forward does not take, and the large maps
    (sweep-family forward) do not run the pair: the size is 0 and the calls return
    GSPN_ERR_UNSUPPORTED before any launch."""
    assert g.hsave_size(g.make_desc(1, 2, 32, 32, 0, 15, g.F32, per_dir=1)) == 0
    assert g.hsave_size(g.make_desc(1, 2, 32, 30, 0, 15, g.F32)) == 0
    assert g.hsave_size(g.make_desc(1, 2, 1024, 1024, 1, 15, g.F32)) == 0
    x = torch.zeros(1, 2, 1024, 1024, device="cuda")
    a = torch.zeros(4, 1, 1, 3, 1024, 1024, device="cuda")
    with pytest.raises(g.GspnError):
        g.forward_save(x, a, x, x, 1, 15)


def test_autograd_uses_the_pair():
    wl = small_case(2, 3, 40, 48, mask=15, wmode=0, dtype="f32", seed=41)
    t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True, seed=42)
    leaves = [t[k].clone().requires_grad_(True) for k in ("x", "a", "lam", "u")]
    assert g.hsave_size(g.desc_for(t["x"], 0, 15)) > 0
    y = g.gspn(*leaves, 0, 15)
    y.backward(t["dy"])
    torch.cuda.synchronize()
    ref = oracle.backward(f64(t["x"]), f64(t["a"]), f64(t["lam"]), f64(t["u"]), f64(t["dy"]), 0, 15)
    for name, leaf, rr in zip(("dx", "da", "dlam", "du"), leaves, ref):
        assert_close(f64(leaf.grad), rr, grad_tol("f32", rr), f"autograd {name}")
