"""The end-to-end entry point from host buffers (gspn_forward_host: copies in, forward, copy of y
out, on one stream) against the float64 oracle, with shared and per-direction lambda / u."""
import pytest
import torch

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
import oracle
from gspn_inputs import small_case

from _cases import assert_close, f64, fwd_tol

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("per_dir", [0, 1])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape,mask,wmode", [((2, 3, 24, 40), 15, 0), ((1, 2, 300, 64), 9, 1)])
def test_forward_host_matches_oracle(per_dir, dtype, shape, mask, wmode):
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype=dtype, seed=sum(shape) + 17 * per_dir)
    t = gspn_inputs.make_inputs(wl, device="cpu", per_dir=bool(per_dir))
    host = {k: v.contiguous().pin_memory() for k, v in t.items()}
    hy = torch.empty_like(host["x"]).pin_memory()
    desc = g.make_desc(*shape, wmode, mask, 0 if dtype == "f32" else 1, per_dir=per_dir)
    dev = torch.empty(g.forward_host_buffer_size(desc), dtype=torch.uint8, device="cuda")
    g.forward_host(desc, host["x"], host["a"], host["lam"], host["u"], hy, dev)
    torch.cuda.synchronize()
    ref = oracle.forward(f64(t["x"]), f64(t["a"]), f64(t["lam"]), f64(t["u"]), wmode, mask, per_dir=per_dir)
    assert_close(f64(hy), ref, fwd_tol(dtype, ref), f"host path per_dir={per_dir}")
