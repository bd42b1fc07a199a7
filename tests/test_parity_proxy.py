"""Compressive channel proxy (projection, propagation in proxy space, projection back) against the
float64 oracle: both storage dtypes, scans on the plane and sweep families, a chunked variant,
and argument validation."""
import numpy as np
import pytest
import torch

import linear_spatial_propagation_gspn_b200 as g
import oracle

from _cases import assert_close, f64, fwd_tol

pytestmark = pytest.mark.gpu


def _inputs(N, C, Cp, H, W, mask, wmode, dtype, seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    D = bin(mask).count("1")
    Cw = 1 if wmode else Cp

    def rn(*shape, scale=1.0):
        return (torch.randn(*shape, generator=gen, device="cuda") * scale).to(dt)

    x = rn(N, C, H, W)
    p_in = rn(Cp, C, scale=1.0 / np.sqrt(C))
    p_out = rn(C, Cp, scale=1.0 / np.sqrt(Cp))
    a = rn(D, N, Cw, 3, H, W)
    lam = torch.rand(N, Cp, H, W, generator=gen, device="cuda").to(dt)
    u = rn(N, Cp, H, W)
    return x, p_in, a, lam, u, p_out


@pytest.mark.parametrize("shape", [(2, 16, 4, 40, 48), (1, 24, 8, 64, 1024), (1, 96, 12, 56, 56)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("wmode", [0, 1])
def test_proxy_forward(shape, dtype, wmode):
    N, C, Cp, H, W = shape
    x, p_in, a, lam, u, p_out = _inputs(N, C, Cp, H, W, 15, wmode, dtype, seed=sum(shape) + wmode)
    y = g.proxy_forward(x, p_in, a, lam, u, p_out, wmode, 15)
    torch.cuda.synchronize()
    ref = oracle.proxy_forward(f64(x), f64(p_in), f64(a), f64(lam), f64(u), f64(p_out), wmode, 15)
    assert_close(f64(y), ref, fwd_tol(dtype, ref), f"proxy {shape} {dtype}")


@pytest.mark.parametrize("chunk", [4, 16])
def test_proxy_forward_chunked(chunk):
    x, p_in, a, lam, u, p_out = _inputs(1, 32, 8, 48, 64, 15, 1, "f32", seed=chunk)
    y = g.proxy_forward(x, p_in, a, lam, u, p_out, 1, 15, chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle.proxy_forward(f64(x), f64(p_in), f64(a), f64(lam), f64(u), f64(p_out), 1, 15, chunk=chunk)
    assert_close(f64(y), ref, fwd_tol("f32", ref), f"proxy chunk {chunk}")


def test_proxy_rejects_bad_shapes():
    x, p_in, a, lam, u, p_out = _inputs(1, 8, 2, 16, 16, 15, 1, "f32", seed=1)
    with pytest.raises(ValueError):
        g.proxy_forward(x, p_out, a, lam, u, p_in, 1, 15)


# bf16 shapes whose projections run on the tensor cores (C, C_proxy and H*W multiples of 8):
# several pixel tiles and a ragged last one, output-row tiles with padding (C_proxy 24 -> 32 rows,
# 1152 -> 5 tiles of 240), contraction lengths below, at and far above one 64-wide stage, and
# more than one batch item.
TC_SHAPES = [(1, 24, 8, 64, 1024), (2, 64, 16, 32, 40), (1, 256, 48, 16, 72), (2, 320, 24, 8, 24),
             (1, 1152, 144, 16, 64), (3, 136, 64, 24, 24)]


@pytest.mark.parametrize("shape", TC_SHAPES)
@pytest.mark.parametrize("wmode", [0, 1])
def test_proxy_tensor_core_projections(shape, wmode):
    N, C, Cp, H, W = shape
    x, p_in, a, lam, u, p_out = _inputs(N, C, Cp, H, W, 15, wmode, "bf16", seed=3 * sum(shape) + wmode)
    y = g.proxy_forward(x, p_in, a, lam, u, p_out, wmode, 15)
    torch.cuda.synchronize()
    ref = oracle.proxy_forward(f64(x), f64(p_in), f64(a), f64(lam), f64(u), f64(p_out), wmode, 15)
    assert_close(f64(y), ref, fwd_tol("bf16", ref), f"proxy tensor-core {shape}")
    y2 = g.proxy_forward(x, p_in, a, lam, u, p_out, wmode, 15)
    torch.cuda.synchronize()
    assert torch.equal(y, y2), "two runs differ"
