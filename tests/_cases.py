"""Shared helpers for the GPU parity tests: run libgspn and the float64 oracle on the same
seeded inputs and compare with the tolerances of the library's contract:
  fp32 forward:  max|d| <= 1e-5 * max(1, max|ref|)
  bf16 forward:  max|d| <= 2e-2 * max|ref|   (oracle on the same bf16-rounded inputs)
  gradients:     max|d| <= 1e-4 * max(1, max|ref grad|) per tensor (fp32), 2e-2 * max|ref| (bf16)
"""
import numpy as np
import torch

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
import oracle

TOL_F32 = 1e-5
TOL_BF16 = 2e-2
TOL_GRAD_F32 = 1e-4


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def fwd_tol(dtype, ref):
    m = float(np.abs(ref).max()) if ref.size else 0.0
    return TOL_F32 * max(1.0, m) if dtype == "f32" else TOL_BF16 * max(m, 1e-30)


def grad_tol(dtype, ref):
    m = float(np.abs(ref).max()) if ref.size else 0.0
    return TOL_GRAD_F32 * max(1.0, m) if dtype == "f32" else TOL_BF16 * max(m, 1e-30)


def assert_close(got, ref, tol, what):
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err <= tol, f"{what}: max|d| = {err:.3e} > tol {tol:.3e} (max|ref| = {np.abs(ref).max():.3e})"
    return err


def run_forward(wl, algo=g.ALGO_AUTO, inputs=None, chunk=0):
    t = inputs or gspn_inputs.make_inputs(wl, device="cuda")
    y = g.forward(t["x"], t["a"], t["lam"], t["u"], wl.wmode, wl.mask, algo=algo, chunk=chunk)
    torch.cuda.synchronize()
    return t, y


def check_forward(wl, algo=g.ALGO_AUTO, chunk=0):
    t, y = run_forward(wl, algo, chunk=chunk)
    ref = oracle.forward(f64(t["x"]), f64(t["a"]), f64(t["lam"]), f64(t["u"]), wl.wmode, wl.mask, chunk=chunk)
    return assert_close(f64(y), ref, fwd_tol(wl.dtype, ref), f"forward {wl.name} algo={algo} chunk={chunk}")


def check_backward(wl, algo=g.ALGO_AUTO, chunk=0):
    t = gspn_inputs.make_inputs(wl, device="cuda", with_dy=True)
    got = g.backward(t["x"], t["a"], t["lam"], t["u"], t["dy"], wl.wmode, wl.mask, algo=algo, chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle.backward(f64(t["x"]), f64(t["a"]), f64(t["lam"]), f64(t["u"]), f64(t["dy"]), wl.wmode, wl.mask,
                          chunk=chunk)
    errs = []
    for name, gg, rr in zip(("dx", "da", "dlam", "du"), got, ref):
        errs.append(assert_close(f64(gg), rr, grad_tol(wl.dtype, rr),
                                 f"backward {name} {wl.name} algo={algo} chunk={chunk}"))
    return errs
