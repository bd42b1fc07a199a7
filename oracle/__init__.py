"""Float64 CPU oracle of the GSPN 4-direction line-scan propagation.

TEST INFRASTRUCTURE ONLY. The oracle is what the CUDA library is checked against. Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` / reference legs
may import it. It shares no code with the CUDA library (``linear_spatial_propagation_gspn_b200``)
and neither imports the other.

Two independent implementations live here:

* ``gspn_oracle.c`` (loaded through ctypes): the recurrence, in the scan order the pages
  describe ("GSPN-2: Efficient Parallel Sequence Modeling" paper notes, section
  "2D spatial propagation review"), forward and backward.
* ``brute.py``: the closed form ``H = G X`` with ``G`` block lower-triangular whose blocks are
  products of the per-line propagation matrices (same notes, the linear-attention reading at
  the end of "Optimisation 2: compact channel propagation"). Written with NumPy matrices and
  no shared code with the C file, so the two check each other.

Every function takes/returns float64 NumPy arrays in the layouts documented in
``gspn_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gspn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DIR_TB, DIR_BT, DIR_LR, DIR_RL = 1, 2, 4, 8
DIRS = (DIR_TB, DIR_BT, DIR_LR, DIR_RL)


def build(force: bool = False) -> str:
    """Compile ``gspn_oracle.c`` into ``liboracle.so`` (plain gcc, IEEE float64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        args = [ctypes.c_int] * 5 + [ctypes.c_uint]
        lib.gspn_ref_forward.argtypes = args + [dp] * 5
        lib.gspn_ref_forward.restype = ctypes.c_int
        lib.gspn_ref_backward.argtypes = args + [dp] * 9
        lib.gspn_ref_backward.restype = ctypes.c_int
        lib.gspn_ref_forward_ex.argtypes = args + [ctypes.c_int, ctypes.c_int] + [dp] * 5
        lib.gspn_ref_forward_ex.restype = ctypes.c_int
        lib.gspn_ref_backward_ex.argtypes = args + [ctypes.c_int, ctypes.c_int] + [dp] * 9
        lib.gspn_ref_backward_ex.restype = ctypes.c_int
        if lib.gspn_ref_abi_version() != 3:
            raise RuntimeError("stale oracle build; rebuild with oracle.build(force=True)")
        _lib = lib
    return _lib


def popcount(mask: int) -> int:
    return bin(mask & 15).count("1")


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check_shapes(x, a, lam, u, wmode, mask, per_dir=0):
    N, C, H, W = x.shape
    Cw = 1 if wmode else C
    want_a = (popcount(mask), N, Cw, 3, H, W)
    if a.shape != want_a:
        raise ValueError(f"logits shape {a.shape}, expected {want_a}")
    want_lu = ((popcount(mask),) if per_dir else ()) + x.shape
    if lam.shape != want_lu or u.shape != want_lu:
        raise ValueError(f"lam and u must be {want_lu}")
    return N, C, H, W


def forward(x, a, lam, u, wmode: int = 0, mask: int = 15, chunk: int = 0, per_dir: int = 0) -> np.ndarray:
    """y = u * sum_{d in mask} h^d, float64. ``wmode`` 0 = per-channel, 1 = shared; ``chunk``
    > 0: local propagation within image-aligned chunks of that many lines (0 = global);
    ``per_dir`` = 1: lam and u have a direction axis and y = sum_d u_d * h^d(lam_d x)."""
    x, a, lam, u = _f64(x), _f64(a), _f64(lam), _f64(u)
    N, C, H, W = _check_shapes(x, a, lam, u, wmode, mask, per_dir)
    y = np.empty_like(x)
    rc = _load().gspn_ref_forward_ex(N, C, H, W, int(wmode), int(mask), int(chunk), int(per_dir), _ptr(x), _ptr(a),
                                     _ptr(lam), _ptr(u), _ptr(y))
    if rc:
        raise RuntimeError(f"gspn_ref_forward failed ({rc})")
    return y


def backward(x, a, lam, u, dy, wmode: int = 0, mask: int = 15, chunk: int = 0, per_dir: int = 0):
    """Returns (dx, da, dlam, du), float64, for the loss sum(dy * y)."""
    x, a, lam, u, dy = _f64(x), _f64(a), _f64(lam), _f64(u), _f64(dy)
    N, C, H, W = _check_shapes(x, a, lam, u, wmode, mask, per_dir)
    if dy.shape != x.shape:
        raise ValueError("dy must have the shape of x")
    dx, dlam, du = np.empty_like(x), np.empty_like(lam), np.empty_like(u)
    da = np.empty_like(a)
    rc = _load().gspn_ref_backward_ex(N, C, H, W, int(wmode), int(mask), int(chunk), int(per_dir), _ptr(x), _ptr(a),
                                      _ptr(lam), _ptr(u), _ptr(dy), _ptr(dx), _ptr(da), _ptr(dlam), _ptr(du))
    if rc:
        raise RuntimeError(f"gspn_ref_backward failed ({rc})")
    return dx, da, dlam, du


def proxy_forward(x, p_in, a, lam, u, p_out, wmode: int = 1, mask: int = 15, chunk: int = 0) -> np.ndarray:
    """Compressive channel proxy ("GSPN-2: Efficient Parallel Sequence Modeling" paper notes,
    section "Optimisation 2: compact channel propagation"): per pixel xp = P_in x (C_proxy x C
    matrix over channels), the propagation in proxy space, then y = P_out yp (C x C_proxy), all in
    float64. The channel products are numpy's (a library primitive as a step); lam, u and the
    logits are in proxy space."""
    x, p_in, p_out = _f64(x), _f64(p_in), _f64(p_out)
    xp = np.einsum("pc,nchw->nphw", p_in, x)
    yp = forward(xp, a, lam, u, wmode, mask, chunk)
    return np.einsum("cp,nphw->nchw", p_out, yp)


def plane_inputs(x, a, lam, u, n: int, c: int, wmode: int):
    """Slices the inputs of one (n, c) plane as an N=1, C=1 problem (both weight modes).

    Output planes are independent given their own x, lambda, u and the logits of their
    (n, c) (per-channel) or (n) (shared), so any plane of a large problem can be checked
    on its own.
    """
    cw = 0 if wmode else c
    return (x[n:n + 1, c:c + 1], a[:, n:n + 1, cw:cw + 1], lam[n:n + 1, c:c + 1], u[n:n + 1, c:c + 1])
