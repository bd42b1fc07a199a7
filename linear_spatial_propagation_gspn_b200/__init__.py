"""Python binding of libgspn, the sm_100a implementation of the GSPN 4-direction line scan.

Argument marshalling only: every step of the propagation runs in the CUDA kernels of
``libgspn.so`` (built in-tree by ``build.py``). PyTorch provides device memory and streams;
no computation on this path happens in PyTorch or on the CPU. If the library is missing the
calls raise instead of falling back.

Operation (see ``include/gspn.h`` for the full contract):
    h_{-1} = 0, h_i = w_i h_{i-1} + lam_i * x_i along each scan direction,
    y = u * sum_{d in dir_mask} h^d,
with w_i tridiagonal and row-stochastic, formed from sigmoid logits normalised over the
in-range neighbours ("Parallel Sequence Modeling via Generalized Spatial Propagation
Network" summary, section "Approach"; "GSPN-2: Efficient Parallel Sequence Modeling" paper
notes, sections "2D spatial propagation review" and "Optimisation 2: compact channel
propagation").
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build_mod

LIB_PATH = _build_mod.LIB

GSPN_OK, GSPN_ERR_INVALID_ARG, GSPN_ERR_UNSUPPORTED, GSPN_ERR_ALIGNMENT = 0, 1, 2, 3
GSPN_ERR_WORKSPACE, GSPN_ERR_CUDA, GSPN_ERR_DEVICE_TIMEOUT = 4, 5, 6
F32, BF16 = 0, 1
PER_CHANNEL, SHARED = 0, 1
DIR_TB, DIR_BT, DIR_LR, DIR_RL, DIR_ALL = 1, 2, 4, 8, 15
ALGO_AUTO, ALGO_GENERIC, ALGO_PLANE, ALGO_SWEEP, ALGO_BAND = 0, 1, 2, 3, 4
ALGO_NAMES = {ALGO_GENERIC: "generic", ALGO_PLANE: "plane", ALGO_SWEEP: "sweep", ALGO_BAND: "band"}


class GspnDesc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("C", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("wmode", ctypes.c_int), ("dir_mask", ctypes.c_uint), ("dtype", ctypes.c_int),
                ("algo", ctypes.c_int), ("chunk", ctypes.c_int), ("per_dir", ctypes.c_int)]


class GspnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None

# (name, restype, argtypes) of every symbol include/gspn.h declares.
_VP, _SZ, _I, _U64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_ulonglong
_DP = ctypes.POINTER(GspnDesc)
SIGNATURES = {
    "gspn_workspace_size": (_SZ, [_DP, _I]),
    "gspn_selected_algo": (_I, [_DP, _I]),
    "gspn_forward": (_I, [_DP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "gspn_backward": (_I, [_DP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "gspn_forward_timed": (_I, [_DP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP, _I, ctypes.POINTER(_I)]),
    "gspn_forward_host_buffer_size": (_SZ, [_DP]),
    "gspn_forward_host": (_I, [_DP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "gspn_device_status": (_I, [_VP, _VP]),
    "gspn_debug_wait_timeout": (_I, [_VP, _SZ, _U64, _VP]),
    "gspn_copy_ceiling": (_I, [_VP, _VP, _SZ, _VP]),
    "gspn_forward_noalloc": (_I, [_DP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "gspn_hsave_size": (_SZ, [_DP]),
    "gspn_forward_save": (_I, [_DP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "gspn_backward_saved": (_I, [_DP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "gspn_proxy_workspace_size": (_SZ, [_DP, _I]),
    "gspn_proxy_forward": (_I, [_DP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "gspn_status_string": (ctypes.c_char_p, [_I]),
    "gspn_version": (_I, []),
}


def build(force: bool = False) -> str:
    """Compiles libgspn.so in-tree (nvcc, sm_100a)."""
    return _build_mod.build(force=force)


def lib():
    """The loaded libgspn. Raises if it has not been built: there is no fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgspn.so is not built ({LIB_PATH}); run "
                               "`python -m linear_spatial_propagation_gspn_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().gspn_status_string(int(s)).decode()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return F32
    if t == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t} (float32 or bfloat16)")


def make_desc(N, C, H, W, wmode=PER_CHANNEL, dir_mask=DIR_ALL, dtype=F32, algo=ALGO_AUTO, chunk=0,
              per_dir=0) -> GspnDesc:
    return GspnDesc(int(N), int(C), int(H), int(W), int(wmode), int(dir_mask), int(dtype), int(algo), int(chunk),
                    int(per_dir))


def desc_for(x: torch.Tensor, wmode: int, dir_mask: int, algo: int = ALGO_AUTO, chunk: int = 0,
             per_dir: int = 0) -> GspnDesc:
    N, C, H, W = x.shape
    return make_desc(N, C, H, W, wmode, dir_mask, _dtype_code(x.dtype), algo, chunk, per_dir)


def _lu_shape(x: torch.Tensor, dir_mask: int, per_dir: int):
    return ((bin(dir_mask & 15).count("1"),) if per_dir else ()) + tuple(x.shape)


def workspace_size(desc: GspnDesc, backward: bool = False) -> int:
    return int(lib().gspn_workspace_size(ctypes.byref(desc), int(backward)))


def selected_algo(desc: GspnDesc, backward: bool = False) -> int:
    return int(lib().gspn_selected_algo(ctypes.byref(desc), int(backward)))


def logits_shape(N, C, H, W, wmode, dir_mask):
    return (bin(dir_mask & 15).count("1"), N, 1 if wmode == SHARED else C, 3, H, W)


def _check(tensors, like: torch.Tensor):
    for name, t in tensors.items():
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.device.type != "cuda":
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dtype != like.dtype:
            raise TypeError(f"{name} has dtype {t.dtype}, expected {like.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def _stream_ptr(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def alloc_workspace(desc: GspnDesc, backward: bool, device) -> torch.Tensor:
    n = workspace_size(desc, backward)
    if n == 0:
        raise GspnError(GSPN_ERR_UNSUPPORTED, "workspace size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def forward(x, a, lam, u, wmode: int = PER_CHANNEL, dir_mask: int = DIR_ALL, algo: int = ALGO_AUTO,
            y=None, ws=None, stream=None, chunk: int = 0, per_dir: int = 0) -> torch.Tensor:
    """y = u * sum_d h^d. x, lam, u: (N, C, H, W); a: (D, N, Cw, 3, H, W); all one dtype.
    chunk > 0: local propagation within image-aligned chunks of that many lines. per_dir = 1:
    lam and u are (D, N, C, H, W) and y = sum_d u_d * h^d(lam_d * x)."""
    _check({"x": x, "a": a, "lam": lam, "u": u}, x)
    if tuple(a.shape) != logits_shape(*x.shape, wmode, dir_mask):
        raise ValueError(f"logits shape {tuple(a.shape)}, expected {logits_shape(*x.shape, wmode, dir_mask)}")
    if tuple(lam.shape) != _lu_shape(x, dir_mask, per_dir) or tuple(u.shape) != _lu_shape(x, dir_mask, per_dir):
        raise ValueError(f"lam and u must be {_lu_shape(x, dir_mask, per_dir)}")
    desc = desc_for(x, wmode, dir_mask, algo, chunk, per_dir)
    if y is None:
        y = torch.empty_like(x)
    _check({"y": y}, x)
    if ws is None:
        ws = alloc_workspace(desc, False, x.device)
    s = lib().gspn_forward(ctypes.byref(desc), x.data_ptr(), a.data_ptr(), lam.data_ptr(), u.data_ptr(),
                           y.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    if s != GSPN_OK:
        raise GspnError(s, "gspn_forward")
    return y


def backward(x, a, lam, u, dy, wmode: int = PER_CHANNEL, dir_mask: int = DIR_ALL, algo: int = ALGO_AUTO,
             out=None, ws=None, stream=None, chunk: int = 0, per_dir: int = 0):
    """Gradients (dx, da, dlam, du) of sum(dy * y)."""
    _check({"x": x, "a": a, "lam": lam, "u": u, "dy": dy}, x)
    if tuple(a.shape) != logits_shape(*x.shape, wmode, dir_mask):
        raise ValueError("logits shape mismatch")
    if tuple(lam.shape) != _lu_shape(x, dir_mask, per_dir) or tuple(u.shape) != _lu_shape(x, dir_mask, per_dir):
        raise ValueError(f"lam and u must be {_lu_shape(x, dir_mask, per_dir)}")
    desc = desc_for(x, wmode, dir_mask, algo, chunk, per_dir)
    if out is None:
        out = (torch.empty_like(x), torch.empty_like(a), torch.empty_like(lam), torch.empty_like(u))
    dx, da, dlam, du = out
    _check({"dx": dx, "da": da, "dlam": dlam, "du": du}, x)
    if ws is None:
        ws = alloc_workspace(desc, True, x.device)
    s = lib().gspn_backward(ctypes.byref(desc), x.data_ptr(), a.data_ptr(), lam.data_ptr(), u.data_ptr(),
                            dy.data_ptr(), dx.data_ptr(), da.data_ptr(), dlam.data_ptr(), du.data_ptr(),
                            ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    if s != GSPN_OK:
        raise GspnError(s, "gspn_backward")
    return dx, da, dlam, du


def hsave_size(desc: GspnDesc) -> int:
    """Bytes of the per-direction h that gspn_forward_save keeps (0: the pair does not apply)."""
    return int(lib().gspn_hsave_size(ctypes.byref(desc)))


def forward_save(x, a, lam, u, wmode: int = PER_CHANNEL, dir_mask: int = DIR_ALL, y=None, hsave=None, ws=None,
                 stream=None, chunk: int = 0):
    """Training forward: y and each direction's h (a flat fp32 tensor) for backward_saved."""
    _check({"x": x, "a": a, "lam": lam, "u": u}, x)
    if tuple(a.shape) != logits_shape(*x.shape, wmode, dir_mask):
        raise ValueError("logits shape mismatch")
    desc = desc_for(x, wmode, dir_mask, chunk=chunk)
    nb = hsave_size(desc)
    if nb == 0:
        raise GspnError(GSPN_ERR_UNSUPPORTED, "gspn_hsave_size")
    if y is None:
        y = torch.empty_like(x)
    if hsave is None:
        hsave = torch.empty(nb // 4, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = alloc_workspace(desc, False, x.device)
    s = lib().gspn_forward_save(ctypes.byref(desc), x.data_ptr(), a.data_ptr(), lam.data_ptr(), u.data_ptr(),
                                y.data_ptr(), hsave.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    if s != GSPN_OK:
        raise GspnError(s, "gspn_forward_save")
    return y, hsave


def backward_saved(x, a, lam, u, dy, hsave, wmode: int = PER_CHANNEL, dir_mask: int = DIR_ALL, out=None, ws=None,
                   stream=None, chunk: int = 0):
    """Gradients of sum(dy * y) from the h kept by forward_save (no recompute of the scans)."""
    _check({"x": x, "a": a, "lam": lam, "u": u, "dy": dy}, x)
    desc = desc_for(x, wmode, dir_mask, chunk=chunk)
    if out is None:
        out = (torch.empty_like(x), torch.empty_like(a), torch.empty_like(lam), torch.empty_like(u))
    dx, da, dlam, du = out
    if ws is None:
        ws = alloc_workspace(desc, True, x.device)
    s = lib().gspn_backward_saved(ctypes.byref(desc), x.data_ptr(), a.data_ptr(), lam.data_ptr(), u.data_ptr(),
                                  dy.data_ptr(), hsave.data_ptr(), dx.data_ptr(), da.data_ptr(), dlam.data_ptr(),
                                  du.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    if s != GSPN_OK:
        raise GspnError(s, "gspn_backward_saved")
    return dx, da, dlam, du


def proxy_forward(x, p_in, a, lam, u, p_out, wmode: int = SHARED, dir_mask: int = DIR_ALL, algo: int = ALGO_AUTO,
                  y=None, ws=None, stream=None, chunk: int = 0) -> torch.Tensor:
    """Compressive channel proxy: y = P_out . propagate(P_in . x) per pixel. x: (N, C, H, W);
    p_in: (Cp, C); p_out: (C, Cp); a, lam, u in proxy space (C = Cp); all one dtype."""
    _check({"x": x, "p_in": p_in, "a": a, "lam": lam, "u": u, "p_out": p_out}, x)
    N, C, H, W = x.shape
    Cp = p_in.shape[0]
    if tuple(p_in.shape) != (Cp, C) or tuple(p_out.shape) != (C, Cp):
        raise ValueError(f"projection shapes {tuple(p_in.shape)}, {tuple(p_out.shape)}; expected ({Cp}, {C}), ({C}, {Cp})")
    if tuple(lam.shape) != (N, Cp, H, W) or tuple(u.shape) != (N, Cp, H, W):
        raise ValueError("lam and u must be (N, C_proxy, H, W)")
    if tuple(a.shape) != logits_shape(N, Cp, H, W, wmode, dir_mask):
        raise ValueError(f"logits shape {tuple(a.shape)}, expected {logits_shape(N, Cp, H, W, wmode, dir_mask)}")
    desc = make_desc(N, Cp, H, W, wmode, dir_mask, _dtype_code(x.dtype), algo, chunk)
    if y is None:
        y = torch.empty_like(x)
    _check({"y": y}, x)
    if ws is None:
        nb = int(lib().gspn_proxy_workspace_size(ctypes.byref(desc), C))
        if nb == 0:
            raise GspnError(GSPN_ERR_UNSUPPORTED, "gspn_proxy_workspace_size")
        ws = torch.empty(nb, dtype=torch.uint8, device=x.device)
    s = lib().gspn_proxy_forward(ctypes.byref(desc), C, x.data_ptr(), p_in.data_ptr(), a.data_ptr(), lam.data_ptr(),
                                 u.data_ptr(), p_out.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(),
                                 _stream_ptr(stream))
    if s != GSPN_OK:
        raise GspnError(s, "gspn_proxy_forward")
    return y


def forward_timed(x, a, lam, u, y, ws, desc: GspnDesc, events, stream=None) -> int:
    """gspn_forward recording ``events`` (materialised torch.cuda.Event objects, two per launch)
    around each kernel launch; returns the number of launches."""
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    n = ctypes.c_int(0)
    s = lib().gspn_forward_timed(ctypes.byref(desc), x.data_ptr(), a.data_ptr(), lam.data_ptr(), u.data_ptr(),
                                 y.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream), arr, len(events),
                                 ctypes.byref(n))
    if s != GSPN_OK:
        raise GspnError(s, "gspn_forward_timed")
    return n.value


def forward_host_buffer_size(desc: GspnDesc) -> int:
    return int(lib().gspn_forward_host_buffer_size(ctypes.byref(desc)))


def forward_host(desc: GspnDesc, hx, ha, hlam, hu, hy, dev: torch.Tensor, stream=None):
    """End-to-end forward from host tensors (pinned for asynchronous copies) into host ``hy``."""
    for name, t in {"hx": hx, "ha": ha, "hlam": hlam, "hu": hu, "hy": hy}.items():
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    s = lib().gspn_forward_host(ctypes.byref(desc), hx.data_ptr(), ha.data_ptr(), hlam.data_ptr(), hu.data_ptr(),
                                hy.data_ptr(), dev.data_ptr(), dev.numel() * dev.element_size(),
                                _stream_ptr(stream))
    if s != GSPN_OK:
        raise GspnError(s, "gspn_forward_host")
    return hy


def device_status(ws: torch.Tensor, stream=None) -> int:
    return int(lib().gspn_device_status(ws.data_ptr(), _stream_ptr(stream)))


def debug_wait_timeout(ws: torch.Tensor, limit_ns: int, stream=None) -> int:
    return int(lib().gspn_debug_wait_timeout(ws.data_ptr(), ws.numel(), int(limit_ns), _stream_ptr(stream)))


def copy_ceiling(src: torch.Tensor, dst: torch.Tensor, stream=None):
    nbytes = src.numel() * src.element_size()
    s = lib().gspn_copy_ceiling(src.data_ptr(), dst.data_ptr(), nbytes, _stream_ptr(stream))
    if s != GSPN_OK:
        raise GspnError(s, "gspn_copy_ceiling")


class GSPNFunction(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run in libgspn."""

    @staticmethod
    def forward(ctx, x, a, lam, u, wmode, dir_mask, chunk=0, per_dir=0):
        ctx.wmode, ctx.dir_mask, ctx.chunk, ctx.per_dir = wmode, dir_mask, chunk, per_dir
        ctx.saved_h = per_dir == 0 and hsave_size(desc_for(x, wmode, dir_mask, chunk=chunk)) > 0
        if ctx.saved_h:   # keep each direction's h: the backward then skips recomputing the scans
            y, hsave = forward_save(x, a, lam, u, wmode, dir_mask, chunk=chunk)
            ctx.save_for_backward(x, a, lam, u, hsave)
            return y
        ctx.save_for_backward(x, a, lam, u)
        return forward(x, a, lam, u, wmode, dir_mask, chunk=chunk, per_dir=per_dir)

    @staticmethod
    def backward(ctx, dy):
        if ctx.saved_h:
            x, a, lam, u, hsave = ctx.saved_tensors
            dx, da, dlam, du = backward_saved(x, a, lam, u, dy.contiguous(), hsave, ctx.wmode, ctx.dir_mask,
                                              chunk=ctx.chunk)
        else:
            x, a, lam, u = ctx.saved_tensors
            dx, da, dlam, du = backward(x, a, lam, u, dy.contiguous(), ctx.wmode, ctx.dir_mask, chunk=ctx.chunk,
                                        per_dir=ctx.per_dir)
        return dx, da, dlam, du, None, None, None, None


def gspn(x, a, lam, u, wmode: int = PER_CHANNEL, dir_mask: int = DIR_ALL, chunk: int = 0, per_dir: int = 0):
    """Differentiable GSPN propagation (libgspn forward and backward); chunk > 0 = local;
    per_dir = 1: per-direction lam and u (D, N, C, H, W)."""
    return GSPNFunction.apply(x, a, lam, u, wmode, dir_mask, chunk, per_dir)
