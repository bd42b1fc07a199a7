"""Seeded synthetic inputs for the GSPN line-scan workloads.

This module only draws random numbers of the right shapes, distributions and storage
dtypes. It holds none of the propagation arithmetic, so both the CUDA library's callers and
the float64 oracle's callers may use it.

Workloads (shapes follow the pages' timing tables: 1024x1024 maps with batch 16 and 8 channels
and with batch 1 and 1152 channels, "GSPN-2: Efficient Parallel Sequence Modeling" paper notes,
sections "Cumulative optimisation effect" and "Effect of each optimisation under different
workloads"; 56x56 with 96 channels is a classifier-stage map; 64x64 with 192 channels is the
training-step shape):

=========  ====  =====  ======  ===========  =========  ======  ==============
name        N     C      HxW    directions   weights    dtype   logits draw
=========  ====  =====  ======  ===========  =========  ======  ==============
tiny        1     4      16x16  TB only      per-chan   f32     N(0, 1)
classifier  128   96     56x56  all 4        per-chan   bf16    N(0, 1)
highres     16    8      1024^2 all 4        shared     f32     N(0, 1)
wide        1     1152   1024^2 all 4        shared     bf16    N(0, std 2)
train       32    192    64x64  all 4        per-chan   f32     N(0, 1)
=========  ====  =====  ======  ===========  =========  ======  ==============

x ~ N(0, 1), lambda ~ U(0, 1), u ~ N(0, 1), upstream dy ~ N(0, 1). bf16 workloads draw in
float32 and round once to bfloat16 (round to nearest even); those rounded values are what
both sides consume. Draw order: x, a, lambda, u, dy, all from one ``torch.Generator`` on the
target device seeded with the workload's seed (0 for ``tiny``, 1..4 for the others).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

F32, BF16 = "f32", "bf16"
PER_CHANNEL, SHARED = 0, 1
ALL_DIRS = 15


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    C: int
    H: int
    W: int
    mask: int
    wmode: int
    dtype: str
    a_std: float
    seed: int

    @property
    def D(self) -> int:
        return bin(self.mask).count("1")

    @property
    def Cw(self) -> int:
        return 1 if self.wmode == SHARED else self.C

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == F32 else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == F32 else 2

    @property
    def numel(self) -> int:
        return self.N * self.C * self.H * self.W

    @property
    def a_numel(self) -> int:
        return self.D * self.N * self.Cw * 3 * self.H * self.W

    def compulsory_fwd_bytes(self) -> int:
        """x, lambda, u read once, y written once, logits read once (storage dtype)."""
        return (4 * self.numel + self.a_numel) * self.elem_bytes

    def compulsory_bwd_bytes(self) -> int:
        """Reads dy, x, lambda, u, a; writes dx, dlambda, du, da (storage dtype)."""
        return (7 * self.numel + 2 * self.a_numel) * self.elem_bytes

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 16, 16, 1, PER_CHANNEL, F32, 1.0, 0),
    "classifier": Workload("classifier", 128, 96, 56, 56, ALL_DIRS, PER_CHANNEL, BF16, 1.0, 1),
    "highres": Workload("highres", 16, 8, 1024, 1024, ALL_DIRS, SHARED, F32, 1.0, 2),
    "wide": Workload("wide", 1, 1152, 1024, 1024, ALL_DIRS, SHARED, BF16, 2.0, 3),
    "train": Workload("train", 32, 192, 64, 64, ALL_DIRS, PER_CHANNEL, F32, 1.0, 4),
}


def make_inputs(wl: Workload, device="cpu", with_dy: bool = False, seed: int | None = None,
                per_dir: bool = False):
    """Returns a dict with x, a, lam, u (and dy) in the workload's storage dtype on ``device``.
    ``per_dir``: lam and u get a leading direction axis of length D (one map per direction)."""
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed if seed is None else seed)
    shp = (wl.N, wl.C, wl.H, wl.W)
    ashp = (wl.D, wl.N, wl.Cw, 3, wl.H, wl.W)
    dt = wl.torch_dtype
    out = {}
    out["x"] = torch.randn(shp, generator=g, device=device, dtype=torch.float32).to(dt)
    a = torch.randn(ashp, generator=g, device=device, dtype=torch.float32)
    if wl.a_std != 1.0:
        a.mul_(wl.a_std)
    out["a"] = a.to(dt)
    del a
    lu = ((wl.D,) if per_dir else ()) + shp
    out["lam"] = torch.rand(lu, generator=g, device=device, dtype=torch.float32).to(dt)
    out["u"] = torch.randn(lu, generator=g, device=device, dtype=torch.float32).to(dt)
    if with_dy:
        out["dy"] = torch.randn(shp, generator=g, device=device, dtype=torch.float32).to(dt)
    return out


def small_case(N, C, H, W, mask=ALL_DIRS, wmode=PER_CHANNEL, dtype=F32, a_std=1.0, seed=0) -> Workload:
    return Workload(f"case{N}x{C}x{H}x{W}", N, C, H, W, mask, wmode, dtype, a_std, seed)
