"""Host-side checks of libgspn (no GPU needed): the library loads, exports every symbol that
include/*.h declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import glob
import os
import re

import pytest

import linear_spatial_propagation_gspn_b200 as g

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"GSPN_API\s+[\w\s\*]+?\b(gspn_\w+)\s*\(", src))
    return sorted(names)


def test_header_declares_symbols():
    assert "gspn_forward" in declared_symbols() and "gspn_backward" in declared_symbols()


@pytest.mark.parametrize("name", declared_symbols())
def test_library_exports_symbol(name):
    L = g.lib()
    assert hasattr(L, name), name
    assert name in g.SIGNATURES, f"binding has no signature for {name}"


def test_version_and_strings():
    assert g.lib().gspn_version() >= 1
    for s in range(7):
        assert g.status_string(s)


def desc(**kw):
    base = dict(N=2, C=3, H=16, W=16, wmode=0, dir_mask=15, dtype=0, algo=0)
    base.update(kw)
    return g.make_desc(**base)


@pytest.mark.parametrize("bad", [dict(N=0), dict(C=-1), dict(H=0), dict(W=0), dict(dir_mask=0), dict(dir_mask=16),
                                 dict(wmode=2), dict(dtype=7), dict(algo=9), dict(chunk=-1), dict(per_dir=2)])
def test_invalid_descriptor(bad):
    d = desc(**bad)
    assert g.workspace_size(d) == 0
    assert g.selected_algo(d) == -1
    fake = 0x10000
    s = g.lib().gspn_forward(ctypes.byref(d), fake, fake, fake, fake, fake, fake, 1 << 20, None)
    assert s == g.GSPN_ERR_INVALID_ARG


def test_null_and_misaligned_pointers():
    d = desc()
    ws = g.workspace_size(d)
    fake = 0x10000
    L = g.lib()
    assert L.gspn_forward(ctypes.byref(d), None, fake, fake, fake, fake, fake, ws, None) == g.GSPN_ERR_INVALID_ARG
    assert L.gspn_forward(ctypes.byref(d), fake + 4, fake, fake, fake, fake, fake, ws, None) == g.GSPN_ERR_ALIGNMENT
    assert L.gspn_forward(ctypes.byref(d), fake, fake, fake, fake, fake, fake, ws - 1, None) == g.GSPN_ERR_WORKSPACE
    wsb = g.workspace_size(d, True)
    args = [fake] * 9
    assert L.gspn_backward(ctypes.byref(d), *args, fake, wsb - 16, None) == g.GSPN_ERR_WORKSPACE
    args[4] = fake + 8
    assert L.gspn_backward(ctypes.byref(d), *args, fake, wsb, None) == g.GSPN_ERR_ALIGNMENT


def test_forced_family_support():
    # plane family only takes maps that fit on chip; sweep only large aligned maps
    big = desc(H=1024, W=1024, algo=g.ALGO_PLANE)
    assert g.selected_algo(big) == -1 and g.workspace_size(big) == 0
    gen = desc(H=17, W=33, algo=g.ALGO_GENERIC)
    assert g.selected_algo(gen) == g.ALGO_GENERIC
    assert g.workspace_size(gen) >= 256


def test_workspace_sizes_monotone():
    small = g.workspace_size(desc(H=8, W=8, algo=g.ALGO_GENERIC), True)
    large = g.workspace_size(desc(H=64, W=64, algo=g.ALGO_GENERIC), True)
    assert 256 <= small < large


def test_wait_probe_rejects_long_limits():
    assert g.lib().gspn_debug_wait_timeout(0x10000, 1 << 12, 10 ** 10, None) == g.GSPN_ERR_INVALID_ARG
    assert g.lib().gspn_debug_wait_timeout(0x10000, 16, 1000, None) == g.GSPN_ERR_INVALID_ARG
