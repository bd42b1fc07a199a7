"""Local (chunked) propagation against the float64 oracle in every kernel family: chunk lengths
that divide the scan axis and ones that leave a short last chunk (which the descending scans
meet first), chunk 1 (pure injection), and chunks as long as the map (the global scan); forward
in every family, backward in the ones that have it."""
import pytest

import gspn_inputs
import linear_spatial_propagation_gspn_b200 as g
from gspn_inputs import small_case

from _cases import check_backward, check_forward

pytestmark = pytest.mark.gpu

CHUNKS = [1, 3, 8, 17, 64]


@pytest.mark.parametrize("chunk", CHUNKS)
@pytest.mark.parametrize("shape", [(1, 3, 24, 40), (2, 2, 17, 33)])
@pytest.mark.parametrize("mask", [15, 1, 2, 4, 8])
@pytest.mark.parametrize("wmode", [0, 1])
def test_generic_forward_chunked(chunk, shape, mask, wmode):
    wl = small_case(*shape, mask=mask, wmode=wmode, dtype="f32", seed=sum(shape) + mask + chunk)
    check_forward(wl, g.ALGO_GENERIC, chunk=chunk)


@pytest.mark.parametrize("chunk", CHUNKS)
@pytest.mark.parametrize("mask", [15, 2, 8])
@pytest.mark.parametrize("wmode", [0, 1])
def test_generic_backward_chunked(chunk, mask, wmode):
    wl = small_case(1, 2, 19, 21, mask=mask, wmode=wmode, dtype="f32", seed=31 + mask + chunk)
    check_backward(wl, g.ALGO_GENERIC, chunk=chunk)


@pytest.mark.parametrize("chunk", CHUNKS)
@pytest.mark.parametrize("shape", [(2, 3, 56, 56), (1, 2, 37, 64)])
@pytest.mark.parametrize("mask", [15, 2, 8])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_plane_forward_chunked(chunk, shape, mask, dtype):
    wl = small_case(*shape, mask=mask, wmode=0, dtype=dtype, seed=3 * sum(shape) + mask + chunk)
    check_forward(wl, g.ALGO_PLANE, chunk=chunk)


@pytest.mark.parametrize("chunk", CHUNKS)
@pytest.mark.parametrize("mask", [15, 1, 8])
def test_plane_backward_chunked(chunk, mask):
    wl = small_case(2, 2, 40, 28, mask=mask, wmode=0, dtype="f32", seed=41 + mask + chunk)
    check_backward(wl, g.ALGO_PLANE, chunk=chunk)


@pytest.mark.parametrize("chunk", CHUNKS + [100])
@pytest.mark.parametrize("shape", [(1, 3, 64, 1024), (1, 2, 1024, 64), (2, 2, 72, 40), (1, 2, 37, 40)])
@pytest.mark.parametrize("mask", [15, 5, 10])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sweep_forward_chunked(chunk, shape, mask, dtype):
    """Both vertical kernels (fixed 1024-lane and generic widths), the lane-major hand-over and
    the column-tile fallback (37 x 40: rows not 16-byte multiples in bf16)."""
    wl = small_case(*shape, mask=mask, wmode=1, dtype=dtype, seed=5 * sum(shape) + mask + chunk)
    check_forward(wl, g.ALGO_SWEEP, chunk=chunk)


def test_negative_chunk_rejected():
    d = g.make_desc(1, 1, 8, 8, chunk=-1)
    assert g.selected_algo(d) == -1
    assert g.workspace_size(d) == 0
