"""Pins for the float64 oracle (CPU only).

The oracle is checked against things other than itself:
  * the closed matrix form H = G X built independently with NumPy (``oracle/brute.py``),
  * hand-derived values (``tests/golden/hand_cases.json``),
  * the row-stochastic fixed point and the constant-input closed form,
  * direction equivalences under flips and transposes,
  * W = 1 reducing to ``numpy.cumsum`` and H = 1 (single step) reducing to z,
  * the stability bound, linearity and mode equivalence,
  * central finite differences and the adjoint dot-product identity for the backward.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import brute

HERE = os.path.dirname(os.path.abspath(__file__))
DIRS = (1, 2, 4, 8)


def rand_case(rng, N, C, H, W, mask=15, wmode=0, a_std=1.0):
    D = bin(mask).count("1")
    Cw = 1 if wmode else C
    x = rng.standard_normal((N, C, H, W))
    a = rng.standard_normal((D, N, Cw, 3, H, W)) * a_std
    lam = rng.uniform(0, 1, (N, C, H, W))
    u = rng.standard_normal((N, C, H, W))
    return x, a, lam, u


# ----------------------------------------------------------------------------- brute force G
SHAPES = [(4, 5), (6, 6), (5, 3), (1, 4), (4, 1), (2, 2), (3, 1), (1, 1), (3, 7)]


@pytest.mark.parametrize("H,W", SHAPES)
@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("mask", [1, 2, 4, 8, 15, 5, 10, 3, 12, 9])
def test_recurrence_matches_block_triangular_G(H, W, wmode, mask):
    rng = np.random.default_rng(1000 * H + 10 * W + mask + 7 * wmode)
    x, a, lam, u = rand_case(rng, 2, 2, H, W, mask, wmode)
    y_rec = oracle.forward(x, a, lam, u, wmode, mask)
    y_mat = brute.forward(x, a, lam, u, wmode, mask)
    np.testing.assert_allclose(y_rec, y_mat, rtol=0, atol=1e-12 * max(1.0, np.abs(y_mat).max()))


# ----------------------------------------------------------------------------- hand-derived
def _val(s):
    if s == "ln2":
        return math.log(2.0)
    if s == "-ln2":
        return -math.log(2.0)
    return float(Fraction(s))


def _load_golden():
    with open(os.path.join(HERE, "golden", "hand_cases.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _load_golden()["cases"], ids=lambda c: c["name"])
def test_hand_derived_forward(case):
    N, C, H, W, mask, wmode = (case[k] for k in ("N", "C", "H", "W", "mask", "wmode"))
    D = bin(mask).count("1")
    a = np.zeros((D, N, C, 3, H, W))
    for k in range(3):
        a[:, :, :, k] = _val(case["logits_k"][k])
    x = np.array(case["x"], dtype=np.float64).reshape(N, C, H, W)
    lam = np.full_like(x, case["lam"])
    u = np.full_like(x, case["u"])
    want = np.array([[_val(v) for v in row] for row in case["y"]]).reshape(N, C, H, W)
    got = oracle.forward(x, a, lam, u, wmode, mask)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


@pytest.mark.parametrize("case", _load_golden()["grad_cases"], ids=lambda c: c["name"])
def test_hand_derived_backward(case):
    N, C, H, W, mask, wmode = (case[k] for k in ("N", "C", "H", "W", "mask", "wmode"))
    x = np.array(case["x"], dtype=np.float64).reshape(N, C, H, W)
    dy = np.array(case["dy"], dtype=np.float64).reshape(N, C, H, W)
    a = np.zeros((1, N, C, 3, H, W))
    lam = np.ones_like(x)
    u = np.ones_like(x)
    dx, da, dlam, du = oracle.backward(x, a, lam, u, dy, wmode, mask)
    grid = lambda rows: np.array([[_val(v) for v in r] for r in rows]).reshape(N, C, H, W)
    np.testing.assert_allclose(dx, grid(case["dx"]), atol=1e-14)
    np.testing.assert_allclose(dlam, grid(case["dlam"]), atol=1e-14)
    np.testing.assert_allclose(du, grid(case["du"]), atol=1e-14)
    want_da = np.zeros_like(da)
    want_da[0, 0, 0, :, 1, 0] = [_val(v) for v in case["da_step1_lane0"]]
    np.testing.assert_allclose(da, want_da, atol=1e-14)


# ----------------------------------------------------------------------------- invariants
def _first_line_mask(d, H, W):
    m = np.zeros((H, W))
    if d == 1:
        m[0, :] = 1
    elif d == 2:
        m[H - 1, :] = 1
    elif d == 4:
        m[:, 0] = 1
    else:
        m[:, W - 1] = 1
    return m


@pytest.mark.parametrize("d", DIRS)
@pytest.mark.parametrize("H,W", [(7, 5), (1, 6), (6, 1), (9, 9)])
def test_row_stochastic_fixed_point(d, H, W):
    """lambda*x = 1 on the first line of the scan and 0 after it => h == 1 everywhere."""
    rng = np.random.default_rng(d * 31 + H)
    a = rng.standard_normal((1, 1, 1, 3, H, W)) * 3.0
    x = _first_line_mask(d, H, W)[None, None]
    lam = np.ones_like(x)
    u = np.ones_like(x)
    y = oracle.forward(x, a, lam, u, 0, d)
    np.testing.assert_allclose(y, 1.0, rtol=0, atol=1e-13)


@pytest.mark.parametrize("d", DIRS)
def test_constant_input_closed_form(d):
    """Constant z => h_i = (i+1) z exactly (each row of w sums to 1)."""
    H, W = 6, 4
    rng = np.random.default_rng(5 + d)
    a = rng.standard_normal((1, 1, 1, 3, H, W))
    x = np.full((1, 1, H, W), 0.75)
    lam = np.full_like(x, 2.0)
    y = oracle.forward(x, a, lam, np.ones_like(x), 0, d)
    r = np.arange(H)[:, None] * np.ones((1, W))
    c = np.ones((H, 1)) * np.arange(W)[None, :]
    step = {1: r, 2: H - 1 - r, 4: c, 8: W - 1 - c}[d]
    np.testing.assert_allclose(y[0, 0], 1.5 * (step + 1), rtol=1e-14)


@pytest.mark.parametrize("H,W", [(5, 7), (6, 6), (1, 3)])
def test_direction_equivalences(H, W):
    """Other directions are top->bottom on flipped / transposed arrays (k is not permuted)."""
    rng = np.random.default_rng(H * 100 + W)
    x, a, lam, u = rand_case(rng, 1, 2, H, W, mask=1)
    tb = lambda X, A, L, U: oracle.forward(X, A, L, U, 0, 1)
    fH = lambda t: np.ascontiguousarray(t[..., ::-1, :])
    fW = lambda t: np.ascontiguousarray(t[..., :, ::-1])
    T = lambda t: np.ascontiguousarray(np.swapaxes(t, -1, -2))
    # BT = flipH . TB . flipH
    bt = oracle.forward(x, a, lam, u, 0, 2)
    np.testing.assert_allclose(bt, fH(tb(fH(x), fH(a), fH(lam), fH(u))), atol=1e-13)
    # LR = T . TB . T
    lr = oracle.forward(x, a, lam, u, 0, 4)
    np.testing.assert_allclose(lr, T(tb(T(x), T(a), T(lam), T(u))), atol=1e-13)
    # RL = T . flip . TB . flip . T  (flip of the transposed rows = flip of image columns)
    rl = oracle.forward(x, a, lam, u, 0, 8)
    g = lambda t: fH(T(t))
    ginv = lambda t: T(fH(t))
    np.testing.assert_allclose(rl, ginv(tb(g(x), g(a), g(lam), g(u))), atol=1e-13)
    # all four = sum of singles
    a4 = np.concatenate([a] * 4, axis=0)
    all4 = oracle.forward(x, a4, lam, u, 0, 15)
    np.testing.assert_allclose(all4, tb(x, a, lam, u) + bt + lr + rl, atol=1e-12)


def test_single_lane_is_cumsum():
    """W = 1: the only in-range neighbour is the lane itself (w = 1), so TB = cumsum along H."""
    rng = np.random.default_rng(3)
    x, a, lam, u = rand_case(rng, 2, 3, 9, 1, mask=3)
    z = lam * x
    y = oracle.forward(x, a, lam, u, 0, 3)
    want = u * (np.cumsum(z, axis=2) + np.cumsum(z[:, :, ::-1], axis=2)[:, :, ::-1])
    np.testing.assert_allclose(y, want, rtol=1e-13, atol=1e-13)


def test_single_step_is_injection():
    """H = 1: TB and BT have one step, so h = lambda * x."""
    rng = np.random.default_rng(4)
    x, a, lam, u = rand_case(rng, 1, 2, 1, 7, mask=3)
    np.testing.assert_allclose(oracle.forward(x, a, lam, u, 0, 3), 2 * u * lam * x, atol=1e-14)


def test_sigmoid_matches_library_expit():
    """Single interior lane, two steps: h1 = sum_k expit(a_k) h0[k] / sum expit + z1."""
    from scipy.special import expit
    rng = np.random.default_rng(9)
    a = rng.standard_normal((1, 1, 1, 3, 2, 3)) * 4
    x = np.array([[[[1.0, -2.0, 0.5], [0.0, 0.0, 0.0]]]])
    y = oracle.forward(x, a, np.ones_like(x), np.ones_like(x), 0, 1)
    s = expit(a[0, 0, 0, :, 1, 1])
    np.testing.assert_allclose(y[0, 0, 1, 1], (s * x[0, 0, 0]).sum() / s.sum(), rtol=1e-14)


@pytest.mark.parametrize("d", DIRS)
def test_stability_bound(d):
    """||h_i||_inf <= ||h_{i-1}||_inf + ||z_i||_inf (rows of w are convex combinations)."""
    H, W = 12, 10
    rng = np.random.default_rng(11 + d)
    x, a, lam, u = rand_case(rng, 1, 1, H, W, mask=d, a_std=5.0)
    h = oracle.forward(x, a, lam, np.ones_like(u), 0, d)[0, 0]
    z = (lam * x)[0, 0]
    to_scan = {1: lambda t: t, 2: lambda t: t[::-1], 4: lambda t: t.T, 8: lambda t: t[:, ::-1].T}[d]
    hs, zs = to_scan(h), to_scan(z)
    for i in range(1, hs.shape[0]):
        assert np.abs(hs[i]).max() <= np.abs(hs[i - 1]).max() + np.abs(zs[i]).max() + 1e-12


def test_shared_equals_per_channel_broadcast():
    rng = np.random.default_rng(21)
    x, a, lam, u = rand_case(rng, 2, 3, 5, 6, mask=15, wmode=1)
    y_sh = oracle.forward(x, a, lam, u, 1, 15)
    y_pc = oracle.forward(x, np.repeat(a, 3, axis=2), lam, u, 0, 15)
    np.testing.assert_allclose(y_sh, y_pc, rtol=1e-15, atol=1e-15)
    dy = rng.standard_normal(x.shape)
    g_sh = oracle.backward(x, a, lam, u, dy, 1, 15)
    g_pc = oracle.backward(x, np.repeat(a, 3, axis=2), lam, u, dy, 0, 15)
    for k in (0, 2, 3):
        np.testing.assert_allclose(g_sh[k], g_pc[k], atol=1e-13)
    np.testing.assert_allclose(g_sh[1], g_pc[1].sum(axis=2, keepdims=True), atol=1e-12)


def test_linearity_and_gate_scaling():
    rng = np.random.default_rng(22)
    x, a, lam, u = rand_case(rng, 1, 2, 6, 5)
    x2 = rng.standard_normal(x.shape)
    f = lambda X, U=u: oracle.forward(X, a, lam, U, 0, 15)
    np.testing.assert_allclose(f(2.5 * x - x2), 2.5 * f(x) - f(x2), atol=1e-12)
    np.testing.assert_allclose(f(x, 3 * u), 3 * f(x), atol=1e-12)


def test_extreme_logits_finite():
    rng = np.random.default_rng(23)
    x, a, lam, u = rand_case(rng, 1, 1, 8, 8)
    a = rng.uniform(-60, 60, a.shape)
    y = oracle.forward(x, a, lam, u, 0, 15)
    assert np.isfinite(y).all()
    np.testing.assert_allclose(y, brute.forward(x, a, lam, u, 0, 15), atol=1e-11 * np.abs(y).max())


# ----------------------------------------------------------------------------- backward
def _loss(x, a, lam, u, dy, wmode, mask):
    return float((dy * oracle.forward(x, a, lam, u, wmode, mask)).sum())


@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("mask", [1, 2, 4, 8, 15])
def test_backward_finite_differences(wmode, mask):
    rng = np.random.default_rng(40 + mask + 100 * wmode)
    x, a, lam, u = rand_case(rng, 1, 2, 5, 4, mask, wmode)
    dy = rng.standard_normal(x.shape)
    grads = oracle.backward(x, a, lam, u, dy, wmode, mask)
    args = [x, a, lam, u]
    eps = 1e-6
    for gi, ai in ((0, 0), (1, 1), (2, 2), (3, 3)):
        base = args[ai]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = base[idx]
            base[idx] = old + eps
            lp = _loss(*args, dy, wmode, mask)
            base[idx] = old - eps
            lm = _loss(*args, dy, wmode, mask)
            base[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        g = grads[gi]
        scale = max(1.0, np.abs(fd).max())
        assert np.abs(g - fd).max() <= 1e-6 * scale, (gi, np.abs(g - fd).max())


def test_backward_zero_on_first_step_logits():
    """Step-0 logits multiply h_{-1} = 0, so their gradient is exactly zero."""
    rng = np.random.default_rng(50)
    x, a, lam, u = rand_case(rng, 1, 1, 4, 5, mask=15)
    _, da, _, _ = oracle.backward(x, a, lam, u, rng.standard_normal(x.shape), 0, 15)
    assert np.all(da[0, :, :, :, 0, :] == 0)       # TB: row 0
    assert np.all(da[1, :, :, :, -1, :] == 0)      # BT: last row
    assert np.all(da[2, :, :, :, :, 0] == 0)       # LR: column 0
    assert np.all(da[3, :, :, :, :, -1] == 0)      # RL: last column
    # out-of-range neighbours never get a gradient
    assert np.all(da[0, :, :, 0, :, 0] == 0) and np.all(da[0, :, :, 2, :, -1] == 0)
    assert np.all(da[2, :, :, 0, 0, :] == 0) and np.all(da[2, :, :, 2, -1, :] == 0)


@pytest.mark.parametrize("wmode", [0, 1])
def test_adjoint_dot_product(wmode):
    """y is linear in x: <dy, y(v)> == <dx(dy), v> (dx is the transpose applied to dy)."""
    rng = np.random.default_rng(60 + wmode)
    _, a, lam, u = rand_case(rng, 2, 3, 7, 6, 15, wmode)
    v = rng.standard_normal(lam.shape)
    dy = rng.standard_normal(lam.shape)
    lhs = float((dy * oracle.forward(v, a, lam, u, wmode, 15)).sum())
    dx, _, _, _ = oracle.backward(v, a, lam, u, dy, wmode, 15)
    rhs = float((dx * v).sum())
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs))


def test_transpose_matches_brute_jacobian():
    """dz for one direction equals J^T g with J built column by column from the matrix form."""
    rng = np.random.default_rng(70)
    H, W = 4, 3
    for d_i, d in enumerate(DIRS):
        x, a, lam, u = rand_case(rng, 1, 1, H, W, mask=d)
        dy = rng.standard_normal(x.shape)
        J = brute.jacobian_z(a[0, 0, 0], d, H, W)
        g = (dy * u).reshape(-1)
        dz = J.T @ g
        dx, _, dlam, _ = oracle.backward(x, a, lam, u, dy, 0, d)
        np.testing.assert_allclose(dx.reshape(-1), lam.reshape(-1) * dz, atol=1e-12)
        np.testing.assert_allclose(dlam.reshape(-1), x.reshape(-1) * dz, atol=1e-12)


def test_mutation_is_detected():
    """A planted mistake (k order reversed) in a copy of the inputs breaks the G check."""
    rng = np.random.default_rng(80)
    x, a, lam, u = rand_case(rng, 1, 1, 4, 5, mask=1)
    good = brute.forward(x, a, lam, u, 0, 1)
    wrong = oracle.forward(x, a[:, :, :, ::-1].copy(), lam, u, 0, 1)
    assert np.abs(good - wrong).max() > 1e-3


# ----------------------------------------------------------------------------- local (chunked) scans
# Reading: with chunk length K the image is cut into K-line chunks along each direction's scan
# axis, aligned to image line 0, and propagation never crosses a chunk boundary.

def _slot_of(mask, d):
    return bin(mask & (d - 1)).count("1")


@pytest.mark.parametrize("wmode", [0, 1])
def test_chunk_at_least_the_map_is_global(wmode):
    rng = np.random.default_rng(70 + wmode)
    x, a, lam, u = rand_case(rng, 1, 2, 6, 5, 15, wmode)
    y0 = oracle.forward(x, a, lam, u, wmode, 15)
    for k in (6, 7, 100):
        assert np.array_equal(oracle.forward(x, a, lam, u, wmode, 15, chunk=k), y0)


@pytest.mark.parametrize("mask", [1, 2, 4, 8, 15, 6])
def test_chunk_of_one_line_is_pure_injection(mask):
    """K = 1: every line starts a chunk, h = z everywhere, y = u * D * lambda * x."""
    rng = np.random.default_rng(80 + mask)
    x, a, lam, u = rand_case(rng, 2, 2, 5, 7, mask, 0)
    y = oracle.forward(x, a, lam, u, 0, mask, chunk=1)
    D = bin(mask).count("1")
    assert np.abs(y - u * D * lam * x).max() <= 1e-12


@pytest.mark.parametrize("d", [1, 2, 4, 8])
@pytest.mark.parametrize("K", [2, 3, 4])
def test_chunked_scan_is_the_global_scan_of_each_block(d, K):
    """A chunked single-direction scan equals the global scan run separately on each
    image-aligned block of K lines (rows for TB/BT, columns for LR/RL), including the short
    last block; this pins the block alignment for the descending scans too."""
    rng = np.random.default_rng(90 + d + 10 * K)
    H, W = 7, 8
    x, a, lam, u = rand_case(rng, 1, 2, H, W, d, 0)
    y = oracle.forward(x, a, lam, u, 0, d, chunk=K)
    vertical = d in (1, 2)
    L = H if vertical else W
    ref = np.zeros_like(y)
    for s0 in range(0, L, K):
        sl = slice(s0, min(L, s0 + K))
        if vertical:
            blk = [t[:, :, sl, :] for t in (x, lam, u)]
            ab = a[:, :, :, :, sl, :]
            ref[:, :, sl, :] = oracle.forward(blk[0], ab, blk[1], blk[2], 0, d)
        else:
            blk = [t[:, :, :, sl] for t in (x, lam, u)]
            ab = a[:, :, :, :, :, sl]
            ref[:, :, :, sl] = oracle.forward(blk[0], ab, blk[1], blk[2], 0, d)
    assert np.abs(y - ref).max() <= 1e-12


def test_chunked_directions_add_up():
    """The 4-direction chunked result is the sum of the single-direction chunked results."""
    rng = np.random.default_rng(95)
    x, a, lam, u = rand_case(rng, 1, 2, 6, 9, 15, 1)
    y = oracle.forward(x, a, lam, u, 1, 15, chunk=4)
    parts = sum(oracle.forward(x, a[_slot_of(15, d):_slot_of(15, d) + 1], lam, u, 1, d, chunk=4) for d in (1, 2, 4, 8))
    assert np.abs(y - parts).max() <= 1e-12


@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("mask,K", [(15, 2), (1, 3), (2, 3), (8, 2)])
def test_chunked_backward_finite_differences(wmode, mask, K):
    rng = np.random.default_rng(97 + mask + 7 * K + 100 * wmode)
    x, a, lam, u = rand_case(rng, 1, 2, 5, 5, mask, wmode)
    dy = rng.standard_normal(x.shape)
    grads = oracle.backward(x, a, lam, u, dy, wmode, mask, chunk=K)
    args = [x, a, lam, u]
    eps = 1e-6

    def loss():
        return float((dy * oracle.forward(*args, wmode, mask, chunk=K)).sum())

    for gi in range(4):
        base = args[gi]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = base[idx]
            base[idx] = old + eps
            lp = loss()
            base[idx] = old - eps
            lm = loss()
            base[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        scale = max(1.0, np.abs(fd).max())
        assert np.abs(grads[gi] - fd).max() <= 1e-6 * scale, (gi, np.abs(grads[gi] - fd).max())


def test_chunk_start_logits_have_zero_gradient():
    """The weights of a chunk's first line multiply h = 0: their logit gradient is zero."""
    rng = np.random.default_rng(99)
    x, a, lam, u = rand_case(rng, 1, 1, 7, 5, 1, 0)   # TB only
    dy = rng.standard_normal(x.shape)
    _, da, _, _ = oracle.backward(x, a, lam, u, dy, 0, 1, chunk=3)
    for r in (0, 3, 6):
        assert np.all(da[0, 0, 0, :, r, :] == 0.0)
    assert np.abs(da[0, 0, 0, :, 1, :]).max() > 0.0


# ----------------------------------------------------------------------------- channel proxy
def _proxy_case(rng, N, C, Cp, H, W, mask=15, wmode=1):
    x = rng.standard_normal((N, C, H, W))
    _, a, lam, u = rand_case(rng, N, Cp, H, W, mask, wmode)
    p_in = rng.standard_normal((Cp, C)) / np.sqrt(C)
    p_out = rng.standard_normal((C, Cp)) / np.sqrt(Cp)
    return x, p_in, a, lam, u, p_out


def test_proxy_with_identity_projections_is_the_plain_propagation():
    rng = np.random.default_rng(200)
    x, _, a, lam, u, _ = _proxy_case(rng, 2, 3, 3, 5, 6)
    eye = np.eye(3)
    y = oracle.proxy_forward(x, eye, a, lam, u, eye, 1, 15)
    assert np.abs(y - oracle.forward(x, a, lam, u, 1, 15)).max() <= 1e-12


def test_proxy_matches_pixel_loops():
    """The channel products written as explicit loops over pixels and channels (pins the
    operand orientation of both projections)."""
    rng = np.random.default_rng(201)
    N, C, Cp, H, W = 2, 5, 3, 4, 3
    x, p_in, a, lam, u, p_out = _proxy_case(rng, N, C, Cp, H, W)
    xp = np.zeros((N, Cp, H, W))
    for n in range(N):
        for q in range(Cp):
            for c in range(C):
                xp[n, q] += p_in[q, c] * x[n, c]
    yp = oracle.forward(xp, a, lam, u, 1, 15)
    y = np.zeros((N, C, H, W))
    for n in range(N):
        for c in range(C):
            for q in range(Cp):
                y[n, c] += p_out[c, q] * yp[n, q]
    assert np.abs(oracle.proxy_forward(x, p_in, a, lam, u, p_out, 1, 15) - y).max() <= 1e-12


def test_proxy_selecting_one_channel():
    """C_proxy = 1 with P_in = e_k^T and P_out = e_k: channel k is propagated alone, the others
    come out zero."""
    rng = np.random.default_rng(202)
    N, C, H, W, k = 1, 4, 5, 5, 2
    x, _, a, lam, u, _ = _proxy_case(rng, N, C, 1, H, W)
    p_in = np.zeros((1, C)); p_in[0, k] = 1.0
    p_out = np.zeros((C, 1)); p_out[k, 0] = 1.0
    y = oracle.proxy_forward(x, p_in, a, lam, u, p_out, 1, 15)
    assert np.abs(y[:, k:k + 1] - oracle.forward(x[:, k:k + 1], a, lam, u, 1, 15)).max() <= 1e-12
    assert np.all(np.delete(y, k, axis=1) == 0.0)


# ----------------------------------------------------------------------------- per-direction lambda / u
def _per_dir_case(rng, N, C, H, W, mask, wmode):
    x, a, lam, u = rand_case(rng, N, C, H, W, mask, wmode)
    D = bin(mask).count("1")
    lam_d = rng.uniform(0.0, 1.0, (D,) + x.shape)
    u_d = rng.standard_normal((D,) + x.shape)
    return x, a, lam_d, u_d


def test_per_direction_with_equal_slots_is_the_shared_form():
    rng = np.random.default_rng(300)
    x, a, lam, u = rand_case(rng, 1, 2, 5, 6, 15, 1)
    lam_d, u_d = np.stack([lam] * 4), np.stack([u] * 4)
    y = oracle.forward(x, a, lam_d, u_d, 1, 15, per_dir=1)
    assert np.abs(y - oracle.forward(x, a, lam, u, 1, 15)).max() <= 1e-12
    dy = rng.standard_normal(x.shape)
    gs = oracle.backward(x, a, lam, u, dy, 1, 15)
    gd = oracle.backward(x, a, lam_d, u_d, dy, 1, 15, per_dir=1)
    assert np.abs(gd[0] - gs[0]).max() <= 1e-12          # dx
    assert np.abs(gd[1] - gs[1]).max() <= 1e-12          # da
    assert np.abs(gd[2].sum(0) - gs[2]).max() <= 1e-12   # sum_d dlam_d = dlam
    assert np.abs(gd[3].sum(0) - gs[3]).max() <= 1e-12   # sum_d du_d = du


@pytest.mark.parametrize("mask", [15, 6, 9])
def test_per_direction_is_the_sum_of_single_direction_scans(mask):
    """y = sum_d u_d * h^d(lam_d x): each term is the single-direction scan with that slot's
    lambda and u (pins the slot order of the direction axis)."""
    rng = np.random.default_rng(310 + mask)
    x, a, lam_d, u_d = _per_dir_case(rng, 2, 2, 5, 7, mask, 0)
    y = oracle.forward(x, a, lam_d, u_d, 0, mask, per_dir=1)
    ref = np.zeros_like(x)
    for s, d in enumerate([d for d in (1, 2, 4, 8) if mask & d]):
        ref += oracle.forward(x, a[s:s + 1], lam_d[s], u_d[s], 0, d)
    assert np.abs(y - ref).max() <= 1e-12


@pytest.mark.parametrize("wmode", [0, 1])
@pytest.mark.parametrize("mask", [15, 5])
def test_per_direction_backward_finite_differences(wmode, mask):
    rng = np.random.default_rng(320 + mask + 10 * wmode)
    x, a, lam_d, u_d = _per_dir_case(rng, 1, 2, 4, 5, mask, wmode)
    dy = rng.standard_normal(x.shape)
    grads = oracle.backward(x, a, lam_d, u_d, dy, wmode, mask, per_dir=1)
    args = [x, a, lam_d, u_d]
    eps = 1e-6

    def loss():
        return float((dy * oracle.forward(*args, wmode, mask, per_dir=1)).sum())

    for gi in range(4):
        base = args[gi]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = base[idx]
            base[idx] = old + eps
            lp = loss()
            base[idx] = old - eps
            lm = loss()
            base[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        scale = max(1.0, np.abs(fd).max())
        assert np.abs(grads[gi] - fd).max() <= 1e-6 * scale, (gi, np.abs(grads[gi] - fd).max())
