"""Closed-form (matrix) form of the GSPN line scan, for tiny maps.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

"GSPN-2: Efficient Parallel Sequence Modeling" (paper notes), end of section
"Optimisation 2: compact channel propagation", reads the unrolled recurrence as linear
attention: stacking the lines of one scan, ``H = G X`` with ``G`` block lower-triangular,
``G_ii = I`` and ``G_ij = w_i w_{i-1} ... w_{j+1}`` for ``j < i``. This module builds that
``G`` explicitly with dense NumPy matrices, and maps directions onto the top->bottom scan
with array flips and transposes (not index arithmetic), so it shares neither code nor
formulation with ``gspn_oracle.c``.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit

_FLIPS = {
    # direction bit: (image -> scan-major array, scan-major array -> image)
    1: (lambda A: A, lambda S: S),                                    # TB
    2: (lambda A: A[::-1, :], lambda S: S[::-1, :]),                 # BT
    4: (lambda A: A.T, lambda S: S.T),                                # LR
    8: (lambda A: A[:, ::-1].T, lambda S: S.T[:, ::-1]),              # RL
}


def line_matrix(logits3: np.ndarray) -> np.ndarray:
    """Dense M x M propagation matrix of one line from its (3, M) logits.

    Row j has entries at columns j-1, j, j+1 (those inside [0, M)), equal to the sigmoid of
    the corresponding logit divided by the sum of the in-range sigmoids.
    """
    M = logits3.shape[1]
    Wm = np.zeros((M, M))
    for j in range(M):
        cols = [j + k - 1 for k in range(3)]
        s = np.array([expit(logits3[k, j]) if 0 <= cols[k] < M else 0.0 for k in range(3)])
        s = s / s.sum()
        for k in range(3):
            if 0 <= cols[k] < M:
                Wm[j, cols[k]] = s[k]
    return Wm


def g_matrix(line_mats) -> np.ndarray:
    """Block lower-triangular G (L*M x L*M) with G_ii = I, G_ij = W_i ... W_{j+1}."""
    L = len(line_mats)
    M = line_mats[0].shape[0]
    G = np.zeros((L * M, L * M))
    for j in range(L):
        P = np.eye(M)
        for i in range(j, L):
            if i > j:
                P = line_matrix_product(line_mats[i], P)
            G[i * M:(i + 1) * M, j * M:(j + 1) * M] = P
    return G


def line_matrix_product(Wi: np.ndarray, P: np.ndarray) -> np.ndarray:
    return Wi @ P


def scan_plane(z: np.ndarray, logits3: np.ndarray, d: int) -> np.ndarray:
    """One direction on one H x W plane: returns h in image coordinates.

    ``z`` is (H, W); ``logits3`` is (3, H, W) in image coordinates.
    """
    to_scan, to_img = _FLIPS[d]
    zs = np.ascontiguousarray(to_scan(z))                    # (L, M)
    As = np.stack([np.ascontiguousarray(to_scan(logits3[k])) for k in range(3)])  # (3, L, M)
    L, M = zs.shape
    mats = [line_matrix(As[:, i, :]) for i in range(L)]
    G = g_matrix(mats)
    hs = (G @ zs.reshape(-1)).reshape(L, M)
    return np.ascontiguousarray(to_img(hs))


def forward(x, a, lam, u, wmode: int = 0, mask: int = 15) -> np.ndarray:
    """y = u * sum_d (G_d applied to lam * x), by explicit matrices. Tiny maps only."""
    x, a, lam, u = (np.asarray(t, dtype=np.float64) for t in (x, a, lam, u))
    N, C, H, W = x.shape
    y = np.zeros_like(x)
    for n in range(N):
        for c in range(C):
            z = lam[n, c] * x[n, c]
            acc = np.zeros((H, W))
            slot = 0
            for d in (1, 2, 4, 8):
                if mask & d:
                    acc += scan_plane(z, a[slot, n, 0 if wmode else c], d)
                    slot += 1
            y[n, c] = u[n, c] * acc
    return y


def jacobian_z(logits3: np.ndarray, d: int, H: int, W: int) -> np.ndarray:
    """(HW x HW) matrix mapping z (image, flattened) to h^d (image, flattened)."""
    J = np.zeros((H * W, H * W))
    for p in range(H * W):
        e = np.zeros(H * W)
        e[p] = 1.0
        J[:, p] = scan_plane(e.reshape(H, W), logits3, d).reshape(-1)
    return J
