"""Comparison helpers for GPU-vs-oracle parity (no method arithmetic here).

Tolerances follow the stated bar: codes bit-exact except coordinates whose
oracle rotated value lies within 1e-5 (relative) of the decision boundary
between the two indices -- relative to max(|B|, 1/sqrt(d_pad)) because the
middle boundary is 0 -- and those must be fewer than 1e-4 of all
coordinates; QJL sign bits exact except where |z_i| <= 1e-5 rho; norms,
scores and attention outputs within 1e-3 relative.
"""
import math

import numpy as np

from oracle import tq_oracle as o

CODE_WINDOW = 1e-5
CODE_WINDOW_FRACTION = 1e-4
REL_TOL = 1e-3


def u32(t):
    """torch int32 tensor of packed words -> numpy uint32."""
    return t.detach().cpu().numpy().view(np.uint32)


def check_codes(gpu_idx, ora_idx, ora_y, boundaries, d_pad, what="codes"):
    """Returns (n_mismatch, bad_rows mask).  Asserts every mismatch is a
    neighbouring cell inside the boundary window and the count is small."""
    gpu_idx = np.asarray(gpu_idx)
    ora_idx = np.asarray(ora_idx)
    mism = gpu_idx != ora_idx
    n = int(mism.sum())
    if n:
        a = gpu_idx[mism]
        b = ora_idx[mism]
        y = ora_y[mism]
        assert np.all(np.abs(a - b) == 1), f"{what}: mismatch by more than one cell"
        B = boundaries[np.minimum(a, b)]
        win = CODE_WINDOW * np.maximum(np.abs(B), 1.0 / math.sqrt(d_pad))
        assert np.all(np.abs(y - B) <= win), f"{what}: mismatch outside the boundary window"
    assert n <= max(CODE_WINDOW_FRACTION * gpu_idx.size, 0), \
        f"{what}: {n} window mismatches of {gpu_idx.size}"
    return n, mism.reshape(mism.shape[0], -1).any(axis=1)


def check_signs(gpu_words, ora_words, ora_z, ora_rho, m, skip_rows=None):
    g = o.unpack_signs(gpu_words, m)
    r = o.unpack_signs(ora_words, m)
    mism = g != r
    if skip_rows is not None:
        mism[skip_rows] = False
    if mism.any():
        z = ora_z[mism]
        rho = np.broadcast_to(ora_rho[:, None], ora_z.shape)[mism]
        assert np.all(np.abs(z) <= CODE_WINDOW * rho), "sign bit flipped outside the window"
    return int(mism.sum())


def rel_err(a, b, floor):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.abs(a - b) / np.maximum(np.abs(b), floor)


def assert_close_rel(gpu, ora, floor, tol=REL_TOL, what="values", mask=None):
    e = rel_err(gpu, ora, floor)
    if mask is not None:
        e = e[mask]
    worst = float(e.max()) if e.size else 0.0
    assert worst <= tol, f"{what}: max relative error {worst:.3g} > {tol}"
    return worst
