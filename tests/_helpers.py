"""Shared test helpers: run the oracle on the same inputs the GPU reads, and
measure how far each fp64 grid coordinate sits from its rounding boundary."""

from __future__ import annotations

import math

import numpy as np

import oracle
from oracle import attention as A


def boundary_distance_rows(s64, valid, mode, K, calib, rounding, window):
    """Distance of each element's fp64 coordinate (u for K-interval, log2
    units for PoT) to the nearest boundary where its decision changes."""
    m = A._map_rows(s64, valid, mode, K, calib, rounding, window, 15, 0)
    if mode == A.ROWMAX_POT:
        x = m["x"]
        return np.abs(x - np.floor(x) - 0.5)
    if mode == A.EXACT:
        return np.full(s64.shape, np.inf)
    u = m["u"]
    if rounding == A.HARD:
        d = np.abs(u - np.floor(u) - 0.5)
    else:
        fr = u - np.floor(u)
        d = np.minimum(fr, 1 - fr)
    # fixed-window keys below the window sit on the clamp: any coordinate
    # under 0 gives node 0, so only the clamp edge itself is a boundary
    return d


def scores64(q, k, c, causal, rows=None):
    """fp64 scores of (b, h) slices; q, k are float64 [S, D]."""
    S = k.shape[0]
    rr = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    s = c * (q[rr] @ k.T)
    if causal:
        valid = np.arange(S)[None, :] <= rr[:, None]
    else:
        valid = np.ones_like(s, dtype=bool)
    return s, valid


def default_c(D, q_descale=1.0, k_descale=1.0, scale=None):
    sc = 1.0 / math.sqrt(D) if scale is None else scale
    return float(np.float32(np.float32(sc) * np.float32(q_descale)) * np.float32(k_descale))


def err_stats(got, want):
    d = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(want, dtype=np.float64))
    return float(d.max()), float(d.mean())
