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


def bf16_step(x):
    """The bf16 spacing at |x| (8 significand bits)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def to_bf16(x):
    """x rounded to bf16 (round to nearest even), as float64."""
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def check_bf16_output(got, want, tol_max=1e-2, tol_mean=1e-3, what=""):
    """A bf16 kernel output against the fp64 oracle rounded to the same bf16
    format: |got - bf16(want)| <= tol_max everywhere, except that where one
    bf16 step exceeds tol_max (|want| >= 2) the two may sit on adjacent bf16
    codes (two values a hair apart can round to neighbours); and the mean
    |got - want| <= tol_mean."""
    g = np.asarray(got, dtype=np.float64)
    w = np.asarray(want, dtype=np.float64)
    d = np.abs(g - to_bf16(w))
    allow = np.maximum(tol_max, bf16_step(w))
    ratio = d / allow
    worst = float(np.max(ratio))
    mean = float(np.abs(g - w).mean())
    at = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
    assert worst <= 1.0 and mean <= tol_mean, (what, float(d.max()), worst, mean, tuple(
        int(i) for i in at), float(g[at]), float(w[at]), int((ratio > 1.0).sum()))
    return float(d.max()), mean


def check_decisions(d, got_idx, causal, mode, K, calib, rounding, window, heads=None,
                    row_block=1024, below_policy=0):
    """Kernel decisions (the forward's debug dump) against fp64 rounding:
    agreement >= 99.9 % and every mismatch within 1e-3 of a boundary; masked
    keys read -1 (or the buffer's fill value -7 in key tiles the kernel never
    visits).  ``got_idx`` is the [B,H,S,S] dump, or a dict {(b, h): [S,S]}
    holding only the heads checked.  below_policy 1: flushed keys read -2 on
    both sides."""
    if mode == A.EXACT:
        return
    q = d["q"].double().numpy() * d["q_descale"]
    k = d["k"].double().numpy() * d["k_descale"]
    B, H, S, D = q.shape
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    total = bad = 0
    for (b, h) in heads:
        g_all = got_idx[(b, h)] if isinstance(got_idx, dict) else got_idx[b, h]
        for r0 in range(0, S, row_block):
            rr = np.arange(r0, min(S, r0 + row_block))
            s = (q[b, h, rr] @ k[b, h].T) / math.sqrt(D)
            valid = (np.arange(S)[None, :] <= rr[:, None]) if causal \
                else np.ones((len(rr), S), bool)
            m = A._map_rows(s, valid, mode, K, calib, rounding, window, 15, below_policy)
            ref = m["idx"]
            dist = boundary_distance_rows(s, valid, mode, K, calib, rounding, window)
            g = np.asarray(g_all[rr], dtype=np.int64)
            assert np.all((g[~valid] == -1) | (g[~valid] == -7))
            mism = (g != ref) & valid
            assert np.all(dist[mism] <= 1e-3), (b, h, np.argwhere(mism & (dist > 1e-3))[:5])
            bad += int(mism.sum())
            total += int(valid.sum())
    assert bad <= 1e-3 * total, (bad, total)
    return bad, total
