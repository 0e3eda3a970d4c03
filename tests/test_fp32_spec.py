"""Pins for the C restatement of the fp32 weight-map specification.

The fp32 spec is the bit-exact target of the GPU map (the fused forward's
own per-element arithmetic on raw products r, with the score scale c folded
into one fused multiply-add).  Here it is checked against the fp64 oracle
(itself pinned in test_oracle_pins.py) on the scores s = c r: decisions agree
except within a small distance of a rounding boundary (where fp32 and fp64
may legitimately round differently), and weights agree to fp32 accuracy.
Its own exp is checked against float64 exp over the range the grid uses.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import attention as A
from oracle import spec


def test_spec_exp_accuracy():
    x = np.linspace(-86.0, 0.0, 400001, dtype=np.float32)   # n >= -125: no flush
    y = spec.spec_exp(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(y - ref) / ulp) < 1.0          # faithful rounding
    assert spec.spec_exp(np.zeros(1, np.float32))[0] == 1.0
    assert spec.spec_exp(np.array([-200.0, -np.inf], np.float32)).tolist() == [0.0, 0.0]


def _boundary_distance(s64, valid, mode, K, calib, rounding, W):
    """Distance (in u units, or log2 units for PoT) from each element's fp64
    coordinate to the nearest rounding boundary of its map."""
    hi = np.where(valid, s64, -np.inf).max(1, keepdims=True)
    lo = np.where(valid, s64, np.inf).min(1, keepdims=True)
    if mode in (A.TRUNCATED, A.UNIFORM):
        return np.abs(s64 - (hi - 4.0)) / math.log(2.0)
    if mode == A.ROWMAX_POT:
        x = (hi - s64) * A.LOG2E
        return np.abs(x - np.floor(x) - 0.5)
    lo_c = lo if calib == A.MINMAX else hi - W
    u = np.clip((s64 - lo_c) / ((hi - lo_c) / K), 0, K)
    if rounding == A.HARD:
        return np.abs(u - np.floor(u) - 0.5)
    fr = u - np.floor(u)
    return np.minimum(fr, 1 - fr)


CASES = [(A.EXACT, 4, 0, 1, 0), (A.ROWMAX_POT, 4, 0, 1, 0), (A.ROWMAX_POT, 4, 0, 1, 1),
         (A.TRUNCATED, 4, 0, 1, 0), (A.UNIFORM, 4, 0, 1, 0)] + \
    [(A.KINTERVAL, K, c, r, 0) for K in (1, 4, 16, 64) for c in (0, 1) for r in (0, 1)] + \
    [(A.KINTERVAL, 4, 1, 1, 1), (A.KINTERVAL, 16, 1, 0, 1)]

# score scales: none, 1/sqrt(128), and 1/sqrt(128) times two e4m3 descales
SCALES = [1.0, 0.08838834764831845, 0.08838834764831845 * 0.0121 * 0.0098]


@pytest.mark.parametrize("c", SCALES)
@pytest.mark.parametrize("mode,K,calib,rounding,below", CASES)
def test_spec_matches_fp64_oracle(mode, K, calib, rounding, below, c):
    rng = np.random.default_rng(31 + K + 100 * mode + 10 * calib + rounding)
    R, S = 256, 300
    c32 = np.float32(c)
    # raw products whose scores c*r spread like N(0, 3^2)
    r32 = (rng.normal(0, 3.0, size=(R, S)) / float(c32)).astype(np.float32)
    vl = rng.integers(1, S + 1, size=R).astype(np.int32)
    vl[:4] = [1, 2, S, S]
    valid = np.arange(S)[None, :] < vl[:, None]
    W = 6.0
    w32, idx32, hi32, lo32 = spec.spec_map(r32, vl, mode, K=K, calib=calib, rounding=rounding,
                                           window=W, pot_floor=15, below_policy=below, c=c)
    s64 = float(c32) * r32.astype(np.float64)
    w64, idx64, hi64, _ = oracle.weight_map(s64, valid, mode, K=K, calib=calib,
                                            rounding=rounding, window=W, pot_floor=15,
                                            below_policy=below)
    # hi = c * max r rounded once to fp32
    assert np.array_equal(hi32, hi64.astype(np.float32))
    if mode in (A.EXACT, A.TRUNCATED):
        # the spec gives the exponent x of 2^x (-inf for a cut key)
        w32 = np.where(valid, np.exp2(w32.astype(np.float64)), 0.0)
    dist = _boundary_distance(s64, valid, mode, K, calib, rounding, W)
    agree = idx32 == idx64
    assert np.all(agree | (dist < 1e-4)), np.argwhere(~agree & (dist >= 1e-4))[:5]
    assert agree.mean() > 0.999
    ok = agree & valid
    # weights are anchored at 1 for the row max; fp32 evaluation of the grid
    # coordinate (slope c*K/a rounded once, then one fused multiply-add)
    # carries an absolute error of a few ulp of |r * c * K / a|, which the
    # interpolation slope (<= 1 per unit of u) carries into w
    np.testing.assert_allclose(w32[ok], w64[ok], rtol=4e-6, atol=8e-6)
    assert np.all(w32[~valid] == 0) and np.all(idx32[~valid] == -1)


def test_spec_nan_propagates_to_the_row_statistics():
    r = np.array([[1.0, np.nan, -2.0], [1.0, 0.5, -2.0]], np.float32)
    vl = np.array([3, 3], np.int32)
    _, _, hi, lo = spec.spec_map(r, vl, A.KINTERVAL, K=4, calib=A.MINMAX, rounding=A.HARD)
    assert np.isnan(hi[0]) and np.isnan(lo[0])
    assert hi[1] == 1.0 and lo[1] == -2.0


def test_spec_pot_is_exact_power_of_two_and_one_at_max():
    rng = np.random.default_rng(3)
    s = rng.normal(0, 4.0, size=(64, 128)).astype(np.float32)
    vl = np.full(64, 128, np.int32)
    w, idx, hi, _ = spec.spec_map(s, vl, A.ROWMAX_POT, pot_floor=15)
    assert np.all(w[np.arange(64), s.argmax(1)] == 1.0)
    assert np.all(w == np.exp2(-idx.astype(np.float64)).astype(np.float32))
    assert idx.min() >= 0 and idx.max() <= 15


def test_spec_hard_hits_grid_and_degenerate_rows():
    s = np.array([[0.5, 0.5, 0.5], [0.0, -1.5, -4.0]], np.float32)
    vl = np.array([3, 3], np.int32)
    w, idx, _, _ = spec.spec_map(s, vl, A.KINTERVAL, K=4, calib=A.MINMAX, rounding=A.HARD)
    assert w[0].tolist() == [1.0, 1.0, 1.0]
    assert idx[1].tolist() == [4, 2, 0]          # 2.5 rounds to even
    w2, idx2, _, _ = spec.spec_map(s, vl, A.KINTERVAL, K=4, calib=A.MINMAX, rounding=A.INTERP)
    assert idx2[1].tolist() == [3, 2, 0]
