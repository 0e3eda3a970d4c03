"""Pins for the oracle's online-anchor maps (attn_fwd_online).

The reading: key tiles in increasing key order, each anchored at the row's
running maximum after it ("Rowmax-H15 in FlashAttention-4 on B200", wiki
flowchart: QK tile -> row max (anchor) -> power-of-two weights -> PV), with
earlier accumulators carried over by 2^-k (Rowmax-PoT, k the rounded anchor
move) or exp(a_old - a_new) (K-interval fixed window, exact).  Each test
checks the recursive oracle against something else: the two-sweep maps
where both readings must agree, softmax, a closed form of every key's final
weight evaluated independently, a hand-worked row, and invariants.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A
from approximate_softmax_attention_b200 import inputs

LN2 = math.log(2.0)


def test_exact_online_is_softmax():
    d = inputs.draw(1, 2, 300, 64, seed=5, peaked=True)
    for causal in (False, True):
        got = A.attn_fwd_online(d["q"], d["k"], d["v"], causal, A.EXACT)
        q, k, v = (d[n].double() for n in ("q", "k", "v"))
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal)
        np.testing.assert_allclose(got["O"], ref.numpy(), atol=1e-12)
        s = (q @ k.transpose(-1, -2)) / 8.0
        if causal:
            s = s.masked_fill(torch.ones(300, 300, dtype=torch.bool).triu(1), -float("inf"))
        np.testing.assert_allclose(got["LSE"], torch.logsumexp(s, -1).numpy(), atol=1e-12)


@pytest.mark.parametrize("mode,K,rnd,below", [(A.ROWMAX_POT, 4, A.HARD, 0),
                                              (A.ROWMAX_POT, 4, A.HARD, 1),
                                              (A.KINTERVAL, 4, A.HARD, 0),
                                              (A.KINTERVAL, 16, A.INTERP, 0),
                                              (A.KINTERVAL, 4, A.INTERP, 1)])
def test_single_tile_equals_two_sweep(mode, K, rnd, below):
    """With every key in one tile the first anchor is the final maximum, so the
    online map is the two-sweep map."""
    d = inputs.draw(1, 2, 120, 64, seed=6, peaked=True)
    for causal in (False, True):
        on = A.attn_fwd_online(d["q"], d["k"], d["v"], causal, mode, K=K, rounding=rnd,
                               window=6.0, below_policy=below, want_idx=True)
        tw = A.attn_fwd(d["q"], d["k"], d["v"], causal, mode, K=K, calib=A.FIXED_WINDOW,
                        rounding=rnd, window=6.0, below_policy=below, want_idx=True)
        np.testing.assert_allclose(on["O"], tw["O"], atol=1e-13)
        np.testing.assert_allclose(on["LSE"], tw["LSE"], atol=1e-13)
        assert np.array_equal(on["idx"], tw["idx"])


def _one_row(scores, vals, D=4):
    """q, k, v of one query row whose scores are exactly `scores` (scale 1):
    q = e_0, k_j = scores[j] e_0."""
    S = len(scores)
    q = np.zeros((1, 1, S, D))
    q[0, 0, :, 0] = 1.0
    k = np.zeros((1, 1, S, D))
    k[0, 0, :, 0] = scores
    v = np.zeros((1, 1, S, D))
    v[0, 0, :, :] = np.asarray(vals)[:, None] * np.arange(1, D + 1)[None, :]
    return q, k, v


def test_max_in_first_tile_equals_two_sweep():
    """Keys in decreasing score order: the anchor never moves."""
    rng = np.random.default_rng(0)
    s = np.sort(rng.normal(0, 2.0, 9))[::-1]
    q, k, v = _one_row(s, rng.normal(size=9))
    for mode, kw in [(A.ROWMAX_POT, {}), (A.KINTERVAL, dict(K=4, rounding=A.INTERP))]:
        on = A.attn_fwd_online(q, k, v, False, mode, scale=1.0, tile=3, **kw)
        tw = A.attn_fwd(q, k, v, False, mode, scale=1.0, calib=A.FIXED_WINDOW, **kw)
        np.testing.assert_allclose(on["O"][0, 0, 0], tw["O"][0, 0, 0], atol=1e-13)
        np.testing.assert_allclose(on["LSE"][0, 0, 0], tw["LSE"][0, 0, 0], atol=1e-13)


def test_hand_worked_pot_row():
    """Scores 0, -0.6, 0.6, -5 (log2 units), tiles of two keys.  Tile 0:
    anchor 0, exponents 0 and rne(0.6) = 1.  Tile 1: anchor 0.6, move
    rne(0.6) = 1 halves the carried weights; exponents 0 and rne(5.6) = 6.
    Final weights 1/2, 1/4, 1, 1/64 -- where the two-sweep map gives 1/2,
    1/2 (rne(1.2) = 1), 1, 1/64."""
    x = np.array([0.0, -0.6, 0.6, -5.0])
    vals = np.array([1.0, 2.0, 3.0, 4.0])
    q, k, v = _one_row(x * LN2, vals)
    got = A.attn_fwd_online(q, k, v, False, A.ROWMAX_POT, scale=1.0, tile=2, want_idx=True)
    w = np.array([0.5, 0.25, 1.0, 1.0 / 64])
    # every row of this one-row-per-position layout sees the same scores
    np.testing.assert_allclose(got["O"][0, 0, 0, 0], (w * vals).sum() / w.sum(), rtol=1e-14)
    np.testing.assert_allclose(got["LSE"][0, 0, 0], 0.6 * LN2 + math.log(w.sum()),
                               rtol=1e-14)
    assert got["idx"][0, 0, 0].tolist() == [0, 1, 0, 6]
    two = A.attn_fwd(q, k, v, False, A.ROWMAX_POT, scale=1.0)
    w2 = np.array([0.5, 0.5, 1.0, 1.0 / 64])
    np.testing.assert_allclose(two["O"][0, 0, 0, 0], (w2 * vals).sum() / w2.sum(), rtol=1e-14)


def _closed_form(s, mode, K, rounding, W, N, below, tile):
    """Every key's final weight written out directly (no recursion): the
    anchor of key j's tile is the prefix maximum up to the end of that tile;
    PoT carries 2^-(sum of the rounded anchor moves after the tile), the
    fixed-window grid exp(a_tile - a_last)."""
    S = len(s)
    T = (S + tile - 1) // tile
    a = [max(s[:min(S, (t + 1) * tile)]) for t in range(T)]
    moves = [0] + [int(np.rint((a[t] - a[t - 1]) / LN2)) for t in range(1, T)]
    w = []
    for j in range(S):
        t = j // tile
        if mode == A.ROWMAX_POT:
            n = int(np.rint((a[t] - s[j]) / LN2))
            loc = 0.0 if (below and n > N) else 2.0 ** -min(n, N)
            w.append(loc * 2.0 ** -sum(moves[t + 1:]))
        else:
            dl = W / K
            u = (s[j] - (a[t] - W)) / dl
            if below and u < 0:
                loc = 0.0
            else:
                u = min(max(u, 0.0), K)
                if rounding == A.HARD:
                    loc = math.exp(-(K - int(np.rint(u))) * dl)
                else:
                    kk = min(int(math.floor(u)), K - 1)
                    f = u - kk
                    loc = (1 - f) * math.exp(-(K - kk) * dl) + f * math.exp(-(K - kk - 1) * dl)
            w.append(loc * math.exp(a[t] - a[-1]))
    return np.array(w), a[-1]


@pytest.mark.parametrize("mode,K,rnd,below", [(A.ROWMAX_POT, 4, A.HARD, 0),
                                              (A.ROWMAX_POT, 4, A.HARD, 1),
                                              (A.KINTERVAL, 2, A.HARD, 0),
                                              (A.KINTERVAL, 4, A.INTERP, 0),
                                              (A.KINTERVAL, 3, A.INTERP, 1)])
@pytest.mark.parametrize("tile", [1, 2, 3])
def test_closed_form_tiny_rows(mode, K, rnd, below, tile):
    rng = np.random.default_rng(100 + tile + 7 * K + below)
    for _ in range(40):
        S = int(rng.integers(1, 8))
        s = rng.normal(0, 2.5, S)
        vals = rng.normal(size=S)
        q, k, v = _one_row(s, vals)
        got = A.attn_fwd_online(q, k, v, False, mode, K=K, rounding=rnd, scale=1.0,
                                window=3.0, pot_floor=5, below_policy=below, tile=tile)
        w, alast = _closed_form(s, mode, K, rnd, 3.0, 5, below, tile)
        if w.sum() == 0:
            continue
        np.testing.assert_allclose(got["O"][0, 0, 0, 0], (w * vals).sum() / w.sum(),
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got["LSE"][0, 0, 0], alast + math.log(w.sum()), atol=1e-12)
        if mode == A.ROWMAX_POT:
            nz = w[w > 0]
            assert np.all(np.exp2(np.rint(np.log2(nz))) == nz)       # powers of two


def test_shift_and_within_tile_permutation_invariance():
    d = inputs.draw(1, 1, 256, 64, seed=8, peaked=True)
    q, k, v = (d[n].double().numpy() for n in ("q", "k", "v"))
    # a shift of every score of a row by 0.37: one extra component
    q2 = np.concatenate([q, np.ones((1, 1, 256, 1))], -1)
    k2 = np.concatenate([k, np.full((1, 1, 256, 1), 0.37 * 8.0)], -1)
    for mode, kw in [(A.ROWMAX_POT, {}), (A.KINTERVAL, dict(K=16, rounding=A.INTERP))]:
        base = A.attn_fwd_online(q, k, v, False, mode, scale=1.0 / 8.0, **kw)
        sh = A.attn_fwd_online(q2, k2, v, False, mode, scale=1.0 / 8.0, **kw)
        np.testing.assert_allclose(sh["O"], base["O"], atol=1e-12)
        np.testing.assert_allclose(sh["LSE"], base["LSE"] + 0.37, atol=1e-12)
        perm = np.concatenate([np.random.default_rng(1).permutation(128),
                               128 + np.random.default_rng(2).permutation(128)])
        pm = A.attn_fwd_online(q, k[:, :, perm], v[:, :, perm], False, mode, scale=1.0 / 8.0,
                               **kw)
        np.testing.assert_allclose(pm["O"], base["O"], atol=1e-12)


def test_nonfinite_rows():
    q, k, v = _one_row(np.array([0.0, -np.inf, -1.0, np.nan]), np.arange(4.0))
    got = A.attn_fwd_online(q, k, v, False, A.ROWMAX_POT, scale=1.0, tile=2)
    assert np.isnan(got["O"]).all()           # the NaN reaches the anchor
    q, k, v = _one_row(np.array([0.0, -np.inf, -1.0, -2.0]), np.arange(4.0))
    got = A.attn_fwd_online(q, k, v, False, A.EXACT, scale=1.0, tile=2)
    w = np.exp([0.0, -np.inf, -1.0, -2.0])
    np.testing.assert_allclose(got["O"][0, 0, 0, 0], (w * np.arange(4.0)).sum() / w.sum())
