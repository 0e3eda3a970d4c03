"""Pins for the fp64 oracle's forward maps and attention forward.

Each test checks the oracle against something other than itself: hand-worked
decisions (tests/golden/hand_example.json), an independent brute-force
formulation on tiny rows (nearest node by distance, interpolant by segment
search, nearest power of two by scanning), torch's softmax attention for the
exact map, and invariants the definitions fix.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A
from approximate_softmax_attention_b200 import inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def _load_hand():
    with open(os.path.join(HERE, "golden", "hand_example.json")) as f:
        return json.load(f)


def _expected_from_decisions(case, s):
    K = case["K"]
    n = len(s)
    if case["mode"] == A.EXACT:
        hi = max(s)
        return [math.exp(x - hi) for x in s]
    if case["mode"] == A.ROWMAX_POT:
        return [0.0 if e == -2 else 2.0 ** (-e) for e in case["exponents"]]
    d = case["delta"]
    if case["rounding"] == A.HARD:
        return [0.0 if m == -2 else math.exp(-(K - m) * d) for m in case["nodes"]]
    out = []
    for kk, f in zip(case["lower"], case["frac"]):
        out.append((1 - f) * math.exp(-(K - kk) * d) + f * math.exp(-(K - kk - 1) * d))
    assert len(out) == n
    return out


@pytest.mark.parametrize("row_i,case_i", [(r, c) for r, row in enumerate(_load_hand()["rows"])
                                          for c in range(len(row["cases"]))])
def test_hand_worked_decisions(row_i, case_i):
    row = _load_hand()["rows"][row_i]
    case = row["cases"][case_i]
    s = np.array([row["scores"]])
    valid = np.ones_like(s, dtype=bool)
    w, idx, hi, lo = oracle.weight_map(
        s, valid, case["mode"], K=case["K"], calib=case["calib"],
        rounding=case["rounding"], window=case["window"],
        pot_floor=case.get("pot_floor", 15), below_policy=case["below"])
    exp_w = np.array(_expected_from_decisions(case, row["scores"]))
    np.testing.assert_allclose(w[0], exp_w, rtol=1e-14, atol=1e-300)
    if case["mode"] == A.KINTERVAL:
        want = case["nodes"] if case["rounding"] == A.HARD else case["lower"]
        assert list(idx[0]) == want
    if case["mode"] == A.ROWMAX_POT:
        assert list(idx[0]) == case["exponents"]


def test_hand_example_probabilities():
    # p = w / sum(w) for the first hand row, the closed forms written out
    e = math.exp
    s = np.array([[0.0, -1.0, -2.5, -4.0]])
    v = np.ones_like(s, dtype=bool)
    cases = {
        (A.KINTERVAL, 0, 1): [1, e(-1), e(-2), e(-4)],
        (A.KINTERVAL, 0, 0): [1, e(-1), (e(-3) + e(-2)) / 2, e(-4)],
        (A.KINTERVAL, 1, 1): [1, 1, e(-2), e(-4)],
        (A.ROWMAX_POT, 0, 1): [1, 0.5, 1 / 16, 1 / 64],
        (A.EXACT, 0, 1): [1, e(-1), e(-2.5), e(-4)],
    }
    for (mode, cal, rnd), w in cases.items():
        got, _, _, _ = oracle.weight_map(s, v, mode, K=4, calib=cal, rounding=rnd)
        p = got[0] / got[0].sum()
        w = np.array(w)
        np.testing.assert_allclose(p, w / w.sum(), rtol=1e-13)


# ---------------------------------------------------------------- brute force

def _bf_weights(s, mode, K, calib, rounding, W, N, below):
    """Independent formulation: nearest node by distance in score space,
    interpolant by segment search, nearest power of two by scanning."""
    hi = max(s)
    if mode == A.EXACT:
        return [math.exp(x - hi) for x in s]
    if mode == A.ROWMAX_POT:
        out = []
        for x in s:
            lx = (x - hi) / math.log(2.0)          # log2 of the exact weight
            best, bd = None, None
            for n in range(0, 200):
                dd = abs(lx + n)
                if bd is None or dd < bd - 1e-12 or (abs(dd - bd) <= 1e-12 and n % 2 == 0):
                    best, bd = n, dd
            if best > N:
                out.append(0.0 if below else 2.0 ** (-N))
            else:
                out.append(2.0 ** (-best))
        return out
    lo = min(s) if calib == A.MINMAX else hi - W
    if hi - lo <= 0:
        return [1.0] * len(s)
    nodes = [lo + k * (hi - lo) / K for k in range(K + 1)]
    vals = [math.exp(t - hi) for t in nodes]
    out = []
    for x in s:
        if below and calib == A.FIXED_WINDOW and x < lo:
            out.append(0.0)
            continue
        if rounding == A.HARD:
            best, bd = None, None
            for k, t in enumerate(nodes):
                dd = abs(x - t)
                if bd is None or dd < bd - 1e-12 or (abs(dd - bd) <= 1e-12 and k % 2 == 0):
                    best, bd = k, dd
            out.append(vals[best])
        else:
            xc = min(max(x, nodes[0]), nodes[-1])
            for k in range(K):
                if nodes[k] <= xc <= nodes[k + 1]:
                    t = (xc - nodes[k]) / (nodes[k + 1] - nodes[k])
                    out.append(vals[k] + t * (vals[k + 1] - vals[k]))
                    break
    return out


@pytest.mark.parametrize("mode,K,calib,rounding,below", [
    (A.EXACT, 4, 0, 1, 0),
    (A.ROWMAX_POT, 4, 0, 1, 0), (A.ROWMAX_POT, 4, 0, 1, 1),
] + [(A.KINTERVAL, K, c, r, b) for K in (1, 2, 3, 4) for c in (0, 1) for r in (0, 1)
     for b in (0, 1) if not (b == 1 and c == 0)])
def test_brute_force_tiny_rows(mode, K, calib, rounding, below):
    rng = np.random.default_rng(1000 + 97 * mode + 13 * K + 5 * calib + 3 * rounding + below)
    W, N = 3.0, 6
    for L in range(1, 7):
        for _ in range(20):
            s = rng.normal(0, 2.5, size=L)
            w, _, _, _ = oracle.weight_map(s[None, :], np.ones((1, L), bool), mode, K=K,
                                           calib=calib, rounding=rounding, window=W,
                                           pot_floor=N, below_policy=below)
            bf = _bf_weights(list(s), mode, K, calib, rounding, W, N, below)
            np.testing.assert_allclose(w[0], bf, rtol=1e-12, atol=1e-15)


def test_brute_force_attention_tiny():
    # full attention (causal and not) with python loops over rows and keys
    rng = np.random.default_rng(7)
    B, H, S, D = 1, 2, 6, 3
    q = rng.normal(size=(B, H, S, D))
    k = rng.normal(size=(B, H, S, D))
    v = rng.normal(size=(B, H, S, D))
    for causal in (False, True):
        for (mode, cal, rnd) in [(0, 0, 1), (1, 0, 1), (1, 0, 0), (1, 1, 1), (1, 1, 0), (2, 0, 1)]:
            res = oracle.attn_fwd(q, k, v, causal, mode, K=3, calib=cal, rounding=rnd,
                                  window=2.0, pot_floor=5)
            for h in range(H):
                for r in range(S):
                    n = r + 1 if causal else S
                    s = [sum(q[0, h, r, d] * k[0, h, j, d] for d in range(D)) / math.sqrt(D)
                         for j in range(n)]
                    w = _bf_weights(s, mode, 3, cal, rnd, 2.0, 5, 0)
                    Z = sum(w)
                    o = [sum(w[j] / Z * v[0, h, j, d] for j in range(n)) for d in range(D)]
                    np.testing.assert_allclose(res["O"][0, h, r], o, rtol=1e-11, atol=1e-13)
                    assert abs(res["LSE"][0, h, r] - (max(s) + math.log(Z))) < 1e-11
                    assert res["argmax"][0, h, r] == int(np.argmax(s))
                    assert res["argmin"][0, h, r] == int(np.argmin(s))


# ------------------------------------------------------------ library routine

@pytest.mark.parametrize("causal", [False, True])
def test_exact_mode_is_torch_softmax_attention(causal):
    g = torch.Generator().manual_seed(3)
    B, H, S, D = 2, 3, 40, 16
    q = torch.randn(B, H, S, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, H, S, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, H, S, D, generator=g, dtype=torch.float64)
    res = oracle.attn_fwd(q, k, v, causal, A.EXACT)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal)
    np.testing.assert_allclose(res["O"], ref.numpy(), rtol=1e-12, atol=1e-13)
    sc = (q @ k.transpose(-1, -2)) / math.sqrt(D)
    if causal:
        sc = sc.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(res["LSE"], torch.logsumexp(sc, -1).numpy(), rtol=1e-13)


# ------------------------------------------------------------------ invariants

def _rand_scores(seed, R=64, S=97, spread=3.0):
    rng = np.random.default_rng(seed)
    return rng.normal(0, spread, size=(R, S)), np.ones((R, S), bool)


def test_pot_invariants():
    s, v = _rand_scores(11)
    for N in (4, 15):
        w, idx, hi, _ = oracle.weight_map(s, v, A.ROWMAX_POT, pot_floor=N)
        am = np.argmax(s, axis=1)
        assert np.all(w[np.arange(len(s)), am] == 1.0)
        n = -np.log2(w)
        assert np.all(n == np.round(n)) and np.all(n >= 0) and np.all(n <= N)
        assert np.all(idx == n)


@pytest.mark.parametrize("calib", [0, 1])
def test_hard_rounding_hits_only_grid_values(calib):
    s, v = _rand_scores(12)
    for K in (1, 4, 16):
        w, idx, hi, lo = oracle.weight_map(s, v, A.KINTERVAL, K=K, calib=calib, rounding=A.HARD,
                                           window=6.0)
        lo_c = lo if calib == 0 else hi - 6.0
        g = oracle.kint_grid(K, (hi - lo_c) / K)
        for r in range(len(s)):
            assert set(np.unique(w[r])).issubset(set(g[r]))
        assert np.all(w[np.arange(len(s)), np.argmax(s, 1)] == 1.0)


@pytest.mark.parametrize("mode,calib,rnd", [(0, 0, 1), (1, 0, 1), (1, 0, 0), (1, 1, 1), (1, 1, 0), (2, 0, 1)])
def test_rows_sum_to_one_shift_and_permutation(mode, calib, rnd):
    rng = np.random.default_rng(5)
    B, H, S, D = 1, 2, 33, 8
    q = rng.normal(size=(B, H, S, D))
    k = rng.normal(size=(B, H, S, D))
    v = np.eye(S)[None, None].repeat(H, 1)[..., :S]          # O row = p row
    kw = dict(K=4, calib=calib, rounding=rnd, window=4.0)
    res = oracle.attn_fwd(q, k, v, False, mode, **kw)
    P = res["O"]
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=1e-13)
    assert np.all(P >= 0)
    # permutation equivariance of keys
    perm = rng.permutation(S)
    res2 = oracle.attn_fwd(q, k[:, :, perm], v[:, :, perm], False, mode, **kw)
    np.testing.assert_allclose(res2["O"], P, rtol=1e-12, atol=1e-15)
    # shift invariance of the maps: add a constant to every score of a row
    s, valid = A.row_scores(q[0, 0], k[0, 0], 1 / math.sqrt(D), 0, False)
    w1, _, _, _ = oracle.weight_map(s, valid, mode, **kw)
    w2, _, _, _ = oracle.weight_map(s + 2.75, valid, mode, **kw)
    np.testing.assert_allclose(w1, w2, rtol=1e-9, atol=1e-15)


@pytest.mark.parametrize("mode,calib,rnd", [(0, 0, 1), (1, 0, 1), (1, 0, 0), (1, 1, 1), (1, 1, 0), (2, 0, 1)])
def test_all_equal_row_is_uniform(mode, calib, rnd):
    s = np.full((3, 10), -0.75)
    w, _, _, _ = oracle.weight_map(s, np.ones_like(s, bool), mode, K=4, calib=calib,
                                   rounding=rnd)
    p = w / w.sum(1, keepdims=True)
    np.testing.assert_allclose(p, 0.1, rtol=1e-14)


def test_causal_first_row_is_first_value():
    rng = np.random.default_rng(2)
    q, k, v = (rng.normal(size=(1, 1, 8, 4)) for _ in range(3))
    for mode, cal, rnd in [(0, 0, 1), (1, 0, 1), (1, 0, 0), (1, 1, 1), (2, 0, 1)]:
        res = oracle.attn_fwd(q, k, v, True, mode, K=4, calib=cal, rounding=rnd)
        np.testing.assert_allclose(res["O"][0, 0, 0], v[0, 0, 0], rtol=1e-14)


# ------------------------------------------------------------- convergence

def test_interp_minmax_error_bound_and_convergence():
    s, v = _rand_scores(21, R=32, S=200, spread=2.0)
    hi = s.max(1, keepdims=True)
    lo = s.min(1, keepdims=True)
    ex = np.exp(s - hi)
    prev = None
    for K in (4, 16, 64, 256):
        w, _, _, _ = oracle.weight_map(s, v, A.KINTERVAL, K=K, calib=A.MINMAX,
                                       rounding=A.INTERP)
        d = (hi - lo) / K
        bound = d ** 2 / 8 * np.exp(d) * ex
        assert np.all(np.abs(w - ex) <= bound * (1 + 1e-9) + 1e-15)
        err = np.abs(w / w.sum(1, keepdims=True) - ex / ex.sum(1, keepdims=True)).max()
        if prev is not None:
            assert err < prev / 8          # O(1/K^2): 4x more nodes, ~16x smaller
        prev = err
    assert prev < 1e-4


def test_detach_does_not_change_forward():
    # detaching the row extrema is a backward-only switch
    rng = np.random.default_rng(4)
    s = rng.normal(size=(5, 12))
    v = rng.normal(size=(12, 3))
    dO = rng.normal(size=(5, 3))
    valid = np.ones_like(s, bool)
    for cal, rnd in itertools.product((0, 1), (0, 1)):
        _, P1, O1 = A.attn_bwd_rows(s, valid, v, dO, A.KINTERVAL, 4, cal, rnd, A.SURR_PRE, False, 3.0)
        _, P2, O2 = A.attn_bwd_rows(s, valid, v, dO, A.KINTERVAL, 4, cal, rnd, A.SURR_PRE, True, 3.0)
        assert np.array_equal(P1, P2) and np.array_equal(O1, O2)


def test_nonfinite_scores_take_the_maps_limits_or_poison_the_row():
    """A -inf score takes each map's limit at s -> -inf (exact: 0; PoT: the
    floor 2^-N, or 0 when flushed; fixed-window K-interval: the lowest grid
    value g_0, or 0 when flushed); a row whose maximum is NaN or +inf, or
    whose min-max grid would start at -inf, has NaN weights."""
    e = math.exp
    s = np.array([[0.0, -1.0, -np.inf, -2.0],
                  [0.0, np.nan, -1.0, -2.0],
                  [0.0, np.inf, -1.0, -2.0]])
    valid = np.ones_like(s, dtype=bool)
    w, _, _, _ = oracle.weight_map(s, valid, A.EXACT)
    np.testing.assert_allclose(w[0], [1.0, e(-1), 0.0, e(-2)], rtol=1e-15)
    assert np.isnan(w[1]).all() and np.isnan(w[2]).all()
    w, idx, _, _ = oracle.weight_map(s, valid, A.ROWMAX_POT, pot_floor=15)
    assert w[0].tolist() == [1.0, 0.5, 2.0 ** -15, 0.125] and idx[0, 2] == 15
    assert np.isnan(w[1]).all() and np.isnan(w[2]).all()
    w, idx, _, _ = oracle.weight_map(s, valid, A.ROWMAX_POT, pot_floor=15, below_policy=1)
    assert w[0].tolist() == [1.0, 0.5, 0.0, 0.125] and idx[0, 2] == -2
    # fixed window W = 8, K = 4: Delta = 2, g_k = e^{-2(4-k)}; -1 -> u = 3.5 -> 4 (ties to
    # even), -2 -> u = 3, -inf -> clamped to u = 0
    w, idx, _, _ = oracle.weight_map(s, valid, A.KINTERVAL, K=4, calib=A.FIXED_WINDOW,
                                     rounding=A.HARD, window=8.0)
    np.testing.assert_allclose(w[0], [1.0, 1.0, e(-8), e(-2)], rtol=1e-15)
    assert idx[0].tolist() == [4, 4, 0, 3]
    w, idx, _, _ = oracle.weight_map(s, valid, A.KINTERVAL, K=4, calib=A.FIXED_WINDOW,
                                     rounding=A.INTERP, window=8.0, below_policy=1)
    assert w[0, 2] == 0.0 and idx[0, 2] == -2
    w, _, _, _ = oracle.weight_map(s, valid, A.KINTERVAL, K=4, calib=A.MINMAX, rounding=A.HARD)
    assert np.isnan(w).all()
    # the forward: head 0 holds a -inf key (finite output), head 1 a NaN key
    # (every row NaN); D = 1 and q = 1, so the scores are the keys themselves
    q = np.ones((1, 2, 4, 1))
    k = np.array([[0.0, -1.0, -np.inf, -2.0], [0.0, np.nan, -1.0, -2.0]]).reshape(1, 2, 4, 1)
    v = np.arange(8.0).reshape(1, 2, 4, 1)
    res = oracle.attn_fwd(q, k, v, False, A.EXACT, scale=1.0)
    p = np.array([1.0, e(-1), 0.0, e(-2)]) / (1 + e(-1) + e(-2))
    np.testing.assert_allclose(res["O"][0, 0, :, 0], p @ v[0, 0, :, 0], rtol=1e-14)
    assert np.isnan(res["O"][0, 1]).all() and np.isnan(res["LSE"][0, 1]).all()


def test_probe_maps_hand_row_and_limits():
    """Support truncation and uniform weighting ("Approximating Softmax in
    Pretrained LLMs", abstract: positions can be cut, uniform weighting of
    them is damaging), read as: keep the keys within T of the row maximum,
    with their exact weights or with weight 1."""
    e = math.exp
    s = np.array([[0.0, -1.0, -2.5, -4.0]])
    valid = np.ones_like(s, dtype=bool)
    w, idx, _, _ = oracle.weight_map(s, valid, A.TRUNCATED, support=2.6)
    np.testing.assert_allclose(w[0], [1.0, e(-1), e(-2.5), 0.0], rtol=1e-15)
    assert idx[0].tolist() == [0, 0, 0, -2]
    w, idx, _, _ = oracle.weight_map(s, valid, A.UNIFORM, support=2.6)
    assert w[0].tolist() == [1.0, 1.0, 1.0, 0.0]
    # the boundary is inclusive: a key exactly T below the maximum is kept
    w, _, _, _ = oracle.weight_map(s, valid, A.UNIFORM, support=2.5)
    assert w[0].tolist() == [1.0, 1.0, 1.0, 0.0]
    d = inputs.draw(1, 2, 96, 64, seed=21, peaked=True)
    for causal in (False, True):
        ex = oracle.attn_fwd(d["q"], d["k"], d["v"], causal, A.EXACT)
        tr = oracle.attn_fwd(d["q"], d["k"], d["v"], causal, A.TRUNCATED, support=1e9)
        np.testing.assert_allclose(tr["O"], ex["O"], atol=1e-14)
        un = oracle.attn_fwd(d["q"], d["k"], d["v"], causal, A.UNIFORM, support=1e9)
        v = d["v"].double().numpy()
        if causal:
            mean = np.cumsum(v, axis=2) / np.arange(1, 97)[None, None, :, None]
        else:
            mean = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
        np.testing.assert_allclose(un["O"], mean, atol=1e-13)
        # T = 0 keeps the maximum only: O is the value row of the argmax
        t0 = oracle.attn_fwd(d["q"], d["k"], d["v"], causal, A.TRUNCATED, support=0.0)
        am = ex["argmax"]
        np.testing.assert_allclose(t0["O"], np.take_along_axis(v, am[..., None], axis=2),
                                   atol=1e-14)


def test_probe_maps_brute_force_and_monotone_support():
    rng = np.random.default_rng(5)
    for _ in range(30):
        n = int(rng.integers(1, 8))
        s = rng.normal(0, 2.0, (1, n))
        T = float(rng.uniform(0, 4))
        hi = s.max()
        kept = [x >= hi - T for x in s[0]]
        for mode in (A.TRUNCATED, A.UNIFORM):
            w, _, _, _ = oracle.weight_map(s, np.ones_like(s, bool), mode, support=T)
            want = [(math.exp(x - hi) if mode == A.TRUNCATED else 1.0) if k else 0.0
                    for x, k in zip(s[0], kept)]
            np.testing.assert_allclose(w[0], want, rtol=1e-15)
    s = rng.normal(0, 2.0, (16, 40))
    counts = [(oracle.weight_map(s, np.ones_like(s, bool), A.UNIFORM, support=T)[0] > 0).sum()
              for T in (0.0, 0.5, 1.0, 2.0, 4.0, 100.0)]
    assert counts == sorted(counts) and counts[0] == 16 and counts[-1] == s.size
