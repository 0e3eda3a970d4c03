"""Pins for the oracle's backward rules.

Each rule in ``oracle.attn_bwd`` claims to be the exact gradient of a stated
surrogate graph with the forward's integer decisions frozen ("Pretraining
Transformers with Quantized Softmax in Attention", abstract: backward rules
including calibration derivatives; straight-through surrogate before or after
normalization).  The tests below re-state each surrogate graph as a plain
forward function (written here, not taken from the oracle) and compare central
finite differences of it against the oracle's dQ, dK, dV.  Exact mode and the
post-normalization surrogate with detached extrema are also checked against
torch autograd of ordinary softmax attention.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A


def _frozen(s, K, calib, rounding, W):
    """Decisions of the forward map, taken independently of the oracle."""
    R, S = s.shape
    hi = s.max(1)
    lo = s.min(1)
    amax = s.argmax(1)
    amin = s.argmin(1)
    lo_c = lo if calib == A.MINMAX else hi - W
    d = (hi - lo_c) / K
    u = (s - lo_c[:, None]) / d[:, None]
    below = u < 0
    uc = np.clip(u, 0, K)
    if rounding == A.HARD:
        node = np.rint(uc).astype(int)
    else:
        node = np.minimum(np.floor(uc), K - 1).astype(int)
    return dict(amax=amax, amin=amin, below=below, node=node, s0=s.copy(), hi0=hi.copy(),
                lo0=lo_c.copy())


def _F(sv, hi, lo, fr, K, rounding):
    """Forward map with frozen decisions, live in (sv, hi, lo); no clamping."""
    a = hi - lo
    d = a / K
    R, S = sv.shape
    rows = np.arange(R)[:, None]
    kk = np.arange(K + 1)
    g = np.exp(-(K - kk)[None, :] * d[:, None])
    if rounding == A.HARD:
        w = g[rows, fr["node"]]
    else:
        u = (sv - lo[:, None]) / d[:, None]
        k = fr["node"]
        f = u - k
        w = (1 - f) * g[rows, k] + f * g[rows, k + 1]
    return np.where(fr["below"], g[:, :1], w)


def _surrogate_loss(q, k, v, dO, fr, K, calib, rounding, surrogate, detach, W, c):
    s = c * (q @ k.T)
    R = s.shape[0]
    r = np.arange(R)
    if detach:
        hi, lo = fr["hi0"], fr["lo0"]
    else:
        hi = s[r, fr["amax"]]
        lo = s[r, fr["amin"]] if calib == A.MINMAX else hi - W
    if surrogate == A.SURR_NONE:
        w = _F(s, hi, lo, fr, K, rounding)
        p = w / w.sum(1, keepdims=True)
    elif surrogate == A.SURR_PRE:
        w = _F(fr["s0"], hi, lo, fr, K, rounding) + np.exp(s - fr["hi0"][:, None]) \
            - np.exp(fr["s0"] - fr["hi0"][:, None])
        p = w / w.sum(1, keepdims=True)
    else:
        w = _F(fr["s0"], hi, lo, fr, K, rounding)
        sm = np.exp(s - s.max(1, keepdims=True))
        sm /= sm.sum(1, keepdims=True)
        sm0 = np.exp(fr["s0"] - fr["s0"].max(1, keepdims=True))
        sm0 /= sm0.sum(1, keepdims=True)
        p = w / w.sum(1, keepdims=True) + sm - sm0
    return float((dO * (p @ v)).sum())


CASES = [(K, cal, rnd, sur, det) for K in (4, 16) for cal in (0, 1) for rnd in (0, 1)
         for sur in (0, 1, 2) for det in (False, True)]


@pytest.mark.parametrize("K,calib,rounding,surrogate,detach", CASES)
def test_finite_differences_of_surrogate_graph(K, calib, rounding, surrogate, detach):
    rng = np.random.default_rng(100 + K + 7 * calib + 3 * rounding + 11 * surrogate + int(detach))
    S, D = 9, 4
    W = 2.5
    q = rng.normal(size=(S, D))
    k = rng.normal(size=(S, D))
    v = rng.normal(size=(S, D))
    dO = rng.normal(size=(S, D))
    c = 1 / math.sqrt(D)
    res = oracle.attn_bwd(q[None, None], k[None, None], v[None, None], dO[None, None], False,
                          A.KINTERVAL, K=K, calib=calib, rounding=rounding,
                          surrogate=surrogate, detach_extrema=detach, window=W)
    fr = _frozen(c * (q @ k.T), K, calib, rounding, W)
    h = 1e-6
    for name, X, G in (("q", q, res["dQ"]), ("k", k, res["dK"]), ("v", v, res["dV"])):
        for (i, d) in [(0, 0), (3, 1), (5, 2), (8, 3), (int(fr["amax"][2]), 0),
                       (int(fr["amin"][4]), 1)]:
            Xp = X.copy(); Xp[i, d] += h
            Xm = X.copy(); Xm[i, d] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = Xp
            lp = _surrogate_loss(args["q"], args["k"], args["v"], dO, fr, K, calib, rounding,
                                 surrogate, detach, W, c)
            args[name] = Xm
            lm = _surrogate_loss(args["q"], args["k"], args["v"], dO, fr, K, calib, rounding,
                                 surrogate, detach, W, c)
            fd = (lp - lm) / (2 * h)
            an = G[0, 0, i, d]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, i, d, fd, an)


@pytest.mark.parametrize("rounding", [0, 1])
def test_shift_invariance_sum_of_ds_is_zero(rounding):
    rng = np.random.default_rng(8)
    s = rng.normal(size=(6, 20))
    v = rng.normal(size=(20, 5))
    dO = rng.normal(size=(6, 5))
    ds, _, _ = A.attn_bwd_rows(s, np.ones_like(s, bool), v, dO, A.KINTERVAL, 4, A.MINMAX,
                               rounding, A.SURR_NONE, False, 8.0)
    np.testing.assert_allclose(ds.sum(1), 0.0, atol=1e-13)


def _torch_softmax_grads(q, k, v, dO, causal):
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    (o * torch.tensor(dO)).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_exact_backward_is_autograd(causal):
    rng = np.random.default_rng(9)
    B, H, S, D = 1, 2, 17, 8
    q, k, v, dO = (rng.normal(size=(B, H, S, D)) for _ in range(4))
    res = oracle.attn_bwd(q, k, v, dO, causal, A.EXACT)
    gq, gk, gv = _torch_softmax_grads(q, k, v, dO, causal)
    np.testing.assert_allclose(res["dQ"], gq, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["dK"], gk, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["dV"], gv, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_stored_output_enters_only_through_delta(causal):
    """delta = dO . O is formed from the stored output when one is given.
    Given the exact output it changes nothing; given O + E, delta moves by
    dO . E per row, which for the exact map (dS = P (dP - delta)) moves dQ by
    -c (dO . E) (P K) and dK by -c P^T ((dO . E) Q), and leaves dV alone."""
    rng = np.random.default_rng(12)
    B, H, S, D = 1, 1, 13, 8
    q, k, v, dO = (rng.normal(size=(B, H, S, D)) for _ in range(4))
    c = 1.0 / math.sqrt(D)
    base = oracle.attn_bwd(q, k, v, dO, causal, A.EXACT)
    O = oracle.attn_fwd(q, k, v, causal, A.EXACT)["O"]
    same = oracle.attn_bwd(q, k, v, dO, causal, A.EXACT, O=O)
    for n in ("dQ", "dK", "dV"):
        np.testing.assert_allclose(same[n], base[n], rtol=1e-12, atol=1e-13)
    E = 1e-3 * rng.normal(size=O.shape)
    moved = oracle.attn_bwd(q, k, v, dO, causal, A.EXACT, O=O + E)
    shift = (dO * E).sum(axis=-1)[0, 0]                       # [S]
    s = c * (q[0, 0] @ k[0, 0].T)
    if causal:
        s = np.where(np.tril(np.ones((S, S), bool)), s, -np.inf)
    P = np.exp(s - s.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(moved["dQ"][0, 0] - base["dQ"][0, 0],
                               -c * shift[:, None] * (P @ k[0, 0]), rtol=1e-9, atol=1e-13)
    np.testing.assert_allclose(moved["dK"][0, 0] - base["dK"][0, 0],
                               -c * P.T @ (shift[:, None] * q[0, 0]), rtol=1e-9, atol=1e-13)
    np.testing.assert_allclose(moved["dV"], base["dV"], rtol=0, atol=0)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("calib,rounding", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_post_detached_is_softmax_backward_for_q_and_k(causal, calib, rounding):
    rng = np.random.default_rng(10)
    B, H, S, D = 1, 1, 15, 8
    q, k, v, dO = (rng.normal(size=(B, H, S, D)) for _ in range(4))
    res = oracle.attn_bwd(q, k, v, dO, causal, A.KINTERVAL, K=4, calib=calib,
                          rounding=rounding, surrogate=A.SURR_POST, detach_extrema=True,
                          window=3.0)
    gq, gk, _ = _torch_softmax_grads(q, k, v, dO, causal)
    np.testing.assert_allclose(res["dQ"], gq, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["dK"], gk, rtol=1e-10, atol=1e-12)
    # dV uses the forward's approximate probabilities
    P = np.eye(S)[None, None]
    ident = oracle.attn_fwd(q, k, P, causal, A.KINTERVAL, K=4, calib=calib,
                            rounding=rounding, window=3.0)["O"]
    np.testing.assert_allclose(res["dV"], np.swapaxes(ident, -1, -2) @ dO, rtol=1e-10,
                               atol=1e-12)


@pytest.mark.parametrize("K,calib,rounding,surrogate", [(4, 0, 0, 0), (16, 0, 0, 1), (4, 0, 1, 2),
                                                       (16, 1, 0, 0), (4, 1, 1, 1)])
def test_frozen_decisions_input(K, calib, rounding, surrogate):
    """The optional decisions input: its own decisions reproduce the default
    result exactly, and a decision moved to the neighbouring node gives the
    exact gradient of the surrogate graph frozen at the moved decision
    (central finite differences of the graph re-stated above)."""
    rng = np.random.default_rng(77 + K + calib + rounding + surrogate)
    S, D, W = 9, 4, 2.5
    q, k, v, dO = (rng.normal(size=(S, D)) for _ in range(4))
    c = 1 / math.sqrt(D)
    fr = _frozen(c * (q @ k.T), K, calib, rounding, W)
    args = (q[None, None], k[None, None], v[None, None], dO[None, None], False, A.KINTERVAL)
    kw = dict(K=K, calib=calib, rounding=rounding, surrogate=surrogate, window=W)
    base = oracle.attn_bwd(*args, **kw)
    same = oracle.attn_bwd(*args, decisions=fr["node"][None, None], **kw)
    for n in ("dQ", "dK", "dV"):
        assert np.array_equal(base[n], same[n])
    # move one interior decision by one node (as a boundary-near element may)
    node = fr["node"].copy()
    i, j = 3, 5
    if j in (fr["amax"][i], fr["amin"][i]):
        j = 6
    node[i, j] = node[i, j] + 1 if node[i, j] < K - (1 if rounding == 0 else 0) else node[i, j] - 1
    moved = oracle.attn_bwd(*args, decisions=node[None, None], **kw)
    fr2 = dict(fr)
    fr2["node"] = node
    h = 1e-6
    for name, X, G in (("q", q, moved["dQ"]), ("k", k, moved["dK"]), ("v", v, moved["dV"])):
        for (a, d) in [(3, 1), (5, 2), (0, 0)]:
            Xp = X.copy(); Xp[a, d] += h
            Xm = X.copy(); Xm[a, d] -= h
            ar = {"q": q, "k": k, "v": v}
            ar[name] = Xp
            lp = _surrogate_loss(ar["q"], ar["k"], ar["v"], dO, fr2, K, calib, rounding,
                                 surrogate, False, W, c)
            ar[name] = Xm
            lm = _surrogate_loss(ar["q"], ar["k"], ar["v"], dO, fr2, K, calib, rounding,
                                 surrogate, False, W, c)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - G[0, 0, a, d]) <= 1e-6 * max(1.0, abs(fd)), (name, a, d)


def _pot_surrogate_loss(q, k, v, dO, n0, s0, hi0, surrogate, c):
    """The Rowmax-PoT surrogate graphs with the exponents n0 frozen: none, w =
    2^-n0 (constant); pre, w = 2^-n0 + exp(s - hi0) - exp(s0 - hi0); post, p =
    2^-n0 normalised + softmax(s) - softmax(s0)."""
    s = c * (q @ k.T)
    w0 = np.exp2(-n0)
    if surrogate == A.SURR_NONE:
        p = w0 / w0.sum(1, keepdims=True)
    elif surrogate == A.SURR_PRE:
        w = w0 + np.exp(s - hi0[:, None]) - np.exp(s0 - hi0[:, None])
        p = w / w.sum(1, keepdims=True)
    else:
        sm = np.exp(s - s.max(1, keepdims=True))
        sm /= sm.sum(1, keepdims=True)
        sm0 = np.exp(s0 - s0.max(1, keepdims=True))
        sm0 /= sm0.sum(1, keepdims=True)
        p = w0 / w0.sum(1, keepdims=True) + sm - sm0
    return float((dO * (p @ v)).sum())


@pytest.mark.parametrize("surrogate", [A.SURR_NONE, A.SURR_PRE, A.SURR_POST])
def test_pot_backward_finite_differences(surrogate):
    """Rowmax-PoT under the same surrogate rules: central differences of the
    surrogate graph (exponents frozen, floor N = 4 so some weights sit on it)."""
    rng = np.random.default_rng(7 + surrogate)
    S, D = 9, 4
    q, k, v, dO = (rng.normal(size=(S, D)) for _ in range(4))
    c = 1.5 / math.sqrt(D)
    res = oracle.attn_bwd(q[None, None], k[None, None], v[None, None], dO[None, None], False,
                          A.ROWMAX_POT, surrogate=surrogate, scale=c, pot_floor=4)
    s0 = c * (q @ k.T)
    hi0 = s0.max(1)
    n0 = np.minimum(np.rint((hi0[:, None] - s0) / math.log(2.0)), 4)
    h = 1e-6
    for name, X, G in (("q", q, res["dQ"]), ("k", k, res["dK"]), ("v", v, res["dV"])):
        for (i, d) in [(0, 0), (3, 1), (5, 2), (8, 3), (2, 0)]:
            args = {"q": q, "k": k, "v": v}
            Xp = X.copy(); Xp[i, d] += h
            Xm = X.copy(); Xm[i, d] -= h
            args[name] = Xp
            lp = _pot_surrogate_loss(args["q"], args["k"], args["v"], dO, n0, s0, hi0,
                                     surrogate, c)
            args[name] = Xm
            lm = _pot_surrogate_loss(args["q"], args["k"], args["v"], dO, n0, s0, hi0,
                                     surrogate, c)
            np.testing.assert_allclose(G[0, 0, i, d], (lp - lm) / (2 * h), rtol=1e-6,
                                       atol=1e-8)
    if surrogate == A.SURR_NONE:
        assert np.abs(res["dQ"]).max() == 0 and np.abs(res["dK"]).max() == 0
