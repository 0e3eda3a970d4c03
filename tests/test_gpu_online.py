"""GPU parity of the one-sweep forward (opts.anchor = 1) against the oracle,
through the C ABI.

The exact map is softmax under either anchor (the online softmax recursion),
so it is checked against the oracle's two-sweep softmax.  Rowmax-PoT and
fixed-window K-interval anchored at the running maximum after each 128-key
tile are checked against the oracle's attn_fwd_online (the reading pinned in
test_oracle_online.py).  Tolerances as for the two-sweep forward: bf16 O max
abs <= 1e-2, mean <= 1e-3; e4m3 max <= 5e-2; decisions >= 99.9 % with every
mismatch within 1e-3 of a rounding boundary.  A PoT row also takes one
rounding decision per anchor move (the carried factor 2^-rne(move)); rows
where a move lies within 1e-4 (log2 units) of a half-integer can round
either way in fp32 and are left out of the max-error check, and counted.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A
from approximate_softmax_attention_b200 import inputs, qsm

from _helpers import check_bf16_output, err_stats

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LOG2E = 1.0 / math.log(2.0)


def _gpu(x):
    return x.to(DEV).contiguous()


def _run(d, causal, mode, K, rnd, window=8.0, below=0, debug=False, stats=False):
    q, k, v = _gpu(d["q"]), _gpu(d["k"]), _gpu(d["v"])
    B, H, S, D = q.shape
    dbg = torch.full((B, H, S, S), -7, dtype=torch.int8, device=DEV) if debug else None
    res = qsm.attention_forward(q, k, v, causal, mode, K, qsm.CALIB_FIXED_WINDOW, rnd,
                                q_descale=d["q_descale"], k_descale=d["k_descale"],
                                v_descale=d["v_descale"], window=window, below_policy=below,
                                stats=stats, debug_idx=dbg, anchor=qsm.ANCHOR_RUNNING)
    torch.cuda.synchronize()
    out = dict(O=res[0].float().cpu().numpy(), LSE=res[1].cpu().numpy())
    if stats:
        out.update(hi=res[2]["hi"].cpu().numpy(), lo=res[2]["lo"].cpu().numpy())
    if debug:
        out["idx"] = dbg.cpu().numpy()
    return out


def _oracle(d, causal, mode, K, rnd, window=8.0, below=0, want_idx=False, heads=None,
            rows=None):
    kw = dict(q_descale=d["q_descale"], k_descale=d["k_descale"], v_descale=d["v_descale"],
              heads=heads, rows=rows)
    if mode == A.EXACT:
        return oracle.attn_fwd(d["q"], d["k"], d["v"], causal, A.EXACT, want_idx=want_idx, **kw)
    return A.attn_fwd_online(d["q"], d["k"], d["v"], causal, mode, K=K, rounding=rnd,
                             window=window, below_policy=below, want_idx=want_idx, **kw)


def _scores(d, b, h, rows=None):
    q = d["q"][b, h].double().numpy() * d["q_descale"]
    k = d["k"][b, h].double().numpy() * d["k_descale"]
    rr = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    return (q[rr] @ k.T) / math.sqrt(q.shape[1]), rr


def _anchors(s, rr, causal, tile=128):
    """fp64 running maximum after each key's tile, per element, and each
    row's smallest distance of an anchor move (log2 units) to a half-integer."""
    R, S = s.shape
    valid = (np.arange(S)[None, :] <= rr[:, None]) if causal else np.ones((R, S), bool)
    sv = np.where(valid, s, -np.inf)
    T = (S + tile - 1) // tile
    tmax = np.stack([sv[:, t * tile:(t + 1) * tile].max(axis=1) for t in range(T)], 1)
    run = np.maximum.accumulate(tmax, axis=1)
    per_key = np.repeat(run, tile, axis=1)[:, :S]
    with np.errstate(invalid="ignore"):
        mv = np.diff(run, axis=1) * LOG2E
    mv = np.where(np.isfinite(mv) & (mv > 0), mv, 0.0)
    margin = np.where(mv > 0, np.abs(mv - np.floor(mv) - 0.5), np.inf).min(axis=1, initial=np.inf)
    return per_key, margin, valid


def _check_online_decisions(d, got_idx, causal, mode, K, rnd, window, heads):
    """Kernel decisions against the fp64 online reading: >= 99.9 % agreement
    and every mismatch within 1e-3 of a boundary of its tile's coordinate."""
    total = bad = 0
    for (b, h) in heads:
        s, rr = _scores(d, b, h)
        anc, _, valid = _anchors(s, rr, causal)
        ref = A.attn_fwd_online(d["q"][b:b + 1, h:h + 1], d["k"][b:b + 1, h:h + 1],
                                d["v"][b:b + 1, h:h + 1], causal, mode, K=K, rounding=rnd,
                                q_descale=d["q_descale"], k_descale=d["k_descale"],
                                window=window, want_idx=True)["idx"][0, 0].astype(np.int64)
        with np.errstate(invalid="ignore"):
            if mode == A.ROWMAX_POT:
                x = (anc - s) * LOG2E
                dist = np.abs(x - np.floor(x) - 0.5)
            else:
                u = np.clip((s - (anc - window)) / (window / K), 0, K)
                fr = u - np.floor(u)
                dist = np.abs(fr - 0.5) if rnd == A.HARD else np.minimum(fr, 1 - fr)
        g = got_idx[b, h].astype(np.int64)
        assert np.all((g[~valid] == -1) | (g[~valid] == -7))
        mism = (g != ref) & valid
        assert np.all(dist[mism] <= 1e-3), (b, h, np.argwhere(mism & (dist > 1e-3))[:5])
        bad += int(mism.sum())
        total += int(valid.sum())
    assert bad <= 1e-3 * total, (bad, total)


def _compare(d, got, ref, causal, mode, tol_max, tol_mean, heads=None, rows=None):
    """O / LSE against the oracle; PoT rows with an anchor move within 1e-4 of
    a half-integer are excluded from the max check (returned count)."""
    B, H = got["O"].shape[:2]
    heads = heads or [(b, h) for b in range(B) for h in range(H)]
    skipped = 0
    for (b, h) in heads:
        rr = np.arange(got["O"].shape[2]) if rows is None else np.asarray(rows)
        keep = np.ones(len(rr), bool)
        if mode == A.ROWMAX_POT:
            s, _ = _scores(d, b, h, rr)
            _, margin, _ = _anchors(s, rr, causal)
            keep = margin > 1e-4
            skipped += int((~keep).sum())
        go, ro = got["O"][b, h, rr][keep], ref["O"][b, h, rr][keep]
        mx, mean = err_stats(go, ro)
        assert mx <= tol_max and mean <= tol_mean, (b, h, mx, mean)
        np.testing.assert_allclose(got["LSE"][b, h, rr][keep], ref["LSE"][b, h, rr][keep],
                                   atol=5e-3, rtol=1e-4)
    return skipped


ONLINE_MAPS = [(A.EXACT, 4, 1), (A.ROWMAX_POT, 4, 1), (A.KINTERVAL, 4, A.HARD),
               (A.KINTERVAL, 16, A.INTERP), (A.KINTERVAL, 4, A.INTERP),
               (A.KINTERVAL, 12, A.INTERP), (A.KINTERVAL, 6, A.HARD)]


@pytest.mark.parametrize("S,D,causal", [(1, 64, False), (77, 64, True), (200, 128, False),
                                        (384, 128, True), (520, 64, True), (700, 128, False)])
@pytest.mark.parametrize("mode,K,rnd", ONLINE_MAPS)
def test_online_bf16_shapes(S, D, causal, mode, K, rnd):
    d = inputs.draw(1, 2, S, D, seed=S + D + 1, peaked=S > 100)
    got = _run(d, causal, mode, K, rnd, window=6.0, debug=S <= 520, stats=True)
    ref = _oracle(d, causal, mode, K, rnd, window=6.0)
    _compare(d, got, ref, causal, mode, 1e-2, 1e-3)
    np.testing.assert_allclose(got["hi"], ref["hi"], atol=1e-4, rtol=1e-5)
    if mode != A.EXACT and S <= 520:
        _check_online_decisions(d, got["idx"], causal, mode, K, rnd, 6.0, [(0, 0), (0, 1)])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mode,K,rnd", ONLINE_MAPS)
def test_online_fp8(causal, mode, K, rnd):
    d = inputs.draw(1, 2, 640, 128, seed=3, peaked=True, dtype="fp8")
    got = _run(d, causal, mode, K, rnd, debug=True)
    ref = _oracle(d, causal, mode, K, rnd)
    _compare(d, got, ref, causal, mode, 5e-2, 5e-3)
    if mode != A.EXACT:
        _check_online_decisions(d, got["idx"], causal, mode, K, rnd, 8.0, [(0, 0), (0, 1)])


@pytest.mark.parametrize("below", [0, 1])
@pytest.mark.parametrize("mode,K,rnd", [(A.ROWMAX_POT, 4, 1), (A.KINTERVAL, 4, A.HARD),
                                        (A.KINTERVAL, 4, A.INTERP)])
def test_online_below_policy_and_floor(mode, K, rnd, below):
    """Wide scores (scale 6/sqrt(D)) push most keys past the PoT floor / below
    the window, clamped or flushed."""
    d = inputs.draw(1, 2, 384, 128, seed=31, peaked=True)
    q, k, v = _gpu(d["q"]), _gpu(d["k"]), _gpu(d["v"])
    scale = 6.0 / math.sqrt(128)
    O, LSE = qsm.attention_forward(q, k, v, True, mode, K, qsm.CALIB_FIXED_WINDOW, rnd,
                                   scale=scale, window=1.5, pot_floor=6, below_policy=below,
                                   anchor=qsm.ANCHOR_RUNNING)
    torch.cuda.synchronize()
    if mode == A.ROWMAX_POT:
        ref = A.attn_fwd_online(d["q"], d["k"], d["v"], True, mode, scale=scale, pot_floor=6,
                                below_policy=below)
    else:
        ref = A.attn_fwd_online(d["q"], d["k"], d["v"], True, mode, K=K, rounding=rnd,
                                scale=scale, window=1.5, below_policy=below)
    check_bf16_output(O.float().cpu().numpy(), ref["O"], 1e-2, 1e-3, what="O")
    np.testing.assert_allclose(LSE.cpu().numpy(), ref["LSE"], atol=5e-3, rtol=1e-4)


def test_online_nonfinite_rows():
    """A NaN key reaches the running anchor of every row that sees it: those
    rows give NaN; earlier rows are untouched."""
    S, D = 256, 64
    d = inputs.draw(1, 1, S, D, seed=12)
    k = d["k"].float()
    k[0, 0, 100, 5] = float("nan")
    d["k"] = k.to(torch.bfloat16)
    for mode, K, rnd in ONLINE_MAPS[:3]:
        got = _run(d, True, mode, K, rnd)
        ref = _oracle(d, True, mode, K, rnd)
        assert np.array_equal(np.isnan(got["O"]), np.isnan(ref["O"]))
        assert np.isnan(got["O"][0, 0, 100:]).all() and np.isfinite(got["O"][0, 0, :100]).all()
        mx, _ = err_stats(got["O"][0, 0, :100], ref["O"][0, 0, :100])
        assert mx <= 1e-2


def _sampled(name, modes, tol_max, tol_mean, nheads=2, nrows=48):
    w = inputs.WORKLOADS[name]
    d = inputs.draw_workload(w)
    rng = np.random.default_rng(1)
    heads = [(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(nheads)]
    rows = np.unique(np.concatenate([[0, 1, 127, 128, w.S - 1],
                                     rng.integers(0, w.S, size=nrows)]))
    skipped = 0
    for (mode, K, rnd) in modes:
        got = _run(d, w.causal, mode, K, rnd)
        ref = _oracle(d, w.causal, mode, K, rnd, heads=heads, rows=rows)
        skipped += _compare(d, got, ref, w.causal, mode, tol_max, tol_mean, heads, rows)
        assert np.isfinite(got["O"]).all()
    assert skipped <= 2, skipped


@pytest.mark.parametrize("name,tol_max,tol_mean", [("s8k_bf16", 1e-2, 1e-3),
                                                   ("s8k_fp8", 5e-2, 5e-3),
                                                   ("s16k_bf16_causal", 1e-2, 1e-3),
                                                   ("s16k_fp8_causal", 5e-2, 5e-3)])
def test_online_full_size_sampled(name, tol_max, tol_mean):
    """The full 8K non-causal and 16K causal shapes, launched as the bench
    launches them, on sampled rows of two heads: exact, PoT, K-interval K=4
    hard and K=16 interpolation (fixed window)."""
    _sampled(name, [(A.EXACT, 4, 1), (A.ROWMAX_POT, 4, 1), (A.KINTERVAL, 4, A.HARD),
                    (A.KINTERVAL, 16, A.INTERP)], tol_max, tol_mean)


def test_online_exact_timeout_path():
    d = inputs.draw(1, 1, 256, 64, seed=1)
    q, k, v = _gpu(d["q"]), _gpu(d["k"]), _gpu(d["v"])
    O = torch.empty(1, 1, 256, 64, dtype=torch.bfloat16, device=DEV)
    LSE = torch.empty(1, 1, 256, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    opts = qsm.make_opts(status_dev=status, debug_flags=1, anchor=1)
    assert qsm.qsm_attn_fwd(q, k, v, O, LSE, False, qsm.MODE_EXACT, 4, 0, 1, 0,
                            opts) == qsm.QSM_OK
    torch.cuda.synchronize()
    assert int(status.item()) == qsm.QSM_ERR_TIMEOUT
    O2, _ = qsm.attention_forward(q, k, v, False, qsm.MODE_EXACT, anchor=qsm.ANCHOR_RUNNING)
    torch.cuda.synchronize()
    ref = oracle.attn_fwd(d["q"], d["k"], d["v"], False, A.EXACT)
    assert err_stats(O2.float().cpu().numpy(), ref["O"])[0] <= 1e-2
