"""fp64 oracle: weight maps, attention forward, K-interval backward.

TEST INFRASTRUCTURE ONLY (see the package docstring for who may import it).

Everything here is evaluated in float64, one query row at a time (NumPy
vectorises over the rows of a block and over the keys of a row; nothing is
tiled over keys and there is no online rescaling).  Inputs are the values the
GPU reads, decoded exactly to float64 by the caller (bf16 and e4m3 both embed
exactly in float64).

Notation, per (batch b, head h) and query row r:
  valid keys   j in V_r: all j (non-causal) or j <= r (causal, top-left aligned)
  score        s_j = c * (q_r . k_j),   c = scale * q_descale * k_descale
  row extrema  hi = max_j s_j,  lo = min_j s_j  (argmax / argmin: lowest index)

Weight maps (the pages' definitions, with the readings the pages leave open):
  EXACT       w_j = exp(s_j - hi).  "Relative to softmax" is the pages'
              baseline ("Pretraining Transformers with Quantized Softmax in
              Attention", abstract; the wiki flowchart's "old path").
  KINTERVAL   "approximates the exponential using K+1 grid values" with
              "per-row grid calibration" and "interpolation versus hard
              rounding" (same abstract).  Reading used here:
                lo_cal = lo (min-max) or hi - W (fixed-window), a = hi - lo_cal,
                Delta = a / K, nodes t_k = lo_cal + k*Delta,
                grid values g_k = exp(t_k - hi) = exp(-(K-k)*Delta), k = 0..K,
                grid coordinate u_j = clamp((s_j - lo_cal)/Delta, 0, K)
                (u_j = K for every key when a == 0),
                hard rounding  w_j = g_{rint(u_j)}  (round half to even),
                interpolation  k_j = min(floor(u_j), K-1), f_j = u_j - k_j,
                               w_j = (1-f_j) g_{k_j} + f_j g_{k_j+1}.
              Fixed-window keys below the window (s_j < lo_cal) clamp to g_0,
              or are flushed to 0 with below_policy=1.
  ROWMAX_POT  "a coarse logarithmic weight representation anchored at each
              row maximum" / "power-of-two weights" ("Approximating Softmax in
              Pretrained LLMs", abstract; wiki flowchart "Row max -> Power-of-
              two weights").  Reading: x_j = (hi - s_j) * log2(e),
              n_j = min(rint(x_j), N), w_j = 2^-n_j; N (the exponent floor) is a
              parameter, default 15; below_policy=1 flushes rint(x_j) > N to 0.
  Normalisation Z = sum_j w_j, p_j = w_j / Z, O_r = sum_j p_j v_j (* v_descale),
              LSE_r = hi + ln Z.

Backward (K-interval and exact only): the pages name "backward rules,
including calibration derivatives" and "a straight-through surrogate relative
to normalization" (pre / post) without printing them.  The rules coded in
``attn_bwd_rows`` are the exact gradients of these surrogate graphs, with
every integer decision (node index, clamp flag, argmax, argmin) frozen:
  none   w_j = F(s_j; hi, lo_cal)                        (F = the forward map)
  pre    w_j = F(sg(s_j); hi, lo_cal) + e_j - sg(e_j),   e_j = exp(s_j - sg(hi))
  post   p_j = F-normalised(sg(s_j); hi, lo_cal) + p*_j - sg(p*_j),
         p*_j = softmax(s)_j
where sg() stops the gradient, and hi / lo are live (the calibration
derivatives) unless ``detach_extrema``, in which case they are constants.
"""

from __future__ import annotations

import math

import numpy as np

EXACT, KINTERVAL, ROWMAX_POT = 0, 1, 2
TRUNCATED, UNIFORM = 3, 4     # the sensitivity probes of paper B (see _map_rows)
MINMAX, FIXED_WINDOW = 0, 1
INTERP, HARD = 0, 1
SURR_NONE, SURR_PRE, SURR_POST = 0, 1, 2

LOG2E = 1.0 / math.log(2.0)

# index codes returned beside the weights
IDX_MASKED = -1      # key outside V_r
IDX_FLUSHED = -2     # weight forced to 0 by below_policy=1


def row_scores(q_rows: np.ndarray, k: np.ndarray, c: float, row0: int,
               causal: bool):
    """Scores s[r, j] = c * q_r . k_j in fp64 and the validity mask.

    ``q_rows`` holds query rows row0 .. row0+R-1 of one (b, h); ``k`` all keys.
    Causal masking is top-left aligned with equal query and key lengths:
    key j is valid for query row r iff j <= r.
    """
    s = c * (q_rows @ k.T)
    R, S = s.shape
    if causal:
        rows = np.arange(row0, row0 + R)[:, None]
        valid = np.arange(S)[None, :] <= rows
    else:
        valid = np.ones((R, S), dtype=bool)
    return s, valid


def row_stats(s: np.ndarray, valid: np.ndarray):
    """Row max / min over valid keys, with the lowest index among ties."""
    neg = np.where(valid, s, -np.inf)
    pos = np.where(valid, s, np.inf)
    amax = np.argmax(neg, axis=1)          # np.argmax returns the first maximum
    amin = np.argmin(pos, axis=1)
    r = np.arange(s.shape[0])
    return neg[r, amax], pos[r, amin], amax, amin


def kint_grid(K: int, delta: np.ndarray) -> np.ndarray:
    """Grid values g_k = exp(-(K-k) * Delta) for k = 0..K, one row per Delta."""
    kk = np.arange(K + 1, dtype=np.float64)
    return np.exp(-(K - kk)[None, :] * np.asarray(delta, dtype=np.float64)[:, None])


def _map_rows(s, valid, mode, K, calib, rounding, window, pot_floor,
              below_policy, frozen=None, support=4.0):
    """Apply one weight map to a block of rows; returns a dict of per-row and
    per-element quantities (everything the backward needs, decisions frozen).

    ``frozen`` (optional, [R, S] ints): K-interval node decisions to use
    instead of rounding the fp64 coordinate (node for hard rounding, lower
    node for interpolation; entries < 0 are ignored).  The backward rules are
    defined with the forward's decisions held fixed; passing the decisions a
    forward actually took evaluates those rules at that forward.
    """
    hi, lo, amax, amin = row_stats(s, valid)
    R, S = s.shape
    out = dict(hi=hi, lo=lo, argmax=amax, argmin=amin)
    idx = np.full((R, S), IDX_MASKED, dtype=np.int64)
    # Non-finite scores (possible only with non-finite inputs): a row whose
    # maximum is NaN or +inf, or (min-max calibration) whose minimum is -inf,
    # has no defined weights and gets NaN ones; a -inf score in any other row
    # takes the map's limit at s -> -inf (0, the PoT floor, or the clamp to
    # the lowest grid value / the flush).
    bad = ~np.isfinite(hi)
    if mode == KINTERVAL and calib == MINMAX:
        bad = bad | ~np.isfinite(lo)
    badr = bad[:, None] & valid
    if mode == EXACT:
        with np.errstate(invalid="ignore"):
            w = np.where(valid, np.exp(np.where(valid, s, 0.0) - hi[:, None]), 0.0)
        w = np.where(badr, np.nan, w)
        idx[valid] = 0
        out.update(w=w, idx=idx, lo_cal=lo)
        return out
    if mode in (TRUNCATED, UNIFORM):
        # "Approximating Softmax in Pretrained LLMs", abstract: the number of
        # positions can be cut substantially, yet uniform weighting of them
        # is damaging.  Reading: the kept positions are the valid keys within
        # `support` (natural-log units of s) of the row maximum; TRUNCATED
        # keeps their exact weights exp(s - hi), UNIFORM gives each weight 1;
        # every other key gets 0 (decision index -2).
        with np.errstate(invalid="ignore"):
            kept = valid & (s >= hi[:, None] - support)
            e = np.exp(np.where(valid, s, 0.0) - hi[:, None])
        w = np.where(kept, e if mode == TRUNCATED else 1.0, 0.0)
        w = np.where(badr, np.nan, w)
        idx[valid] = IDX_FLUSHED
        idx[kept] = 0
        out.update(w=w, idx=idx, lo_cal=lo, kept=kept)
        return out
    if mode == ROWMAX_POT:
        with np.errstate(invalid="ignore"):
            x = (hi[:, None] - np.where(valid, s, hi[:, None])) * LOG2E
        x = np.where(badr, 0.0, x)
        n = np.rint(x)                               # round half to even
        flushed = valid & (n > pot_floor) if below_policy == 1 else np.zeros_like(valid)
        n = np.minimum(n, pot_floor)
        w = np.where(valid & ~flushed, np.exp2(-n), 0.0)
        w = np.where(badr, np.nan, w)
        idx[valid] = n[valid].astype(np.int64)
        idx[flushed] = IDX_FLUSHED
        out.update(w=w, idx=idx, x=x, lo_cal=lo)
        return out
    if mode != KINTERVAL:
        raise ValueError("unknown mode %r" % (mode,))
    lo_cal = lo if calib == MINMAX else hi - window
    with np.errstate(invalid="ignore"):
        a = hi - lo_cal
    delta = np.where(bad, 1.0, a / K)
    g = kint_grid(K, delta)
    degenerate = ~(a > 0) & ~bad
    with np.errstate(divide="ignore", invalid="ignore"):
        u_raw = (s - lo_cal[:, None]) / delta[:, None]
    u_raw = np.where(degenerate[:, None] | bad[:, None], float(K), u_raw)
    u_raw = np.where(valid, u_raw, float(K))
    below = valid & (u_raw < 0)
    u = np.clip(u_raw, 0.0, float(K))
    rows = np.arange(R)[:, None]
    if rounding == HARD:
        n = np.rint(u).astype(np.int64)
        if frozen is not None:
            n = np.where(valid & (frozen >= 0), frozen, n)
        w = g[rows, n]
        kidx = n
        f = np.zeros_like(u)
    elif rounding == INTERP:
        kidx = np.minimum(np.floor(u), K - 1).astype(np.int64)
        if frozen is not None:
            kidx = np.where(valid & (frozen >= 0), frozen, kidx)
        f = u - kidx
        w = (1.0 - f) * g[rows, kidx] + f * g[rows, kidx + 1]
    else:
        raise ValueError("unknown rounding %r" % (rounding,))
    flushed = below if (below_policy == 1 and calib == FIXED_WINDOW) else np.zeros_like(valid)
    w = np.where(valid & ~flushed, w, 0.0)
    w = np.where(badr, np.nan, w)
    idx[valid] = kidx[valid]
    idx[flushed] = IDX_FLUSHED
    out.update(w=w, idx=idx, u=u, kidx=kidx, f=f, g=g, a=a, delta=delta,
               lo_cal=lo_cal, below=below, flushed=flushed,
               degenerate=degenerate)
    return out


def weight_map(s, valid, mode, K=4, calib=MINMAX, rounding=HARD, window=8.0,
               pot_floor=15, below_policy=0, support=4.0):
    """Weights and decision indices of one map on given scores.

    ``s``: [R, S] scores, ``valid``: [R, S] bool.  Returns (w, idx, hi, lo)
    where idx is the grid node (hard), the lower node (interp), the PoT
    exponent, 0 for exact and for a kept key of the probes, -1 masked, -2
    flushed (or cut, for the probes).
    """
    s = np.asarray(s, dtype=np.float64)
    valid = np.asarray(valid, dtype=bool)
    m = _map_rows(s, valid, mode, K, calib, rounding, window, pot_floor,
                  below_policy, support=support)
    return m["w"], m["idx"], m["hi"], m["lo"]


def _as64(t):
    """Exact float64 copy of a torch tensor or array (bf16/e4m3 embed exactly)."""
    if hasattr(t, "detach"):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def attn_fwd(q, k, v, causal, mode, K=4, calib=MINMAX, rounding=HARD,
             scale=None, q_descale=1.0, k_descale=1.0, v_descale=1.0,
             window=8.0, pot_floor=15, below_policy=0, heads=None,
             rows=None, row_block=512, want_idx=False, support=4.0):
    """Attention forward, [B, H, S, D] inputs.

    Returns a dict with O [B,H,S,D], LSE/hi/lo [B,H,S] float64 and
    argmax/argmin [B,H,S] int64.  ``heads`` (list of (b, h)) and ``rows``
    (array of query rows) restrict the work to a sample; entries outside it
    are NaN / -1.  ``want_idx`` also returns the [B,H,S,S] decision indices
    (small shapes only).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, S, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    c = float(scale) * float(q_descale) * float(k_descale)
    O = np.full((B, H, S, v.shape[-1]), np.nan)
    LSE = np.full((B, H, S), np.nan)
    HI = np.full((B, H, S), np.nan)
    LO = np.full((B, H, S), np.nan)
    AMAX = np.full((B, H, S), -1, dtype=np.int64)
    AMIN = np.full((B, H, S), -1, dtype=np.int64)
    IDX = np.full((B, H, S, S), IDX_MASKED, dtype=np.int8) if want_idx else None
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    row_list = np.arange(S) if rows is None else np.asarray(rows)
    for (b, h) in heads:
        for i0 in range(0, len(row_list), row_block):
            rr = row_list[i0:i0 + row_block]
            if rows is None:
                s, valid = row_scores(q[b, h, rr], k[b, h], c, int(rr[0]), causal)
            else:
                s = c * (q[b, h, rr] @ k[b, h].T)
                valid = (np.arange(S)[None, :] <= rr[:, None]) if causal \
                    else np.ones_like(s, dtype=bool)
            m = _map_rows(s, valid, mode, K, calib, rounding, window,
                          pot_floor, below_policy, support=support)
            Z = m["w"].sum(axis=1)
            p = m["w"] / Z[:, None]
            O[b, h, rr] = (p @ v[b, h]) * float(v_descale)
            LSE[b, h, rr] = m["hi"] + np.log(Z)
            HI[b, h, rr] = m["hi"]
            LO[b, h, rr] = m["lo"]
            AMAX[b, h, rr] = m["argmax"]
            AMIN[b, h, rr] = m["argmin"]
            if want_idx:
                IDX[b, h, rr] = m["idx"].astype(np.int8)
    res = dict(O=O, LSE=LSE, hi=HI, lo=LO, argmax=AMAX, argmin=AMIN)
    if want_idx:
        res["idx"] = IDX
    return res


def attn_bwd_rows(s, valid, v, dO, mode, K=4, calib=MINMAX, rounding=HARD,
                  surrogate=SURR_NONE, detach_extrema=False, window=8.0,
                  below_policy=0, frozen=None, pot_floor=15, O_in=None):
    """Backward of one block of query rows against all keys.

    Returns (dS [R,S], P [R,S], O [R,D]): dS is dL/ds (before the factor c
    that maps it to dQ / dK), P the forward probabilities.  The rules are the
    exact gradients of the surrogate graphs named in the module docstring.
    delta = dO . O is formed from O_in when given (the forward output a
    caller stores and passes back, as the library's backward takes it), else
    from this function's own O = P V.
    Rowmax-PoT (its backward is not derived on the pages; these are the same
    surrogate graphs applied to it): with its exponents frozen a power-of-two
    weight depends neither on its own score nor on the anchor, so only the
    surrogate's direct term remains (none: dS = 0).
    """
    m = _map_rows(s, valid, mode, K, calib, rounding, window, pot_floor,
                  below_policy, frozen)
    w = m["w"]
    Z = w.sum(axis=1)
    P = w / Z[:, None]
    O = P @ v
    dp = dO @ v.T                                   # dp_j = dO_r . v_j
    delta = (dO * (O if O_in is None else O_in)).sum(axis=1)   # dO . O = sum_j p_j dp_j
    gw = np.where(valid, (dp - delta[:, None]) / Z[:, None], 0.0)   # dL/dw_j
    R = s.shape[0]
    rows = np.arange(R)
    if mode == EXACT:
        return np.where(valid, P * (dp - delta[:, None]), 0.0), P, O
    if mode == ROWMAX_POT:
        if surrogate == SURR_NONE:
            ds = np.zeros_like(s)
        elif surrogate == SURR_PRE:
            e = np.where(valid, np.exp(np.where(valid, s, 0.0) - m["hi"][:, None]), 0.0)
            ds = gw * e
        elif surrogate == SURR_POST:
            sm = np.where(valid, s, -np.inf)
            ex = np.where(valid, np.exp(sm - sm.max(axis=1, keepdims=True)), 0.0)
            pstar = ex / ex.sum(axis=1, keepdims=True)
            dstar = (pstar * dp).sum(axis=1)
            ds = np.where(valid, pstar * (dp - dstar[:, None]), 0.0)
        else:
            raise ValueError("unknown surrogate %r" % (surrogate,))
        return ds, P, O
    if mode != KINTERVAL:
        raise ValueError("backward is defined for EXACT, KINTERVAL and ROWMAX_POT")

    g, kidx, f, u = m["g"], m["kidx"], m["f"], m["u"]
    a, delta_grid = m["a"], m["delta"]
    inside = valid & ~m["below"] & ~m["degenerate"][:, None] & ~m["flushed"]
    rr = rows[:, None]
    if rounding == INTERP:
        gk = g[rr, kidx]
        gk1 = g[rr, np.minimum(kidx + 1, K)]
        slope = gk1 - gk                            # dw/du on the interior
        with np.errstate(divide="ignore", invalid="ignore"):
            dF_ds = np.where(inside, slope / delta_grid[:, None], 0.0)
    else:
        gk = g[rr, kidx]
        gk1 = gk
        slope = np.zeros_like(s)
        dF_ds = np.zeros_like(s)

    # direct (own-score) term
    if surrogate == SURR_NONE:
        ds = gw * dF_ds
    elif surrogate == SURR_PRE:
        e = np.where(valid, np.exp(np.where(valid, s, 0.0) - m["hi"][:, None]), 0.0)
        ds = gw * e
    elif surrogate == SURR_POST:
        sm = np.where(valid, s, -np.inf)
        mx = sm.max(axis=1, keepdims=True)
        ex = np.where(valid, np.exp(sm - mx), 0.0)
        pstar = ex / ex.sum(axis=1, keepdims=True)
        dstar = (pstar * dp).sum(axis=1)
        ds = np.where(valid, pstar * (dp - dstar[:, None]), 0.0)
    else:
        raise ValueError("unknown surrogate %r" % (surrogate,))

    if detach_extrema:
        return ds, P, O

    # calibration derivatives: dF_j/dhi and dF_j/dlo with s_j and every
    # integer decision held fixed
    with np.errstate(divide="ignore", invalid="ignore"):
        if calib == MINMAX:
            live = valid & ~m["degenerate"][:, None]
            if rounding == HARD:
                n = kidx
                dF_dhi = np.where(live, -(K - n) / K * gk, 0.0)
                dF_dlo = -dF_dhi
            else:
                mix = ((1.0 - f) * (K - kidx) * gk + f * (K - kidx - 1) * gk1) / K
                dF_dhi = np.where(live, -slope * u / a[:, None] - mix, 0.0)
                dF_dlo = np.where(live, -slope * (K - u) / a[:, None] + mix, 0.0)
            dhi = (gw * dF_dhi).sum(axis=1)
            dlo = (gw * dF_dlo).sum(axis=1)
        else:
            # fixed-window: lo_cal = hi - W, Delta = W/K fixed; the grid values
            # are constants, only u moves with hi (du/dhi = -K/W).
            if rounding == HARD:
                dhi = np.zeros(R)
            else:
                dhi = (gw * np.where(inside, -slope * K / window, 0.0)).sum(axis=1)
            dlo = np.zeros(R)
    ds = ds.copy()
    ds[rows, m["argmax"]] += dhi
    ds[rows, m["argmin"]] += dlo
    return ds, P, O


def attn_bwd(q, k, v, dO, causal, mode, K=4, calib=MINMAX, rounding=HARD,
             surrogate=SURR_NONE, detach_extrema=False, scale=None,
             window=8.0, below_policy=0, heads=None, row_block=512,
             decisions=None, pot_floor=15, O=None):
    """Gradients dQ, dK, dV [B,H,S,D] (float64) of the attention forward.

    ``heads`` restricts the work to a list of (b, h); other heads are NaN.
    ``decisions`` (optional, [B,H,S,S] ints, the forward's per-element node
    decisions) freezes the K-interval decisions at those values.
    ``O`` (optional, [B,H,S,D]) is the stored forward output the backward
    forms delta = dO . O from, as the library's backward does with the O it
    is given; by default the exact output P V.
    """
    q, k, v, dO = _as64(q), _as64(k), _as64(v), _as64(dO)
    O_given = None if O is None else _as64(O)
    B, H, S, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    c = float(scale)
    dQ = np.full((B, H, S, D), np.nan)
    dK = np.full((B, H, S, D), np.nan)
    dV = np.full((B, H, S, D), np.nan)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in heads:
        dK[b, h] = 0.0
        dV[b, h] = 0.0
        for r0 in range(0, S, row_block):
            rr = np.arange(r0, min(S, r0 + row_block))
            s, valid = row_scores(q[b, h, rr], k[b, h], c, r0, causal)
            fz = None if decisions is None else np.asarray(decisions[b, h, rr], dtype=np.int64)
            ds, P, _ = attn_bwd_rows(s, valid, v[b, h], dO[b, h, rr], mode,
                                     K, calib, rounding, surrogate,
                                     detach_extrema, window, below_policy, fz,
                                     pot_floor,
                                     None if O_given is None else O_given[b, h, rr])
            dQ[b, h, rr] = c * (ds @ k[b, h])
            dK[b, h] += c * (ds.T @ q[b, h, rr])
            dV[b, h] += P.T @ dO[b, h, rr]
    return dict(dQ=dQ, dK=dK, dV=dV)


# ---------------------------------------------------------------------------
# Online-anchor maps (one sweep over key tiles)
#
# The pages' kernel is a patch to a one-sweep attention kernel ("Rowmax-H15 in
# FlashAttention-4 on B200", wiki flowchart: QK tile -> row max (anchor) ->
# power-of-two weights -> PV), which only knows the maximum of the keys it has
# visited so far.  The pages do not state how such a kernel anchors its
# weights; the reading coded here (the build's choice) anchors each key tile
# at the running maximum of the row after that tile, in increasing key order,
# and carries the earlier tiles' accumulators over by the factor the anchor's
# move implies:
#
#   tiles t = 0, 1, ... of `tile` consecutive keys; a_t = max(a_{t-1}, max of
#   the row's valid scores in tile t), a_{-1} = -inf (a tile with no valid key
#   of the row changes nothing)
#   Rowmax-PoT   k_t = rne((a_t - a_{t-1}) log2 e) (0 for the row's first
#                tile); n_j = min(rne((a_t - s_j) log2 e), N) (or flushed past
#                N); O <- O 2^-k_t + sum_j 2^-n_j v_j, Z <- Z 2^-k_t + sum 2^-n_j.
#                Every weight stays a power of two.
#   K-interval (fixed window only): the grid of tile t spans [a_t - W, a_t]
#                (step W/K, values g_k = exp(-(K-k) W/K)); w_j read off it by
#                interpolation or hard rounding as in the two-sweep map;
#                O <- O exp(a_{t-1} - a_t) + sum_j w_j v_j, Z likewise.
#   Exact        w_j = exp(s_j - a_t), rescaled by exp(a_{t-1} - a_t): the
#                online softmax recursion, equal to softmax.
#   O_r = O / Z * v_descale, LSE_r = a_last + ln Z.
# Min-max calibration has no online form here: its grid depends on the
# running minimum as well, so the grid would move with nearly every tile.
# ---------------------------------------------------------------------------

def attn_fwd_online(q, k, v, causal, mode, K=4, rounding=HARD, scale=None,
                    q_descale=1.0, k_descale=1.0, v_descale=1.0, window=8.0,
                    pot_floor=15, below_policy=0, tile=128, heads=None,
                    rows=None, row_block=512, want_idx=False):
    """Attention forward with the online-anchor maps (see the block comment
    above); [B, H, S, D] inputs.  K-interval uses fixed-window calibration.
    Returns the dict of attn_fwd (hi = the last anchor = the row maximum; lo =
    hi - W for K-interval, the row minimum otherwise; argmax/argmin -1), with
    ``idx`` the per-element decision against its tile's anchor."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, S, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    c = float(scale) * float(q_descale) * float(k_descale)
    O = np.full((B, H, S, v.shape[-1]), np.nan)
    LSE = np.full((B, H, S), np.nan)
    HI = np.full((B, H, S), np.nan)
    LO = np.full((B, H, S), np.nan)
    IDX = np.full((B, H, S, S), IDX_MASKED, dtype=np.int8) if want_idx else None
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    row_list = np.arange(S) if rows is None else np.asarray(rows)
    delta = window / K
    g = np.exp(-(K - np.arange(K + 1, dtype=np.float64)) * delta)
    for (b, h) in heads:
        for i0 in range(0, len(row_list), row_block):
            rr = row_list[i0:i0 + row_block]
            s = c * (q[b, h, rr] @ k[b, h].T)
            valid = (np.arange(S)[None, :] <= rr[:, None]) if causal \
                else np.ones_like(s, dtype=bool)
            R = len(rr)
            a = np.full(R, -np.inf)
            Z = np.zeros(R)
            acc = np.zeros((R, v.shape[-1]))
            idx = np.full((R, S), IDX_MASKED, dtype=np.int64)
            for t0 in range(0, S, tile):
                cols = slice(t0, min(S, t0 + tile))
                st, vt = s[:, cols], valid[:, cols]
                seen = vt.any(axis=1)
                if not seen.any():
                    continue
                with np.errstate(invalid="ignore"):
                    tmax = np.where(vt, st, -np.inf).max(axis=1, initial=-np.inf)
                    # a NaN score of the tile makes the anchor NaN
                    tmax = np.where(np.isnan(np.where(vt, st, 0.0)).any(axis=1), np.nan, tmax)
                    a_new = np.where(seen, np.maximum(a, tmax), a)
                    first = ~np.isfinite(a) & ~np.isnan(a)      # no key seen yet
                    if mode == ROWMAX_POT:
                        kt = np.where(first, 0.0, np.rint((a_new - a) * LOG2E))
                        fac = np.exp2(-kt)
                    else:
                        fac = np.where(first, 1.0, np.exp(a - a_new))
                fac = np.where(seen, fac, 1.0)
                Z = Z * fac
                acc = acc * fac[:, None]
                with np.errstate(invalid="ignore"):
                    if mode == EXACT:
                        w = np.exp(np.where(vt, st, 0.0) - a_new[:, None])
                        dec = np.zeros_like(st, dtype=np.int64)
                    elif mode == ROWMAX_POT:
                        x = (a_new[:, None] - np.where(vt, st, a_new[:, None])) * LOG2E
                        x = np.where(np.isfinite(a_new)[:, None], x, 0.0)
                        n = np.rint(x)
                        fl = (n > pot_floor) if below_policy == 1 else np.zeros_like(vt)
                        n = np.minimum(n, pot_floor)
                        w = np.where(fl, 0.0, np.exp2(-n))
                        dec = np.where(fl, IDX_FLUSHED, n).astype(np.int64)
                    elif mode == KINTERVAL:
                        lo_t = a_new - window
                        u_raw = (np.where(vt, st, a_new[:, None]) - lo_t[:, None]) / delta
                        u_raw = np.where(np.isfinite(a_new)[:, None], u_raw, float(K))
                        below = u_raw < 0
                        u = np.clip(u_raw, 0.0, float(K))
                        if rounding == HARD:
                            kk = np.rint(u).astype(np.int64)
                            w = g[kk]
                        else:
                            kk = np.minimum(np.floor(u), K - 1).astype(np.int64)
                            f = u - kk
                            w = (1.0 - f) * g[kk] + f * g[kk + 1]
                        fl = below if below_policy == 1 else np.zeros_like(vt)
                        w = np.where(fl, 0.0, w)
                        dec = np.where(fl, IDX_FLUSHED, kk)
                    else:
                        raise ValueError("unknown mode %r" % (mode,))
                w = np.where(vt, w, 0.0)
                Z = Z + w.sum(axis=1)
                acc = acc + w @ v[b, h, cols]
                idx[:, cols] = np.where(vt, dec, IDX_MASKED)
                a = a_new
            bad = ~np.isfinite(a)
            with np.errstate(invalid="ignore", divide="ignore"):
                O[b, h, rr] = np.where(bad[:, None], np.nan, acc / Z[:, None]) * float(v_descale)
                LSE[b, h, rr] = np.where(bad, np.nan, a + np.log(Z))
            HI[b, h, rr] = a
            if mode == KINTERVAL:
                LO[b, h, rr] = a - window
            else:
                LO[b, h, rr] = np.where(valid, s, np.inf).min(axis=1)
            if want_idx:
                IDX[b, h, rr] = idx.astype(np.int8)
    res = dict(O=O, LSE=LSE, hi=HI, lo=LO, argmax=np.full((B, H, S), -1),
               argmin=np.full((B, H, S), -1))
    if want_idx:
        res["idx"] = IDX
    return res
