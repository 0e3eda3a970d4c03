"""GPU parity of the backward (K-interval, exact and Rowmax-PoT maps, bf16,
D = 64 and 128) against the CPU oracle, through the C ABI.

The rules are the oracle's ("Pretraining Transformers with Quantized Softmax
in Attention", abstract: backward rules including calibration derivatives;
straight-through surrogate before or after normalization), whose own pins
are in test_oracle_bwd.py.  The oracle evaluates them at its own fp64
rounding decisions; nothing from the GPU path enters it.  Tolerance (bf16
gradients): against the oracle rounded to bf16, max abs <= 1e-2 (adjacent
bf16 codes allowed where one bf16 step exceeds 1e-2: the first keys of a
causal row reach |dV| > 4), mean abs <= 1e-3.

The kernel's forward takes its rounding decisions in fp32 and may round an
element within rounding error of a grid node the other way (>= 99.9 %
agreement, every mismatch within 1e-3 of a boundary: checked first).  Where
it does, the two sides follow different frozen decisions: the element's own
slope, and the row's calibration sums dhi / dlo, which land on the whole dQ
row and on the dK rows of the row's argmax and argmin.  Those gradient rows
(and the dK / dV rows of the flipped key) are left out of the comparison and
counted; the oracle itself never sees the kernel's decisions.

Both backwards form delta = dO . O from the stored forward output they are
given, as the library's backward does with the O a caller passes back.  Both
get the same one: the oracle's own forward output rounded to bf16, the
format the forward writes (a kernel O would bring a CUDA value into the
oracle; an fp64 O on one side only would test bf16 storage, not the
backward: on a short causal row it moves delta by several percent).
"""

import numpy as np
import pytest
import torch

import oracle
from approximate_softmax_attention_b200 import inputs, qsm

from _helpers import check_bf16_output, check_decisions, to_bf16

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _stored_o(d, causal, mode, K, calib, rnd, window=8.0, heads=None, below=0):
    """The oracle's forward (with its decision indices), whose O rounded to
    bf16 both backwards take as the stored output."""
    return oracle.attn_fwd(d["q"], d["k"], d["v"], causal, mode, K=K, calib=calib, rounding=rnd,
                           window=window, heads=heads, want_idx=True, below_policy=below)


def _run(d, causal, mode, K, calib, rnd, surr, detach, window=8.0, dump=True, O_store=None,
         below=0):
    q, k, v, dO = (d[n].to(DEV).contiguous() for n in ("q", "k", "v", "dO"))
    B, H, S, D = q.shape
    dbg = torch.full((B, H, S, S), -1, dtype=torch.int8, device=DEV) if dump else None
    O, LSE, st = qsm.attention_forward(q, k, v, causal, mode, K, calib, rnd, window=window,
                                       stats=True, debug_idx=dbg, below_policy=below)
    if O_store is not None:
        # heads the oracle left out (NaN) keep the kernel's own output
        Os = torch.from_numpy(np.asarray(O_store, dtype=np.float32)).to(DEV)
        O = torch.where(torch.isnan(Os), O.float(), Os).to(torch.bfloat16).contiguous()
    dQ, dK, dV = qsm.attention_backward(q, k, v, O, dO, LSE, st, causal, mode, K, calib, rnd,
                                        surr, detach_extrema=detach, window=window,
                                        below_policy=below)
    torch.cuda.synchronize()
    out = [dQ.float().cpu().numpy(), dK.float().cpu().numpy(), dV.float().cpu().numpy()]
    return out, (dbg.cpu().numpy() if dump else None)


def _oracle(d, causal, mode, K, calib, rnd, surr, detach, window=8.0, heads=None, O_store=None,
            below=0):
    """The oracle's backward at its own fp64 decisions, delta from the stored
    (bf16) output."""
    return oracle.attn_bwd(d["q"], d["k"], d["v"], d["dO"], causal, mode, K=K, calib=calib,
                           rounding=rnd, surrogate=surr, detach_extrema=detach, window=window,
                           below_policy=below, heads=heads,
                           O=None if O_store is None else to_bf16(O_store))


def _flip_rows(d, dec, causal, mode, K, calib, rnd, window, heads, ref, below=0):
    """Rows of dQ and of dK / dV touched by the kernel forward's decision
    mismatches with fp64 rounding (after checking every mismatch lies within
    1e-3 of a boundary); returns boolean [B,H,S] masks and the count.  ref:
    the oracle's forward with its decision indices."""
    B, H, S, _ = d["q"].shape
    dq = np.zeros((B, H, S), bool)
    dkv = np.zeros((B, H, S), bool)
    if mode != 1 or dec is None:
        return dq, dkv, 0
    check_decisions(d, dec, causal, mode, K, calib, rnd, window, heads, below_policy=below)
    n = 0
    for (b, h) in heads:
        valid = (np.arange(S)[None, :] <= np.arange(S)[:, None]) if causal \
            else np.ones((S, S), bool)
        mism = (dec[b, h].astype(np.int64) != ref["idx"][b, h].astype(np.int64)) & valid
        rows, keys = np.nonzero(mism)
        n += len(rows)
        dq[b, h, rows] = True
        dkv[b, h, keys] = True
        dkv[b, h, ref["argmax"][b, h, rows]] = True
        dkv[b, h, ref["argmin"][b, h, rows]] = True
    return dq, dkv, n


def _check(got, ref, heads=None, tol_max=1e-2, tol_mean=1e-3, skip=None):
    B, H, S, _ = got[0].shape
    heads = heads or [(b, h) for b in range(B) for h in range(H)]
    skip_q, skip_kv = skip if skip is not None else (np.zeros((B, H, S), bool),) * 2
    for g, name in zip(got, ("dQ", "dK", "dV")):
        r = ref[name]
        keep = ~(skip_q if name == "dQ" else skip_kv)
        # rows kept, laid out [head, row, D] so a failure reports where it is
        gg = np.stack([np.where(keep[b, h][:, None], g[b, h], 0.0) for (b, h) in heads])
        rr = np.stack([np.where(keep[b, h][:, None], r[b, h], 0.0) for (b, h) in heads])
        check_bf16_output(gg, rr, tol_max, tol_mean, what=name)


COMBOS = [(K, c, r, s, det) for K in (4, 16) for c in (0, 1) for r in (0, 1)
          for s in (0, 1, 2) for det in (False, True)]


@pytest.mark.parametrize("K,calib,rnd,surr,detach", COMBOS)
@pytest.mark.parametrize("S,causal", [(256, True), (200, False)])
def test_bwd_kinterval_small(S, causal, K, calib, rnd, surr, detach):
    d = inputs.draw(1, 2, S, 64, seed=50 + S, with_dO=True)
    fwd = _stored_o(d, causal, 1, K, calib, rnd, window=6.0)
    got, dec = _run(d, causal, 1, K, calib, rnd, surr, detach, window=6.0, O_store=fwd["O"])
    ref = _oracle(d, causal, 1, K, calib, rnd, surr, detach, window=6.0, O_store=fwd["O"])
    heads = [(0, 0), (0, 1)]
    fq, fkv, n = _flip_rows(d, dec, causal, 1, K, calib, rnd, 6.0, heads, fwd)
    _check(got, ref, skip=(fq, fkv))
    assert fq.sum() <= 0.02 * fq.size, n


@pytest.mark.parametrize("K", [1, 32])
@pytest.mark.parametrize("calib,rnd", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("surr", [1, 2])
def test_bwd_kinterval_extreme_K(K, calib, rnd, surr):
    """K = 1 (one grid segment) and K = 32 (the largest K the backward
    accepts), pre and post surrogate, calibration derivatives on."""
    d = inputs.draw(1, 2, 256, 64, seed=90 + K, with_dO=True)
    fwd = _stored_o(d, True, 1, K, calib, rnd, window=6.0)
    got, dec = _run(d, True, 1, K, calib, rnd, surr, False, window=6.0, O_store=fwd["O"])
    ref = _oracle(d, True, 1, K, calib, rnd, surr, False, window=6.0, O_store=fwd["O"])
    fq, fkv, n = _flip_rows(d, dec, True, 1, K, calib, rnd, 6.0, [(0, 0), (0, 1)], fwd)
    _check(got, ref, skip=(fq, fkv))
    assert fq.sum() <= 0.02 * fq.size, n


@pytest.mark.parametrize("K", [3, 12])
@pytest.mark.parametrize("calib,rnd", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("surr", [1, 2])
def test_bwd_kinterval_non_pow2_K(K, calib, rnd, surr):
    """K not a power of two: the passes evaluate the clamped coordinate itself
    (the saturating form needs K = 2^m), pre and post surrogate."""
    d = inputs.draw(1, 2, 256, 64, seed=130 + K, with_dO=True)
    fwd = _stored_o(d, True, 1, K, calib, rnd, window=6.0)
    got, dec = _run(d, True, 1, K, calib, rnd, surr, False, window=6.0, O_store=fwd["O"])
    ref = _oracle(d, True, 1, K, calib, rnd, surr, False, window=6.0, O_store=fwd["O"])
    fq, fkv, n = _flip_rows(d, dec, True, 1, K, calib, rnd, 6.0, [(0, 0), (0, 1)], fwd)
    _check(got, ref, skip=(fq, fkv))
    assert fq.sum() <= 0.02 * fq.size, n


@pytest.mark.parametrize("K", [4, 5])
@pytest.mark.parametrize("rnd", [0, 1])
@pytest.mark.parametrize("surr", [0, 1, 2])
def test_bwd_kinterval_below_flush(K, rnd, surr):
    """Fixed window with the below-window flush (below_policy = 1, keys below
    hi - W weigh 0): a window of 2.5 puts a large share of the keys below it.
    The passes take the clamped coordinate here, whose sign marks them."""
    W = 2.5
    d = inputs.draw(1, 2, 256, 64, seed=140 + K, with_dO=True)
    fwd = _stored_o(d, True, 1, K, 1, rnd, window=W, below=1)
    got, dec = _run(d, True, 1, K, 1, rnd, surr, False, window=W, O_store=fwd["O"], below=1)
    ref = _oracle(d, True, 1, K, 1, rnd, surr, False, window=W, O_store=fwd["O"], below=1)
    assert (fwd["idx"] == -2).sum() > 0.05 * (fwd["idx"] != -1).sum()   # flushed share
    fq, fkv, n = _flip_rows(d, dec, True, 1, K, 1, rnd, W, [(0, 0), (0, 1)], fwd, below=1)
    _check(got, ref, skip=(fq, fkv))
    assert fq.sum() <= 0.02 * fq.size, n


@pytest.mark.parametrize("S,causal", [(256, True), (200, False), (77, True), (384, False)])
def test_bwd_exact(S, causal):
    d = inputs.draw(1, 2, S, 64, seed=7 + S, with_dO=True)
    fwd = _stored_o(d, causal, 0, 4, 0, 1)
    got, _ = _run(d, causal, 0, 4, 0, 1, 0, False, dump=False, O_store=fwd["O"])
    ref = _oracle(d, causal, 0, 4, 0, 1, 0, False, O_store=fwd["O"])
    _check(got, ref)


@pytest.mark.parametrize("mode,K,calib,rnd", [(1, 4, 0, 1), (1, 16, 0, 0), (1, 4, 1, 1),
                                             (1, 16, 1, 0)])
@pytest.mark.parametrize("surr,detach", [(0, False), (1, False), (2, False), (1, True),
                                         (2, True)])
def test_bwd_training_shape_sampled(mode, K, calib, rnd, surr, detach):
    """B=8, H=12, S=1024, D=64 bf16 causal (124M-GPT attention shape), the
    launch the bench times; the oracle checks three whole heads."""
    w = inputs.WORKLOADS["train_s1k"]
    d = inputs.draw_workload(w)
    heads = [(0, 0), (3, 7), (7, 11)]
    fwd = _stored_o(d, True, mode, K, calib, rnd, heads=heads)
    got, dec = _run(d, True, mode, K, calib, rnd, surr, detach, O_store=fwd["O"])
    ref = _oracle(d, True, mode, K, calib, rnd, surr, detach, heads=heads, O_store=fwd["O"])
    fq, fkv, n = _flip_rows(d, dec, True, mode, K, calib, rnd, 8.0, heads, fwd)
    _check(got, ref, heads=heads, skip=(fq, fkv))
    # the flips are rare: a few rows of the three heads checked
    assert fq.sum() <= 0.01 * 3 * 1024, n
    for g in got:
        assert np.isfinite(g).all()


@pytest.mark.parametrize("surr", [0, 1, 2])
@pytest.mark.parametrize("S,causal", [(256, True), (200, False)])
def test_bwd_rowmax_pot(S, causal, surr):
    """Rowmax-PoT under the surrogate rules (exponents frozen: none gives dQ =
    dK = 0 and only dV; pre and post the surrogate's direct term)."""
    d = inputs.draw(1, 2, S, 64, seed=70 + S, with_dO=True)
    fwd = _stored_o(d, causal, 2, 4, 0, 1)
    got, _ = _run(d, causal, 2, 4, 0, 1, surr, False, dump=False, O_store=fwd["O"])
    ref = _oracle(d, causal, 2, 4, 0, 1, surr, False, O_store=fwd["O"])
    _check(got, ref)
    if surr == 0:
        assert np.abs(got[0]).max() == 0 and np.abs(got[1]).max() == 0


@pytest.mark.parametrize("surr", [1, 2])
def test_bwd_rowmax_pot_training_shape(surr):
    w = inputs.WORKLOADS["train_s1k"]
    d = inputs.draw_workload(w)
    heads = [(1, 2), (6, 9)]
    fwd = _stored_o(d, True, 2, 4, 0, 1, heads=heads)
    got, _ = _run(d, True, 2, 4, 0, 1, surr, False, dump=False, O_store=fwd["O"])
    ref = _oracle(d, True, 2, 4, 0, 1, surr, False, heads=heads, O_store=fwd["O"])
    _check(got, ref, heads=heads)


# ------------------------------------------------------------------ D = 128
# Head dimension 128: two TMEM pairs and half-tile ring stages in both passes
# (64-row Q / dO stages in the dK / dV pass, 64-key K / V stages in the dQ
# pass), 32-column slices per map group in the read-outs.

D128_COMBOS = [(4, 0, 1, 1, False), (16, 0, 0, 2, False), (4, 1, 1, 0, False),
               (16, 1, 0, 1, False), (16, 0, 0, 0, True), (32, 0, 0, 1, False),
               (4, 0, 0, 2, True)]


@pytest.mark.parametrize("K,calib,rnd,surr,detach", D128_COMBOS)
@pytest.mark.parametrize("S,causal", [(256, True), (200, False), (333, True)])
def test_bwd_kinterval_d128(S, causal, K, calib, rnd, surr, detach):
    d = inputs.draw(1, 2, S, 128, seed=130 + S, with_dO=True)
    fwd = _stored_o(d, causal, 1, K, calib, rnd, window=6.0)
    got, dec = _run(d, causal, 1, K, calib, rnd, surr, detach, window=6.0, O_store=fwd["O"])
    ref = _oracle(d, causal, 1, K, calib, rnd, surr, detach, window=6.0, O_store=fwd["O"])
    heads = [(0, 0), (0, 1)]
    fq, fkv, n = _flip_rows(d, dec, causal, 1, K, calib, rnd, 6.0, heads, fwd)
    _check(got, ref, skip=(fq, fkv))
    assert fq.sum() <= 0.02 * fq.size, n


@pytest.mark.parametrize("S,causal", [(256, True), (200, False)])
def test_bwd_exact_d128(S, causal):
    d = inputs.draw(1, 2, S, 128, seed=170 + S, with_dO=True)
    fwd = _stored_o(d, causal, 0, 4, 0, 1)
    got, _ = _run(d, causal, 0, 4, 0, 1, 0, False, dump=False, O_store=fwd["O"])
    ref = _oracle(d, causal, 0, 4, 0, 1, 0, False, O_store=fwd["O"])
    _check(got, ref)


@pytest.mark.parametrize("surr", [1, 2])
def test_bwd_rowmax_pot_d128(surr):
    d = inputs.draw(1, 2, 256, 128, seed=190 + surr, with_dO=True)
    fwd = _stored_o(d, True, 2, 4, 0, 1)
    got, _ = _run(d, True, 2, 4, 0, 1, surr, False, dump=False, O_store=fwd["O"])
    ref = _oracle(d, True, 2, 4, 0, 1, surr, False, O_store=fwd["O"])
    _check(got, ref)


@pytest.mark.parametrize("mode,K,calib,rnd,surr", [(1, 16, 0, 0, 1), (1, 4, 0, 1, 2),
                                                   (1, 16, 1, 0, 2)])
def test_bwd_d128_many_tiles(mode, K, calib, rnd, surr):
    """More query and key tiles than SMs (B2 H48 S512 causal: 384 tiles), so
    every persistent CTA takes several tiles through the rings; the oracle
    checks three whole heads."""
    d = inputs.draw(2, 48, 512, 128, seed=211 + K, with_dO=True)
    heads = [(0, 0), (1, 17), (1, 47)]
    fwd = _stored_o(d, True, mode, K, calib, rnd, heads=heads)
    got, dec = _run(d, True, mode, K, calib, rnd, surr, False, O_store=fwd["O"])
    ref = _oracle(d, True, mode, K, calib, rnd, surr, False, heads=heads, O_store=fwd["O"])
    fq, fkv, n = _flip_rows(d, dec, True, mode, K, calib, rnd, 8.0, heads, fwd)
    _check(got, ref, heads=heads, skip=(fq, fkv))
    assert fq.sum() <= 0.01 * 3 * 512, n
    for g in got:
        assert np.isfinite(g).all()



# ----------------------------------------------------------------- e4m3
# The backward of an e4m3 forward (D = 128): gradients with respect to
# q_descale Q, k_descale K, v_descale V, which the oracle takes as its inputs
# (exact in float64).

def _run_fp8(d, causal, mode, K, calib, rnd, surr, detach, window=8.0, O_store=None):
    q, k, v = (d[n].to(DEV).contiguous() for n in ("q", "k", "v"))
    dO = d["dO"].to(DEV).contiguous()
    B, H, S, D = q.shape
    desc = dict(q_descale=d["q_descale"], k_descale=d["k_descale"], v_descale=d["v_descale"])
    dbg = torch.full((B, H, S, S), -1, dtype=torch.int8, device=DEV)
    O, LSE, st = qsm.attention_forward(q, k, v, causal, mode, K, calib, rnd, window=window,
                                       stats=True, debug_idx=dbg, **desc)
    if O_store is not None:
        Os = torch.from_numpy(np.asarray(O_store, dtype=np.float32)).to(DEV)
        O = torch.where(torch.isnan(Os), O.float(), Os).to(torch.bfloat16).contiguous()
    dQ, dK, dV = qsm.attention_backward(q, k, v, O, dO, LSE, st, causal, mode, K, calib, rnd,
                                        surr, detach_extrema=detach, window=window, **desc)
    torch.cuda.synchronize()
    return [x.float().cpu().numpy() for x in (dQ, dK, dV)], dbg.cpu().numpy()


def _real(d):
    """The tensors the e4m3 codes stand for, in float64."""
    f = lambda t, s: t.to(torch.float32).double().numpy() * float(s)
    return dict(d, q=f(d["q"], d["q_descale"]), k=f(d["k"], d["k_descale"]),
                v=f(d["v"], d["v_descale"]), q_descale=1.0, k_descale=1.0, v_descale=1.0)


@pytest.mark.parametrize("mode,K,calib,rnd,surr,detach",
                         [(1, 4, 0, 1, 1, False), (1, 16, 0, 0, 2, False),
                          (1, 16, 1, 0, 0, False), (1, 4, 1, 1, 2, True), (0, 4, 0, 1, 0, False),
                          (2, 4, 0, 1, 1, False)])
@pytest.mark.parametrize("S,causal", [(256, True), (200, False)])
def test_bwd_fp8(S, causal, mode, K, calib, rnd, surr, detach):
    d = inputs.draw(1, 2, S, 128, seed=240 + S, dtype="fp8", with_dO=True)
    dr = _real(d)
    fwd = _stored_o(dr, causal, mode, K, calib, rnd, window=6.0)
    got, dec = _run_fp8(d, causal, mode, K, calib, rnd, surr, detach, window=6.0, O_store=fwd["O"])
    ref = _oracle(dr, causal, mode, K, calib, rnd, surr, detach, window=6.0, O_store=fwd["O"])
    # (the decision check decodes the e4m3 codes with their descales itself)
    fq, fkv, n = _flip_rows(d, dec if mode == 1 else None, causal, mode, K, calib, rnd, 6.0,
                            [(0, 0), (0, 1)], fwd)
    _check(got, ref, skip=(fq, fkv))
    assert fq.sum() <= 0.02 * fq.size, n


@pytest.mark.parametrize("surr", [1, 2])
@pytest.mark.parametrize("D", [64, 128])
def test_bwd_back_to_back_shared_workspace(surr, D):
    """Backward calls queued back to back on one stream, sharing one
    workspace, without a synchronisation between them (within a call the
    passes after the first start as programmatic dependents of the kernel
    before them): every call's gradients equal those of the same call run
    alone, bit for bit.  Fixed-window hard rounding has no calibration term,
    so no fp32 reductions and the results are deterministic."""
    K, calib, rnd, W = 4, 1, 1, 6.0
    runs = []
    for seed in (160, 161):
        d = inputs.draw(1, 4, 512, D, seed=seed + D, with_dO=True)
        q, k, v, dO = (d[n].to(DEV).contiguous() for n in ("q", "k", "v", "dO"))
        O, LSE, st = qsm.attention_forward(q, k, v, True, 1, K, calib, rnd, window=W, stats=True)
        runs.append((q, k, v, O, dO, LSE, st))

    def bwd(x, ws=None):
        q, k, v, O, dO, LSE, st = x
        return qsm.attention_backward(q, k, v, O, dO, LSE, st, True, 1, K, calib, rnd, surr,
                                      window=W, workspace=ws)

    alone = []
    for x in runs:
        alone.append(bwd(x))
        torch.cuda.synchronize()
    ws = torch.empty(qsm.qsm_attn_bwd_workspace_size(1, 4, 512, D), dtype=torch.uint8, device=DEV)
    queued = [bwd(runs[i % 2], ws) for i in range(6)]
    torch.cuda.synchronize()
    for i, got in enumerate(queued):
        for g, r, name in zip(got, alone[i % 2], ("dQ", "dK", "dV")):
            assert torch.equal(g, r), (i, name)


def _align256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("D", [64, 128])
def test_bwd_post_row_statistics(D):
    """The post surrogate's row pass against plain fp64 softmax statistics:
    LSE*_r = log sum_j exp(s_rj) and delta*_r = sum_j softmax(s_r)_j dO_r.v_j
    over the valid keys.  White box: the pass writes them to the backward
    workspace at byte offset align256(B H S D 4) (after the fp32 calibration
    part of dK), 8 floats a row, LSE* first, then delta*.  The bound is the
    fp32 sums' (and the exponentials') error, far below what the gradient
    tolerances can see: LSE* within 5e-6, and delta* -- a signed sum, whose
    error scales with sum_j p_j |dp_j| rather than with delta* itself --
    within 5e-6 of that scale (both measure below 1e-6 here)."""
    B, H, S = 1, 4, 512
    d = inputs.draw(B, H, S, D, seed=170 + D, with_dO=True)
    q, k, v, dO = (d[n].to(DEV).contiguous() for n in ("q", "k", "v", "dO"))
    O, LSE, st = qsm.attention_forward(q, k, v, True, 1, 4, 1, 1, window=6.0, stats=True)
    ws = torch.zeros(qsm.qsm_attn_bwd_workspace_size(B, H, S, D), dtype=torch.uint8, device=DEV)
    qsm.attention_backward(q, k, v, O, dO, LSE, st, True, 1, 4, 1, 1, 2, window=6.0, workspace=ws)
    torch.cuda.synchronize()
    off = _align256(B * H * S * D * 4)
    rw = ws[off:off + B * H * S * 8 * 4].view(torch.float32).view(B, H, S, 8).cpu().numpy()
    q64, k64, v64, g64 = (d[n].double().numpy() for n in ("q", "k", "v", "dO"))
    s = np.einsum("bhid,bhjd->bhij", q64, k64) / np.sqrt(D)
    s = np.where(np.tril(np.ones((S, S), bool)), s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    Lsum = e.sum(axis=-1)
    lse = m[..., 0] + np.log(Lsum)
    dp = np.einsum("bhid,bhjd->bhij", g64, v64)
    delta = (e * dp).sum(axis=-1) / Lsum
    scale = (e * np.abs(dp)).sum(axis=-1) / Lsum
    err_l = np.abs(rw[..., 0] - lse).max()
    err_d = (np.abs(rw[..., 1] - delta) / scale).max()
    assert err_l <= 5e-6, err_l
    assert err_d <= 5e-6, err_d
