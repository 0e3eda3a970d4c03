"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/qsm.h declares, and rejects bad arguments before
any launch (so these calls never reach the device)."""

import ctypes
import os
import re

import pytest

from approximate_softmax_attention_b200 import qsm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "qsm.h")) as f:
        txt = f.read()
    return sorted(set(re.findall(r"\b(qsm_[a-z0-9_]+)\s*\(", txt)))


def test_header_and_library_agree():
    L = qsm.lib()
    names = _declared()
    assert set(names) == set(qsm.EXPORTED), names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_defaults():
    for s in range(5):
        assert qsm.qsm_status_string(s).startswith("QSM_")
    assert "unknown" in qsm.qsm_status_string(99)
    o = qsm.qsm_opts_default()
    assert (o.dtype, o.scale, o.window, o.pot_floor, o.below_policy) == (0, 0.0, 8.0, 15, 0)
    assert (o.q_descale, o.k_descale, o.v_descale) == (1.0, 1.0, 1.0)
    assert ctypes.sizeof(qsm.QsmOpts) == 120
    assert qsm.QsmOpts.anchor.offset == 108 and qsm.QsmOpts.support.offset == 112
    assert o.support == 4.0
    assert o.anchor == 0


FAKE = 1 << 20          # aligned, never dereferenced: every call below fails validation


def _fwd(**kw):
    a = dict(Q=FAKE, K=FAKE, V=FAKE, O=FAKE, LSE=FAKE, B=1, H=1, S=128, D=64, causal=0, mode=0,
             Kint=4, calib=0, rnd=1, surr=0, opts=None)
    a.update(kw)
    L = qsm.lib()
    return L.qsm_attn_fwd(a["Q"], a["K"], a["V"], a["O"], a["LSE"], a["B"], a["H"], a["S"],
                          a["D"], a["causal"], a["mode"], a["Kint"], a["calib"], a["rnd"],
                          a["surr"], ctypes.byref(a["opts"]) if a["opts"] else None, None)


@pytest.mark.parametrize("kw,want", [
    (dict(B=0), qsm.QSM_ERR_INVALID_ARG), (dict(S=0), qsm.QSM_ERR_INVALID_ARG),
    (dict(S=70000), qsm.QSM_ERR_INVALID_ARG), (dict(D=96), qsm.QSM_ERR_UNSUPPORTED),
    (dict(mode=5), qsm.QSM_ERR_INVALID_ARG), (dict(mode=1, Kint=0), qsm.QSM_ERR_INVALID_ARG),
    (dict(mode=1, Kint=65), qsm.QSM_ERR_INVALID_ARG), (dict(calib=2), qsm.QSM_ERR_INVALID_ARG),
    (dict(rnd=5), qsm.QSM_ERR_INVALID_ARG), (dict(surr=3), qsm.QSM_ERR_INVALID_ARG),
    (dict(causal=2), qsm.QSM_ERR_INVALID_ARG), (dict(Q=0), qsm.QSM_ERR_INVALID_ARG),
    (dict(O=FAKE + 8), qsm.QSM_ERR_INVALID_ARG), (dict(B=300, H=300), qsm.QSM_ERR_UNSUPPORTED),
])
def test_fwd_rejects_bad_arguments(kw, want):
    assert _fwd(**kw) == want


@pytest.mark.parametrize("field,val,want", [
    ("pot_floor", 127, qsm.QSM_ERR_INVALID_ARG), ("pot_floor", -1, qsm.QSM_ERR_INVALID_ARG),
    ("window", 0.0, qsm.QSM_ERR_INVALID_ARG), ("window", float("nan"), qsm.QSM_ERR_INVALID_ARG),
    ("below_policy", 2, qsm.QSM_ERR_INVALID_ARG), ("scale", -1.0, qsm.QSM_ERR_INVALID_ARG),
    ("q_descale", 0.0, qsm.QSM_ERR_INVALID_ARG), ("dtype", 7, qsm.QSM_ERR_INVALID_ARG),
    ("dtype", 1, qsm.QSM_ERR_UNSUPPORTED),           # e4m3 needs D = 128
    ("anchor", 2, qsm.QSM_ERR_INVALID_ARG),
    ("support", -1.0, qsm.QSM_ERR_INVALID_ARG), ("support", float("inf"), qsm.QSM_ERR_INVALID_ARG),
])
def test_fwd_rejects_bad_options(field, val, want):
    o = qsm.qsm_opts_default()
    setattr(o, field, val)
    assert _fwd(opts=o) == want


def test_bwd_rejects_bad_arguments():
    L = qsm.lib()

    def bwd(mode=1, opts=None, dtype=0):
        o = opts or qsm.qsm_opts_default()
        o.dtype = dtype
        return L.qsm_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128,
                              128, 1, mode, 4, 0, 1, 1, ctypes.byref(o), None)
    assert bwd(mode=2) == qsm.QSM_ERR_INVALID_ARG           # PoT backward needs row_hi
    assert bwd(mode=1, dtype=1) == qsm.QSM_ERR_INVALID_ARG  # e4m3 (D = 128): no statistics
    o64 = qsm.qsm_opts_default()
    o64.dtype = 1
    assert L.qsm_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 1,
                          1, 4, 0, 1, 1, ctypes.byref(o64), None) == qsm.QSM_ERR_UNSUPPORTED
    assert bwd(mode=1) == qsm.QSM_ERR_INVALID_ARG           # no row statistics
    o = qsm.qsm_opts_default()
    o.row_hi = o.row_lo = o.row_argmax = o.row_argmin = FAKE
    assert bwd(mode=1, opts=o) == qsm.QSM_ERR_INVALID_ARG   # no workspace
    o.workspace = FAKE
    o.workspace_bytes = 16
    assert bwd(mode=1, opts=o) == qsm.QSM_ERR_INVALID_ARG   # workspace too small
    assert qsm.qsm_attn_bwd_workspace_size(1, 1, 128, 128) > 0
    assert qsm.qsm_attn_bwd_workspace_size(1, 1, 128, 96) == 0


def test_bwd_refuses_unsupported_shapes_before_launch():
    # complete arguments (statistics and a large enough workspace) for shapes
    # the backward's grid tables do not cover: K > 32, at either D
    L = qsm.lib()
    o = qsm.qsm_opts_default()
    o.row_hi = o.row_lo = o.row_argmax = o.row_argmin = FAKE
    o.workspace = FAKE

    def bwd(D, Kint):
        o.workspace_bytes = qsm.qsm_attn_bwd_workspace_size(1, 1, 128, D)
        return L.qsm_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128,
                              D, 1, 1, Kint, 0, 1, 1, ctypes.byref(o), None)
    assert bwd(128, 33) == qsm.QSM_ERR_UNSUPPORTED
    assert bwd(64, 33) == qsm.QSM_ERR_UNSUPPORTED


def test_weight_map_rejects_bad_arguments():
    L = qsm.lib()
    f = L.qsm_weight_map
    assert f(FAKE, FAKE, 0, 10, 1, 4, 0, 1, None, FAKE, None, None, None, None) == \
        qsm.QSM_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 10, 10, 1, 99, 0, 1, None, FAKE, None, None, None, None) == \
        qsm.QSM_ERR_INVALID_ARG
    assert f(0, FAKE, 10, 10, 1, 4, 0, 1, None, FAKE, None, None, None, None) == \
        qsm.QSM_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        qsm._ptr(torch.zeros(4))


def test_noalloc_status_matches_the_workspace_backward():
    """qsm_attn_bwd_noalloc returns the status qsm_attn_bwd returns for the same
    shape errors, before touching any device."""
    L = qsm.lib()
    o = qsm.qsm_opts_default()

    def both(B, S, D):
        a = L.qsm_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, 1, S, D, 1,
                           1, 4, 0, 1, 1, ctypes.byref(o), None)
        b = L.qsm_attn_bwd_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, 1, S,
                                   D, 1, 1, 4, 0, 1, 1, ctypes.byref(o), None)
        return a, b
    assert both(1, 128, 96) == (qsm.QSM_ERR_UNSUPPORTED, qsm.QSM_ERR_UNSUPPORTED)
    assert both(0, 128, 64) == (qsm.QSM_ERR_INVALID_ARG, qsm.QSM_ERR_INVALID_ARG)
    assert both(1, 0, 64) == (qsm.QSM_ERR_INVALID_ARG, qsm.QSM_ERR_INVALID_ARG)


def test_running_anchor_refusals_before_launch():
    """anchor = 1 (the one-sweep maps): no min-max K-interval form, no argument
    statistics, and no backward except for the exact map."""
    o = qsm.qsm_opts_default()
    o.anchor = 1
    assert _fwd(mode=1, calib=0, opts=o) == qsm.QSM_ERR_UNSUPPORTED
    o.row_argmax = FAKE
    assert _fwd(mode=2, opts=o) == qsm.QSM_ERR_UNSUPPORTED
    L = qsm.lib()
    o = qsm.qsm_opts_default()
    o.anchor = 1
    o.row_hi = o.row_lo = o.row_argmax = o.row_argmin = FAKE
    o.workspace = FAKE
    o.workspace_bytes = qsm.qsm_attn_bwd_workspace_size(1, 1, 128, 64)
    assert L.qsm_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64,
                          1, 1, 4, 1, 1, 1, ctypes.byref(o), None) == qsm.QSM_ERR_UNSUPPORTED


def test_probe_refusals_before_launch():
    """The probes are forward-only and anchored at the final row maximum."""
    o = qsm.qsm_opts_default()
    o.anchor = 1
    assert _fwd(mode=3, opts=o) == qsm.QSM_ERR_UNSUPPORTED
    L = qsm.lib()
    o = qsm.qsm_opts_default()
    o.row_hi = o.row_lo = o.row_argmax = o.row_argmin = FAKE
    o.workspace = FAKE
    o.workspace_bytes = qsm.qsm_attn_bwd_workspace_size(1, 1, 128, 64)
    for mode in (3, 4):
        assert L.qsm_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64,
                              1, mode, 4, 0, 1, 1, ctypes.byref(o), None) == qsm.QSM_ERR_UNSUPPORTED
