"""ctypes loader for the C restatement of the fp32 weight-map specification.

TEST INFRASTRUCTURE ONLY.  ``build()`` compiles ``fp32_spec.c`` with gcc
(-O2 -ffp-contract=off, no fast-math) into ``_fp32_spec.so`` beside it.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp32_spec.c")
_LIB = os.path.join(_HERE, "_fp32_spec.so")
_handle = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or \
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def load():
    global _handle
    if _handle is None:
        lib = ctypes.CDLL(build())
        f = lib.spec_map_rows
        f.restype = None
        f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                      ctypes.c_float,
                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                      ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                      ctypes.c_void_p]
        e = lib.spec_exp_vec
        e.restype = None
        e.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        _handle = lib
    return _handle


def spec_exp(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty_like(x)
    load().spec_exp_vec(x.ctypes.data, y.ctypes.data, x.size)
    return y


def spec_map(s, valid_len, mode, K=4, calib=0, rounding=1, window=8.0,
             pot_floor=15, below_policy=0, c=1.0, support=4.0):
    """fp32 map of [rows, cols] raw products ``s`` with score scale ``c``
    (score = c * s); returns (w, idx, hi, lo).  For the exact map ``w`` holds
    the exponent x of the weight 2^x (the GPU evaluates 2^x with its own
    approximate instruction); for the truncated map it holds that exponent
    for a kept key and -inf for a cut one."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    rows, cols = s.shape
    vl = np.ascontiguousarray(valid_len, dtype=np.int32)
    assert vl.shape == (rows,)
    w = np.empty((rows, cols), dtype=np.float32)
    idx = np.empty((rows, cols), dtype=np.int32)
    hi = np.empty(rows, dtype=np.float32)
    lo = np.empty(rows, dtype=np.float32)
    load().spec_map_rows(s.ctypes.data, rows, cols, vl.ctypes.data, float(np.float32(c)),
                         int(mode),
                         int(K), int(calib), int(rounding), float(window),
                         int(pot_floor), int(below_policy), float(support), w.ctypes.data,
                         idx.ctypes.data, hi.ctypes.data, lo.ctypes.data)
    return w, idx, hi, lo
