"""The allocation-free backward entry point, qsm_attn_bwd_noalloc.

It serves callers that cannot allocate device memory when they call the
backward (a plugin whose framework owns all device memory through its own
pool, a latency-critical loop that cannot take cudaMalloc's synchronisation):
its scratch is a fixed array inside the library instead of a caller
workspace.  Through the C ABI, two calls in a row must give what
qsm_attn_bwd gives with a workspace, within the backward's tolerance (max
abs 1e-2, adjacent bf16 codes allowed where one step exceeds it; mean abs
1e-3); a shape whose
scratch exceeds the array is refused before any launch.

This file is collected last on purpose, and it is self-contained, so it
passes alone in a fresh process as well as after the other tests.
"""

import numpy as np
import pytest
import torch

from approximate_softmax_attention_b200 import inputs, qsm

from _helpers import check_bf16_output

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _grads(fn, q, k, v, O, dO, LSE, causal, mode, K, calib, rnd, surr, opts):
    dQ, dK, dV = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = fn(q, k, v, O, dO, LSE, dQ, dK, dV, causal, mode, K, calib, rnd, surr, opts)
    assert st == qsm.QSM_OK, qsm.qsm_status_string(st)
    torch.cuda.synchronize()
    return [t.float().cpu().numpy() for t in (dQ, dK, dV)]


@pytest.mark.parametrize("mode,K,calib,rnd,surr,detach", [
    (1, 4, 0, 1, 1, 0),       # K-interval hard, min-max, pre, calibration on
    (1, 16, 1, 0, 2, 0),      # interpolation, fixed-window, post
    (1, 16, 0, 0, 0, 1),      # interpolation, min-max, no surrogate, detached
    (0, 4, 0, 1, 0, 0),       # exact
])
def test_noalloc_matches_workspace_backward_twice(mode, K, calib, rnd, surr, detach):
    B, H, S, D, causal = 2, 4, 512, 64, True
    assert qsm.qsm_attn_bwd_workspace_size(B, H, S, D) <= qsm.NOALLOC_SCRATCH_BYTES
    d = inputs.draw(B, H, S, D, seed=123, with_dO=True)
    q, k, v, dO = (d[n].to(DEV).contiguous() for n in ("q", "k", "v", "dO"))
    O, LSE, st = qsm.attention_forward(q, k, v, causal, mode, K, calib, rnd, stats=True)
    ws = torch.empty(qsm.qsm_attn_bwd_workspace_size(B, H, S, D), dtype=torch.uint8,
                     device=DEV)
    stat_kw = dict(row_hi=st["hi"], row_lo=st["lo"], row_argmax=st["argmax"],
                   row_argmin=st["argmin"], detach_extrema=detach)
    ref = _grads(qsm.qsm_attn_bwd, q, k, v, O, dO, LSE, causal, mode, K, calib, rnd, surr,
                 qsm.make_opts(workspace=ws, workspace_bytes=ws.numel(), **stat_kw))
    noalloc_opts = qsm.make_opts(**stat_kw)
    for _ in range(2):
        got = _grads(qsm.qsm_attn_bwd_noalloc, q, k, v, O, dO, LSE, causal, mode, K, calib,
                     rnd, surr, noalloc_opts)
        for g, r, name in zip(got, ref, ("dQ", "dK", "dV")):
            check_bf16_output(g, r, 1e-2, 1e-3, what=name)


def test_noalloc_refuses_oversize_before_launch():
    B, H, S, D = 8, 12, 1024, 64
    assert qsm.qsm_attn_bwd_workspace_size(B, H, S, D) > qsm.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(B, H, S, D, dtype=torch.bfloat16, device=DEV)
    L = torch.zeros(B, H, S, dtype=torch.float32, device=DEV)
    st = qsm.qsm_attn_bwd_noalloc(x, x, x, x, x, L, x, x, x, True, qsm.MODE_EXACT, 4, 0, 1, 0)
    assert st == qsm.QSM_ERR_INVALID_ARG
