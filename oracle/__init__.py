"""CPU oracle for approximate-softmax attention -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct statement of what the CUDA
path computes.  It exists so that the GPU kernels can be checked against
something written independently of them.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import, call, link or execute anything in here.  The
product path (``approximate_softmax_attention_b200``) never imports it, and
this package never imports the product path: the two share no code, headers,
tables or constants.

Contents
--------
``attention``  fp64 NumPy restatement of the forward weight maps, the attention
               forward and the K-interval backward (one row at a time,
               vectorised over rows only; no tiling, no online rescaling),
               and the online-anchor maps (attn_fwd_online: the anchor of
               each key tile is the running maximum after it, tiles in key
               order -- a reading of the one-sweep kernel on the pages).
``fp32_spec``  a separately written C restatement of the fp32 weight-map
               specification (the op sequence the GPU map must reproduce bit
               for bit), loaded through ctypes.

Sources (titles of the pages the method is known from):
  * "Pretraining Transformers with Quantized Softmax in Attention" (arXiv
    2609.33591), abstract: K-interval attention, K+1 grid values, per-row
    grid calibration, interpolation vs hard rounding, straight-through
    surrogate before/after normalization, calibration derivatives.
  * "Approximating Softmax in Pretrained LLMs: Model Sensitivity and Kernel
    Acceleration" (arXiv 2609.33586), abstract and the wiki page's tile-loop
    flowchart: Rowmax-PoT, power-of-two weights anchored at the row maximum.

Parity pins: every function here is pinned by tests in ``tests/test_oracle_*.py``
(hand-derived examples, brute force on tiny rows, closed forms, invariants and
finite differences).  Functions without such a pin would say "parity
unpinned" here; at present there are none.
"""

from .attention import (  # noqa: F401
    EXACT, KINTERVAL, ROWMAX_POT, TRUNCATED, UNIFORM,
    MINMAX, FIXED_WINDOW,
    INTERP, HARD,
    SURR_NONE, SURR_PRE, SURR_POST,
    LOG2E,
    row_scores, row_stats, kint_grid, weight_map, attn_fwd, attn_bwd,
    attn_bwd_rows, attn_fwd_online,
)
