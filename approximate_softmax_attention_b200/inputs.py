"""Seeded synthetic inputs for the attention workloads.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, so both the CUDA path's callers (tests, bench) and the
CPU oracle's callers can take their inputs from it.

Recipe (per workload): ``torch.Generator('cpu').manual_seed(seed)``; fp32
``randn`` draws in the order Q, K, V, then dO (training workload only), then
for "peaked" workloads one unit direction u per (b, h) (a normalised randn(D)
draw) and, per (b, h), round(0.01*S) key indices from ``randperm(S)``; those
keys get K[b, h, j] += 3 * u[b, h].  Then the cast: bf16 (round to nearest),
or e4m3 with a per-tensor descale = amax / 448 of the fp32 draw (the stored
code is round-to-nearest of x / descale).

The shapes follow the pages' sequence lengths (2K, 8K, 16K on one B200,
"Approximating Softmax in Pretrained LLMs", abstract) and the 124M-GPT
training shape of "Pretraining Transformers with Quantized Softmax in
Attention" (12 heads of 64 at sequence 1024).  The pages name no dataset for
this path; these synthetic draws stand in for real activations.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    dtype: str              # "bf16" or "fp8"
    causal: bool
    seed: int
    peaked: bool
    with_dO: bool = False
    modes: tuple = field(default_factory=tuple)

    @property
    def shape(self):
        return (self.B, self.H, self.S, self.D)


# (mode, K, calibration, rounding) tuples use the C enum values:
# mode 0 exact / 1 K-interval / 2 Rowmax-PoT; calibration 0 min-max /
# 1 fixed-window; rounding 0 interpolation / 1 hard.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 128, 64, "bf16", False, 0, False,
                     modes=((0, 4, 0, 1), (1, 4, 0, 1), (2, 4, 0, 1))),
    "s2k_bf16_causal": Workload("s2k_bf16_causal", 4, 16, 2048, 128, "bf16",
                                True, 2, True,
                                modes=((0, 16, 0, 0), (2, 16, 0, 0), (1, 16, 0, 0))),
    "s8k_fp8_causal": Workload("s8k_fp8_causal", 2, 16, 8192, 128, "fp8",
                               True, 3, True,
                               modes=((0, 4, 1, 1), (2, 4, 1, 1), (1, 4, 1, 1))),
    "s8k_fp8": Workload("s8k_fp8", 2, 16, 8192, 128, "fp8", False, 3, True,
                        modes=((0, 4, 1, 1), (2, 4, 1, 1), (1, 4, 1, 1))),
    "s8k_bf16": Workload("s8k_bf16", 2, 16, 8192, 128, "bf16", False, 3, True,
                         modes=((0, 4, 1, 1), (2, 4, 1, 1), (1, 4, 1, 1))),
    "s16k_bf16_causal": Workload("s16k_bf16_causal", 1, 32, 16384, 128, "bf16",
                                 True, 4, True,
                                 modes=tuple([(0, 4, 0, 0), (2, 4, 0, 0)] +
                                             [(1, K, c, r) for K in (4, 16)
                                              for c in (0, 1) for r in (0, 1)])),
    "s16k_fp8_causal": Workload("s16k_fp8_causal", 1, 32, 16384, 128, "fp8",
                                True, 4, True,
                                modes=tuple([(0, 4, 0, 0), (2, 4, 0, 0)] +
                                            [(1, K, c, r) for K in (4, 16)
                                             for c in (0, 1) for r in (0, 1)])),
    "train_s1k": Workload("train_s1k", 8, 12, 1024, 64, "bf16", True, 5, False,
                          with_dO=True,
                          modes=((1, 4, 0, 1), (1, 16, 0, 0), (1, 4, 1, 1),
                                 (1, 16, 1, 0))),
    # the backward at head dimension 128 (the forward workloads' D), bf16 and
    # for an e4m3 forward: the training shape's rows with half the heads
    "train_s1k_d128": Workload("train_s1k_d128", 8, 6, 1024, 128, "bf16", True, 5, False,
                               with_dO=True, modes=((1, 4, 0, 1), (1, 16, 1, 0))),
    "train_s1k_d128_fp8": Workload("train_s1k_d128_fp8", 8, 6, 1024, 128, "fp8", True, 5,
                                   False, with_dO=True, modes=((1, 4, 0, 1), (1, 16, 1, 0))),
}


def _e4m3(x: torch.Tensor):
    descale = float(x.abs().max()) / E4M3_MAX
    if descale == 0.0:
        descale = 1.0
    return (x / descale).to(torch.float8_e4m3fn), descale


def draw(B, H, S, D, seed, peaked=False, dtype="bf16", with_dO=False,
         shift=3.0, frac=0.01):
    """Draw Q, K, V (and dO) on the CPU.

    Returns a dict with ``q``, ``k``, ``v`` (torch bf16 or float8_e4m3fn,
    shape [B, H, S, D], contiguous), ``q_descale``/``k_descale``/``v_descale``
    (1.0 for bf16), and ``dO`` (bf16) when requested.
    """
    g = torch.Generator("cpu").manual_seed(int(seed))
    q = torch.randn(B, H, S, D, generator=g, dtype=torch.float32)
    k = torch.randn(B, H, S, D, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, S, D, generator=g, dtype=torch.float32)
    dO = torch.randn(B, H, S, D, generator=g, dtype=torch.float32) if with_dO else None
    if peaked:
        u = torch.randn(B, H, D, generator=g, dtype=torch.float32)
        u = u / u.norm(dim=-1, keepdim=True)
        n = int(round(frac * S))
        for b in range(B):
            for h in range(H):
                idx = torch.randperm(S, generator=g)[:n]
                k[b, h, idx] += shift * u[b, h]
    out = {}
    if dtype == "bf16":
        out.update(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16),
                   v=v.to(torch.bfloat16), q_descale=1.0, k_descale=1.0,
                   v_descale=1.0)
    elif dtype == "fp8":
        q8, qd = _e4m3(q)
        k8, kd = _e4m3(k)
        v8, vd = _e4m3(v)
        out.update(q=q8, k=k8, v=v8, q_descale=qd, k_descale=kd, v_descale=vd)
    else:
        raise ValueError(dtype)
    if dO is not None:
        out["dO"] = dO.to(torch.bfloat16)
    out["scale"] = 1.0 / math.sqrt(D)
    return out


def draw_workload(w: Workload, **over):
    kw = dict(B=w.B, H=w.H, S=w.S, D=w.D, seed=w.seed, peaked=w.peaked,
              dtype=w.dtype, with_dO=w.with_dO)
    kw.update(over)
    return draw(**kw)


def scores_fp32(rows: int, cols: int, seed: int, spread: float = 3.0):
    """Random fp32 score rows for the standalone weight-map test."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    return (spread * torch.randn(rows, cols, generator=g, dtype=torch.float32))
