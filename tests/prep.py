"""Oracle-side preparation of the seeded workloads (test infrastructure).

Every input the CUDA path sees in the parity tests comes from here: raw BF16
X and W from the seeded generator, then the oracle's SmoothQuant factors,
weight quantisation and (for W8A8) the oracle's per-token quantisation of X.
Nothing here is computed by the CUDA path.
"""
from __future__ import annotations

import functools
from typing import Dict, Optional

import torch

import oracle
from w8a8_int8_quantized_sq_b200 import inputs


def bf16_ulp(y: torch.Tensor) -> torch.Tensor:
    """Spacing of BF16 numbers at |y| (fp64); the subnormal spacing at 0."""
    a = y.double().abs().clamp_min(2.0 ** -126)
    return torch.exp2(torch.floor(torch.log2(a)) - 7)


@functools.lru_cache(maxsize=8)
def workload(i: int, M: Optional[int] = None) -> Dict[str, torch.Tensor]:
    wl = inputs.workload(i)
    x = wl.make_x(M)
    w = wl.make_w()
    d: Dict[str, torch.Tensor] = {"x": x, "w": w}
    if wl.smooth:
        s, inv = oracle.smooth_factors(x, w)
        d["s"], d["inv_s"] = s, inv
    else:
        d["s"], d["inv_s"] = None, None
    if wl.variant == "gs128":
        d["q_w"], d["s_blk"] = oracle.quant_weight(w, d["s"], group=128)
    else:
        d["q_w"], d["s_ch"] = oracle.quant_weight(w, d["s"], group=0)
    if wl.variant in ("w8a8", "gs128"):
        d["q_a"], d["s_tok"] = oracle.quant_per_token(x, d["inv_s"])
    return d


def to_cuda(d: Dict[str, Optional[torch.Tensor]]) -> Dict[str, Optional[torch.Tensor]]:
    return {k: (v.cuda() if v is not None else None) for k, v in d.items()}
