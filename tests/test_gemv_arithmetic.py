"""The one-token W8A16 method, checked on the CPU (no GPU needed).

The matrix-vector kernel does not convert and accumulate in floating point:
it forms v = rint(x * 2^sh) with sh = 157 - (bf16 exponent field of max|x|),
splits v into three unsigned bytes and a signed top byte, takes exact
integer dot products of each byte plane with the int8 weight rows, combines
them in int64 and returns bf16(fp64(sum) * s_ch * 2^-sh).  This file restates
those steps in numpy and checks the claims the kernel rests on: |v| < 2^31,
the planes rebuild v, the sum stays below 2^53 at the largest K the kernel
takes, and the result equals the oracle's (fp64 sum, one rounding) on the
W8A16 workload and on tokens with a wide dynamic range.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from w8a8_int8_quantized_sq_b200 import inputs


def _method(x: torch.Tensor, q: torch.Tensor, s_ch: torch.Tensor) -> torch.Tensor:
    bits = x.view(torch.int16).numpy().astype(np.int64) & 0xFFFF
    e_max = int(((bits & 0x7FFF).max() >> 7) & 0xFF)
    sh = 157 - e_max
    v = np.rint(x.float().double().numpy() * 2.0 ** sh).astype(np.int64)  # half to even
    assert np.abs(v).max() < 2 ** 31
    u = v & 0xFFFFFFFF
    planes = [(u >> (8 * p)) & 0xFF for p in range(4)]
    planes[3] = np.where(planes[3] >= 128, planes[3] - 256, planes[3])  # signed top byte
    assert np.array_equal(planes[0] + (planes[1] << 8) + (planes[2] << 16) + (planes[3] << 24), v)
    qq = q.numpy().astype(np.int64)
    total = sum((qq @ planes[p].T) << (8 * p) for p in range(4))  # exact, int64 [N, 1]
    assert np.abs(total).max() < 2 ** 53
    r = total.astype(np.float64) * s_ch.numpy().astype(np.float64)[:, None] * 2.0 ** -sh
    return torch.from_numpy(np.ascontiguousarray(r.T)).to(torch.bfloat16)


def test_largest_k_keeps_the_sum_exact_in_fp64():
    # 480 compute threads x 64 codes: |sum| <= K * 127 * 2^31 < 2^53
    k_max = 480 * 64
    assert k_max * 127 * 2 ** 31 < 2 ** 53


def test_method_matches_the_oracle_on_the_w8a16_workload():
    N, K = 1024, 17408
    x = inputs.gen_x(1, K, 7)
    g = torch.Generator().manual_seed(5)
    q = torch.randint(-127, 128, (N, K), dtype=torch.int8, generator=g)
    s_ch = torch.rand(N, generator=g) * 1e-3 + 1e-5
    y = _method(x, q, s_ch)
    assert torch.equal(y.view(torch.int16), oracle.w8a16_mm(x, q, s_ch).view(torch.int16))


def test_method_on_a_wide_range_token():
    # values far below the largest are rounded in the image; the result
    # still equals the oracle's here, and extreme codes do not overflow
    N, K = 256, 4096
    g = torch.Generator().manual_seed(11)
    mag = torch.pow(2.0, torch.randint(-40, 20, (1, K), generator=g).float())
    x = (torch.randn(1, K, generator=g) * mag).to(torch.bfloat16)
    x[0, :16] = 0.0
    q = torch.randint(-127, 128, (N, K), dtype=torch.int8, generator=g)
    q[0] = 127
    q[1] = -127
    s_ch = torch.rand(N, generator=g) + 0.5
    y = _method(x, q, s_ch)
    assert torch.equal(y.view(torch.int16), oracle.w8a16_mm(x, q, s_ch).view(torch.int16))
