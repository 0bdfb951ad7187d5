"""w8a8_scaled_mm_noalloc, called through the C ABI, against w8a8_scaled_mm
and the CPU oracle.

Some callers of this library cannot allocate device memory: a plugin whose
host framework owns all of it and passes only inputs and outputs, or a
latency-critical thread on which cudaMalloc would synchronise the device.
w8a8_scaled_mm_noalloc serves them by keeping the split-K partial sums in a
fixed array in the library's own static device memory.  Its results must be
the same as those of the workspace entry point and of the oracle, call after
call, since the array keeps the previous call's contents.

The file name makes pytest collect it last, so a run that stops at its first
failure has already run every other test.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import oracle
import w8a8_int8_quantized_sq_b200 as sq

pytestmark = pytest.mark.gpu


def _vp(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(q_a, s_tok, q_w, s_ch, y) -> int:
    M, K = q_a.shape
    N = q_w.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sq.lib().w8a8_scaled_mm_noalloc(_vp(q_a), _vp(s_tok), _vp(q_w), _vp(s_ch), _vp(y),
                                           M, N, K, stream)


def _inputs(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    q_a = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    q_w = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    s_tok = torch.rand(M, generator=g) * 0.1 + 1e-3
    s_ch = torch.rand(N, generator=g) * 1e-3 + 1e-5
    return q_a, s_tok, q_w, s_ch


# Which path each shape takes on a 148-SM B200 (sq_describe_plan):
@pytest.mark.parametrize("M,N,K", [(8, 5120, 5120),    # decode: K parts meet in clusters
                                   (8, 5120, 17408),   # stream-K ranges: partials in scratch
                                   (16, 144, 384),     # two row tiles, ragged, clusters
                                   (32, 256, 1280),    # 10 parts per tile: partials in scratch
                                   (300, 512, 1024)])  # large M: no scratch needed
def test_noalloc_matches_workspace_entry_and_oracle_twice(M, N, K):
    cpu = _inputs(M, N, K, seed=M + N + K)
    q_a, s_tok, q_w, s_ch = [t.cuda() for t in cpu]
    want = oracle.w8a8_scaled_mm(*cpu).view(torch.int16)
    ref = sq.w8a8_scaled_mm(q_a, s_tok, q_w, s_ch)  # entry point with a workspace
    torch.cuda.synchronize()
    # same bar as every W8A8 output test: bit-identical BF16
    assert torch.equal(ref.cpu().view(torch.int16), want)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(q_a, s_tok, q_w, s_ch, y) == 0
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
        assert torch.equal(y.cpu().view(torch.int16), want)
    sq.check_device_error()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    q_a, s_tok, q_w, s_ch = [t.cuda() for t in _inputs(4, 16, 128, seed=1)]
    y = torch.empty((4, 16), dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # more row tiles than the counter region holds: refused before any launch
    rc = sq.lib().w8a8_scaled_mm_noalloc(_vp(q_a), _vp(s_tok), _vp(q_w), _vp(s_ch), _vp(y),
                                         4, 16384 * 128 + 16, 128, stream)
    assert rc == 2
    assert sq.lib().w8a8_scaled_mm_noalloc(None, _vp(s_tok), _vp(q_w), _vp(s_ch), _vp(y),
                                           4, 16, 128, stream) == 1
