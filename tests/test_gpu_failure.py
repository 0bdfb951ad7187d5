"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The self-test kernel waits, with a limit of about a millisecond, on an
mbarrier that nothing arrives on.  Its wait gives up the way every role wait
of the GEMM kernels does (abort flag raised, device error word latched), and
the host sees SQ_ERR_TIMEOUT through sq_check_device_error.  The context must
stay usable: after the error word is cleared, the next calls of the layer
match the oracle.
"""
from __future__ import annotations

import pytest
import torch

import oracle
import w8a8_int8_quantized_sq_b200 as sq
from tests.prep import workload

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_stays_usable():
    sq.check_device_error()  # nothing latched before
    assert sq.selftest_wait_timeout(2_000_000) == 1
    with pytest.raises(sq.SqError) as e:
        sq.check_device_error(reset=True)
    assert e.value.code == 6
    sq.check_device_error()  # the word was cleared
    # the layer still works: decode shape (cluster split-K) and the tiny workload
    for cfg in (1, 0):
        d = workload(cfg)
        ref = oracle.w8a8_scaled_mm(d["q_a"], d["s_tok"], d["q_w"], d["s_ch"])
        y = sq.linear_w8a8(d["x"].cuda(), d["inv_s"].cuda(), d["q_w"].cuda(), d["s_ch"].cuda())
        assert torch.equal(y.cpu().view(torch.int16), ref.view(torch.int16))
    sq.check_device_error()


def test_selftest_rejects_bad_limits():
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    import ctypes
    L = sq.lib()
    assert L.sq_selftest_wait_timeout(0, ctypes.c_void_p(flag.data_ptr()), None) == 2
    assert L.sq_selftest_wait_timeout(5_000_000_000, ctypes.c_void_p(flag.data_ptr()), None) == 2
    assert L.sq_selftest_wait_timeout(1000, None, None) == 1
