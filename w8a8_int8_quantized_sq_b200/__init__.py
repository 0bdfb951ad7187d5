"""Python binding of libsqint8.so (the B200 SmoothQuant W8A8 INT8 linear layer).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI of include/sqint8.h.  PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if the library
cannot be loaded, every call raises.

Functions (CUDA tensors in, CUDA tensors out, on the current stream):
  quant_per_token(x, inv_s)            -> (q_a int8 [M,K], s_tok f32 [M])
  w8a8_scaled_mm(q_a, s_tok, q_w, s_ch) -> y bf16 [M,N]
  w8a8_gs128_mm(q_a, s_tok, q_w, s_blk) -> y bf16 [M,N]
  w8a16_mm(x, q_w, s_ch)               -> y bf16 [M,N]
  w8a8_mm_i32(q_a, q_w)                -> acc int32 [M,N]
  linear_w8a8(x, inv_s, q_w, s_ch)     -> y bf16 [M,N] (quant + GEMM)
  smooth_factors(x, w, cap, floor)     -> (s f32 [K], inv_s f32 [K])
  quant_weight(w, smooth, group)       -> (q_w int8 [N,K], scales)
  fold_norm_weight(w_norm, inv_s)      -> gamma f32 [K]
  rmsnorm_quant(h, gamma, eps, group)  -> (q int8 [M,K], scales, inv_rms f32 [M])
  quant_per_group(x, inv_s)            -> (q_a int8 [M,K], s_a f32 [M,K/128])
  w8a8_pg128_mm(q_a, s_a, q_w, s_blk)  -> y bf16 [M,N]
  w8a16_group_mm(x, q_w, s_grp)        -> y bf16 [M,N]
  quant_fp8_per_group(x, inv_s)        -> (q e4m3 uint8 [M,K], s_a f32 [M,K/128])
  quant_fp8_block(w, smooth)           -> (q e4m3 uint8 [N,K], s_w f32 [N/128,K/128])
  fp8_block_mm(q_a, s_a, q_w, s_w)     -> y bf16 [M,N]
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsqint8.so")

OP_W8A8, OP_GS128, OP_W8A16, OP_W8A8_I32 = 0, 1, 2, 3
OP_PG128, OP_FP8BLK, OP_W8A16_GROUP = 4, 5, 6
_STATUS = {0: "ok", 1: "null pointer", 2: "unsupported shape", 3: "pointer not 16-byte aligned",
           4: "workspace missing or too small", 5: "CUDA error", 6: "kernel wait timed out"}


class SqError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {_STATUS.get(code, 'unknown status')} (sq_status {code})")
        self.code = code


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load libsqint8.so (built by build.py); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m w8a8_int8_quantized_sq_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i64, sz, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_double
            sig = {
                "sq_quant_per_token": [vp, vp, vp, vp, i64, i64, vp],
                "w8a8_scaled_mm": [vp, vp, vp, vp, vp, i64, i64, i64, vp, sz, vp],
                "w8a8_gs128_mm": [vp, vp, vp, vp, vp, i64, i64, i64, vp, sz, vp],
                "w8a16_mm": [vp, vp, vp, vp, i64, i64, i64, vp, sz, vp],
                "w8a8_mm_i32": [vp, vp, vp, i64, i64, i64, vp, sz, vp],
                "w8a8_scaled_mm_noalloc": [vp, vp, vp, vp, vp, i64, i64, i64, vp],
                "sq_w8a8_linear": [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, sz, vp],
                "sq_smooth_factors": [vp, i64, vp, i64, i64, dbl, dbl, vp, vp, vp],
                "sq_quant_weight": [vp, vp, vp, vp, i64, i64, i64, vp],
                "sq_check_device_error": [ctypes.c_int],
                "sq_set_overlap": [ctypes.c_int],
                "sq_describe_plan": [ctypes.c_int, i64, i64, i64, ctypes.c_int, vp],
                "sq_fold_norm_weight": [vp, ctypes.c_int, vp, vp, i64, vp],
                "sq_rmsnorm_quant": [vp, vp, ctypes.c_float, i64, vp, vp, vp, i64, i64, vp],
                "sq_quant_per_group": [vp, vp, vp, vp, i64, i64, vp],
                "w8a8_pg128_mm": [vp, vp, vp, vp, vp, i64, i64, i64, vp, sz, vp],
                "w8a16_group_mm": [vp, vp, vp, vp, i64, i64, i64, vp, sz, vp],
                "sq_quant_fp8_per_group": [vp, vp, vp, vp, i64, i64, vp],
                "sq_quant_fp8_block": [vp, vp, vp, vp, i64, i64, vp],
                "fp8_block_mm": [vp, vp, vp, vp, vp, i64, i64, i64, vp, sz, vp],
                "sq_mma_peak": [ctypes.c_int, ctypes.c_int, vp, vp],
                "sq_selftest_wait_timeout": [i64, vp, vp],
            }
            for name, args in sig.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = ctypes.c_int
            L.sq_workspace_bytes.argtypes = [ctypes.c_int, i64, i64, i64]
            L.sq_workspace_bytes.restype = ctypes.c_size_t
            L.sq_status_string.argtypes = [ctypes.c_int]
            L.sq_status_string.restype = ctypes.c_char_p
            _lib = L
    return _lib


EXPORTS = ("sq_quant_per_token", "w8a8_scaled_mm", "w8a8_gs128_mm", "w8a16_mm",
           "sq_workspace_bytes", "w8a8_mm_i32", "sq_smooth_factors", "sq_quant_weight",
           "sq_check_device_error", "sq_status_string", "w8a8_scaled_mm_noalloc",
           "sq_w8a8_linear", "sq_set_overlap", "sq_describe_plan", "sq_fold_norm_weight",
           "sq_rmsnorm_quant", "sq_quant_per_group", "w8a8_pg128_mm", "w8a16_group_mm",
           "sq_quant_fp8_per_group", "sq_quant_fp8_block", "fp8_block_mm", "sq_mma_peak",
           "sq_selftest_wait_timeout")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise SqError(fn, rc)


# One zero-initialised workspace per (device, stream).  The kernels leave
# their counters at zero, so it is reused without clearing; calls sharing a
# stream are ordered, calls on different streams get different workspaces.
_ws = {}


def workspace(op: int, M: int, N: int, K: int, device) -> Tuple[Optional[torch.Tensor], int]:
    need = lib().sq_workspace_bytes(op, M, N, K)
    if need == 0:
        return None, 0
    dev = torch.device(device)
    key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
    buf = _ws.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.zeros(max(need, 1 << 20), dtype=torch.uint8, device=dev)
        _ws[key] = buf
    return buf, buf.numel()


def reset_workspaces() -> None:
    """Drop cached workspaces (e.g. after a kernel reported a timeout)."""
    _ws.clear()


def quant_per_token(x: torch.Tensor, inv_s: Optional[torch.Tensor] = None):
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check("sq_quant_per_token", lib().sq_quant_per_token(
        _ptr(x), _ptr(inv_s), _ptr(q), _ptr(s), M, K, _stream(x.device)))
    return q, s


def w8a8_scaled_mm(q_a, s_tok, q_w, s_ch, out: Optional[torch.Tensor] = None):
    M, K = q_a.shape
    N = q_w.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    ws, wsb = workspace(OP_W8A8, M, N, K, q_a.device)
    _check("w8a8_scaled_mm", lib().w8a8_scaled_mm(
        _ptr(q_a), _ptr(s_tok), _ptr(q_w), _ptr(s_ch), _ptr(y), M, N, K, _ptr(ws), wsb,
        _stream(q_a.device)))
    return y


def w8a8_scaled_mm_noalloc(q_a, s_tok, q_w, s_ch, out: Optional[torch.Tensor] = None):
    """w8a8_scaled_mm without a workspace, for callers that cannot allocate
    device memory (the library's static scratch holds the split-K partials).
    Calls must not overlap on the GPU."""
    M, K = q_a.shape
    N = q_w.shape[0]
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    _check("w8a8_scaled_mm_noalloc", lib().w8a8_scaled_mm_noalloc(
        _ptr(q_a), _ptr(s_tok), _ptr(q_w), _ptr(s_ch), _ptr(y), M, N, K, _stream(q_a.device)))
    return y


def w8a8_mm_i32(q_a, q_w):
    M, K = q_a.shape
    N = q_w.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device=q_a.device)
    ws, wsb = workspace(OP_W8A8_I32, M, N, K, q_a.device)
    _check("w8a8_mm_i32", lib().w8a8_mm_i32(
        _ptr(q_a), _ptr(q_w), _ptr(acc), M, N, K, _ptr(ws), wsb, _stream(q_a.device)))
    return acc


def w8a8_gs128_mm(q_a, s_tok, q_w, s_blk):
    M, K = q_a.shape
    N = q_w.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    ws, wsb = workspace(OP_GS128, M, N, K, q_a.device)
    _check("w8a8_gs128_mm", lib().w8a8_gs128_mm(
        _ptr(q_a), _ptr(s_tok), _ptr(q_w), _ptr(s_blk), _ptr(y), M, N, K, _ptr(ws), wsb,
        _stream(q_a.device)))
    return y


def w8a16_mm(x, q_w, s_ch):
    M, K = x.shape
    N = q_w.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws, wsb = workspace(OP_W8A16, M, N, K, x.device)
    _check("w8a16_mm", lib().w8a16_mm(
        _ptr(x), _ptr(q_w), _ptr(s_ch), _ptr(y), M, N, K, _ptr(ws), wsb, _stream(x.device)))
    return y


def linear_w8a8(x, inv_s, q_w, s_ch, out: Optional[torch.Tensor] = None):
    """y = W8A8 linear layer in one call (sq_w8a8_linear): per-token quant with
    the 1/s fold, then the GEMM launched as a programmatic dependent."""
    M, K = x.shape
    N = q_w.shape[0]
    q_a = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_tok = torch.empty((M,), dtype=torch.float32, device=x.device)
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws, wsb = workspace(OP_W8A8, M, N, K, x.device)
    _check("sq_w8a8_linear", lib().sq_w8a8_linear(
        _ptr(x), _ptr(inv_s), _ptr(q_w), _ptr(s_ch), _ptr(y), _ptr(q_a), _ptr(s_tok), M, N, K,
        _ptr(ws), wsb, _stream(x.device)))
    return y


def smooth_factors(x, w, cap: float = 16.0, floor: float = 1e-5):
    M, K = x.shape
    N = w.shape[0]
    s = torch.empty((K,), dtype=torch.float32, device=x.device)
    inv = torch.empty((K,), dtype=torch.float32, device=x.device)
    _check("sq_smooth_factors", lib().sq_smooth_factors(
        _ptr(x), M, _ptr(w), N, K, cap, floor, _ptr(s), _ptr(inv), _stream(x.device)))
    return s, inv


def quant_weight(w, smooth: Optional[torch.Tensor] = None, group: int = 0):
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.int8, device=w.device)
    sc = torch.empty((N, K // group) if group else (N,), dtype=torch.float32, device=w.device)
    _check("sq_quant_weight", lib().sq_quant_weight(
        _ptr(w), _ptr(smooth), _ptr(q), _ptr(sc), N, K, group, _stream(w.device)))
    return q, sc


def fold_norm_weight(w_norm, inv_s: Optional[torch.Tensor] = None, zero_centered: bool = True):
    """gamma f32 [K]: the (zero-centred) norm weight with 1/s folded in."""
    K = w_norm.numel()
    g = torch.empty((K,), dtype=torch.float32, device=w_norm.device)
    _check("sq_fold_norm_weight", lib().sq_fold_norm_weight(
        _ptr(w_norm), 1 if zero_centered else 0, _ptr(inv_s), _ptr(g), K, _stream(w_norm.device)))
    return g


def rmsnorm_quant(h, gamma, eps: float, group: int = 0, out=None):
    """Fused RMSNorm + fold + INT8 quantisation: (q, scales, inv_rms); group 0 =
    one scale per token, 128 = one per 128 columns."""
    M, K = h.shape
    if out is None:
        q = torch.empty((M, K), dtype=torch.int8, device=h.device)
        sc = torch.empty((M,) if group in (0, K) else (M, K // group), dtype=torch.float32,
                         device=h.device)
        r = torch.empty((M,), dtype=torch.float32, device=h.device)
    else:
        q, sc, r = out
    _check("sq_rmsnorm_quant", lib().sq_rmsnorm_quant(
        _ptr(h), _ptr(gamma), eps, group, _ptr(q), _ptr(sc), _ptr(r), M, K, _stream(h.device)))
    return q, sc, r


def quant_per_group(x, inv_s: Optional[torch.Tensor] = None):
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _check("sq_quant_per_group", lib().sq_quant_per_group(
        _ptr(x), _ptr(inv_s), _ptr(q), _ptr(s), M, K, _stream(x.device)))
    return q, s


def w8a8_pg128_mm(q_a, s_a, q_w, s_blk):
    M, K = q_a.shape
    N = q_w.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    ws, wsb = workspace(OP_PG128, M, N, K, q_a.device)
    _check("w8a8_pg128_mm", lib().w8a8_pg128_mm(
        _ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_blk), _ptr(y), M, N, K, _ptr(ws), wsb,
        _stream(q_a.device)))
    return y


def w8a16_group_mm(x, q_w, s_grp):
    M, K = x.shape
    N = q_w.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws, wsb = workspace(OP_W8A16_GROUP, M, N, K, x.device)
    _check("w8a16_group_mm", lib().w8a16_group_mm(
        _ptr(x), _ptr(q_w), _ptr(s_grp), _ptr(y), M, N, K, _ptr(ws), wsb, _stream(x.device)))
    return y


def quant_fp8_per_group(x, inv_s: Optional[torch.Tensor] = None):
    """(q E4M3 bit patterns uint8 [M,K], s_a f32 [M, K/128])."""
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _check("sq_quant_fp8_per_group", lib().sq_quant_fp8_per_group(
        _ptr(x), _ptr(inv_s), _ptr(q), _ptr(s), M, K, _stream(x.device)))
    return q, s


def quant_fp8_block(w, smooth: Optional[torch.Tensor] = None):
    """(q E4M3 bit patterns uint8 [N,K], s_w f32 [N/128, K/128])."""
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    s = torch.empty((N // 128, K // 128), dtype=torch.float32, device=w.device)
    _check("sq_quant_fp8_block", lib().sq_quant_fp8_block(
        _ptr(w), _ptr(smooth), _ptr(q), _ptr(s), N, K, _stream(w.device)))
    return q, s


def fp8_block_mm(q_a, s_a, q_w, s_w):
    M, K = q_a.shape
    N = q_w.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    ws, wsb = workspace(OP_FP8BLK, M, N, K, q_a.device)
    _check("fp8_block_mm", lib().fp8_block_mm(
        _ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w), _ptr(y), M, N, K, _ptr(ws), wsb,
        _stream(q_a.device)))
    return y


class PlanInfo(ctypes.Structure):
    """sq_plan_info (include/sqint8.h)."""
    _fields_ = [("kernel", ctypes.c_int32), ("grid", ctypes.c_int32), ("tile_m", ctypes.c_int32),
                ("tile_n", ctypes.c_int32), ("splits", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_uint64)]


def describe_plan(op: int, M: int, N: int, K: int, sms: int) -> dict:
    """The schedule a GEMM call would use on a device with `sms` SMs
    (sq_describe_plan; host only, no GPU needed)."""
    L = lib()
    info = PlanInfo()
    _check("sq_describe_plan", L.sq_describe_plan(op, M, N, K, sms, ctypes.byref(info)))
    return {name: getattr(info, name) for name, _ in PlanInfo._fields_}


def set_overlap(enable: bool) -> None:
    """Launch policy of the calling host thread (sq_set_overlap): when on, the
    GEMM entry points may start streaming their weights while the preceding
    kernel on the stream still runs.  Only for callers whose preceding kernel
    never writes the weights of the next call."""
    _check("sq_set_overlap", lib().sq_set_overlap(1 if enable else 0))


PEAK_I8, PEAK_F8, PEAK_BF16 = 0, 1, 2


def mma_peak(kind: int = PEAK_I8, iters: int = 8192, launches: int = 4, device=None) -> float:
    """Measured dense tensor throughput (tera-ops/s) of the current device
    for one MMA kind: sq_mma_peak launched `launches` times back to back on
    the current stream, each timed with CUDA events on that stream.  Short
    launches (the default) give the burst rate, the best of all but the
    first; long ones (iters ~ 2^21, about 0.3 s each) the rate under the power
    cap, the mean of the second half of the launches."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ops = ctypes.c_double(0.0)
    rates = []
    for i in range(launches):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        _check("sq_mma_peak", lib().sq_mma_peak(kind, iters, _stream(dev), ctypes.byref(ops)))
        b.record()
        b.synchronize()
        rates.append(ops.value / (a.elapsed_time(b) * 1e-3) / 1e12)
    if iters <= 65536:
        return max(rates[1:]) if len(rates) > 1 else rates[0]
    tail = rates[len(rates) // 2:]
    return sum(tail) / len(tail)


def selftest_wait_timeout(limit_cycles: int = 2_000_000, device=None) -> int:
    """Run the timeout self-test kernel (sq_selftest_wait_timeout) and return
    its gave_up flag (1: the wait gave up through its own limit).  The device
    error word is left set: check_device_error() then raises SQ_ERR_TIMEOUT."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    flag = torch.full((1,), -1, dtype=torch.int32, device=dev)
    _check("sq_selftest_wait_timeout",
           lib().sq_selftest_wait_timeout(limit_cycles, _ptr(flag), _stream(dev)))
    return int(flag.item())


def check_device_error(reset: bool = True) -> None:
    """Synchronise; raise SqError if a kernel latched a wait timeout."""
    _check("sq_check_device_error", lib().sq_check_device_error(1 if reset else 0))
