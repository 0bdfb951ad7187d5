"""ctypes wrapper of the CPU oracle (TEST INFRASTRUCTURE ONLY).

Only the tests, the smoke check of the package entry file and the benchmark's
CPU-baseline leg may import this package.  The CUDA library and its Python
binding never import it.  All arrays are CPU torch tensors; BF16 data travels
as its raw 16-bit pattern.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import torch

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        L = _lib
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f64_to_bf16.restype = ctypes.c_uint16
        L.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_get_threads.restype = ctypes.c_int
        vp, i64, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double
        L.oracle_smooth_factors.argtypes = [vp, i64, i64, vp, i64, dbl, dbl, vp, vp]
        L.oracle_fold_weight.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_quant_weight.argtypes = [vp, i64, i64, vp, i64, vp, vp]
        L.oracle_quant_per_token.argtypes = [vp, i64, i64, vp, vp, vp]
        L.oracle_mm_i32.argtypes = [vp, vp, i64, i64, i64, vp, i64, vp]
        L.oracle_epilogue_ch.argtypes = [vp, vp, vp, i64, i64, vp]
        L.oracle_w8a8_scaled_mm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, i64, vp]
        L.oracle_gs128_mm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, i64, vp]
        L.oracle_w8a16_mm.argtypes = [vp, vp, vp, i64, i64, i64, vp, i64, vp, vp]
        flt, i32 = ctypes.c_float, ctypes.c_int
        L.oracle_fold_norm_weight.argtypes = [vp, i64, i32, vp, vp]
        L.oracle_sumsq_f32.argtypes = [vp, i64]
        L.oracle_sumsq_f32.restype = ctypes.c_float
        L.oracle_rmsnorm_quant.argtypes = [vp, i64, i64, vp, flt, i64, vp, vp, vp, vp]
        L.oracle_quant_per_group.argtypes = [vp, i64, i64, vp, vp, vp]
        L.oracle_pg128_mm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, i64, vp]
        L.oracle_dequant_weight_group.argtypes = [vp, vp, i64, i64, vp]
        L.oracle_w8a16_group_mm.argtypes = [vp, vp, vp, i64, i64, i64, vp, i64, vp, vp]
        L.oracle_f32_to_e4m3.argtypes = [flt]
        L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_f32.restype = flt
        L.oracle_quant_fp8_per_group.argtypes = [vp, i64, i64, vp, vp, vp]
        L.oracle_quant_fp8_block.argtypes = [vp, i64, i64, vp, vp, vp]
        L.oracle_fp8_block_mm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, i64, vp, vp]
        for name in ("oracle_smooth_factors", "oracle_fold_weight", "oracle_quant_weight",
                     "oracle_quant_per_token", "oracle_mm_i32", "oracle_epilogue_ch",
                     "oracle_w8a8_scaled_mm", "oracle_gs128_mm", "oracle_w8a16_mm",
                     "oracle_fold_norm_weight", "oracle_rmsnorm_quant",
                     "oracle_quant_per_group", "oracle_pg128_mm",
                     "oracle_dequant_weight_group", "oracle_w8a16_group_mm",
                     "oracle_quant_fp8_per_group", "oracle_quant_fp8_block",
                     "oracle_fp8_block_mm"):
            getattr(L, name).restype = ctypes.c_int
    return _lib


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous(), "oracle takes contiguous CPU tensors"
    return ctypes.c_void_p(t.data_ptr())


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"{what}: oracle rejected its arguments (code {rc})")


def _rows(rows: Optional[Sequence[int]], M: int):
    if rows is None:
        return None, M
    r = torch.as_tensor(list(rows), dtype=torch.int64).contiguous()
    return r, r.numel()


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def threads() -> int:
    return lib().oracle_get_threads()


def f32_to_bf16_bits(v: float) -> int:
    return lib().oracle_f32_to_bf16(v)


def f64_to_bf16_bits(v: float) -> int:
    return lib().oracle_f64_to_bf16(v)


def smooth_factors(x: torch.Tensor, w: torch.Tensor, cap: float = 16.0, floor: float = 1e-5):
    """(s, inv_s), fp32 [K]: max|X_j|^(1/2) / max|W_j|^(1/2), capped (SmoothQuant rule)."""
    M, K = x.shape
    N = w.shape[0]
    s = torch.empty(K, dtype=torch.float32)
    inv = torch.empty(K, dtype=torch.float32)
    _check(lib().oracle_smooth_factors(_p(x.contiguous()), M, K, _p(w.contiguous()), N,
                                       cap, floor, _p(s), _p(inv)), "smooth_factors")
    return s, inv


def fold_weight(w: torch.Tensor, s: Optional[torch.Tensor]) -> torch.Tensor:
    N, K = w.shape
    out = torch.empty((N, K), dtype=torch.float32)
    _check(lib().oracle_fold_weight(_p(w.contiguous()), N, K, _p(s), _p(out)), "fold_weight")
    return out


def quant_weight(w: torch.Tensor, s: Optional[torch.Tensor] = None, group: int = 0):
    """(q_w int8 [N,K], scales fp32 [N] or [N, K/group])."""
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.int8)
    nblk = K // group if group else 1
    sc = torch.empty((N, nblk) if group else (N,), dtype=torch.float32)
    _check(lib().oracle_quant_weight(_p(w.contiguous()), N, K, _p(s), group, _p(q), _p(sc)),
           "quant_weight")
    return q, sc


def quant_per_token(x: torch.Tensor, inv_s: Optional[torch.Tensor] = None):
    """(q_a int8 [M,K], s_tok fp32 [M])."""
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8)
    s = torch.empty(M, dtype=torch.float32)
    _check(lib().oracle_quant_per_token(_p(x.contiguous()), M, K, _p(inv_s), _p(q), _p(s)),
           "quant_per_token")
    return q, s


def mm_i32(q_a: torch.Tensor, q_w: torch.Tensor, rows=None) -> torch.Tensor:
    M, K = q_a.shape
    N = q_w.shape[0]
    r, nr = _rows(rows, M)
    acc = torch.empty((nr, N), dtype=torch.int32)
    _check(lib().oracle_mm_i32(_p(q_a), _p(q_w), M, N, K, _p(r), nr, _p(acc)), "mm_i32")
    return acc


def epilogue_ch(acc: torch.Tensor, s_tok: torch.Tensor, s_ch: torch.Tensor) -> torch.Tensor:
    R, N = acc.shape
    y = torch.empty((R, N), dtype=torch.bfloat16)
    _check(lib().oracle_epilogue_ch(_p(acc.contiguous()), _p(s_tok.contiguous()),
                                    _p(s_ch.contiguous()), R, N, _p(y)), "epilogue_ch")
    return y


def w8a8_scaled_mm(q_a, s_tok, q_w, s_ch, rows=None) -> torch.Tensor:
    M, K = q_a.shape
    N = q_w.shape[0]
    r, nr = _rows(rows, M)
    y = torch.empty((nr, N), dtype=torch.bfloat16)
    _check(lib().oracle_w8a8_scaled_mm(_p(q_a), _p(s_tok), _p(q_w), _p(s_ch), M, N, K,
                                       _p(r), nr, _p(y)), "w8a8_scaled_mm")
    return y


def gs128_mm(q_a, s_tok, q_w, s_blk, rows=None) -> torch.Tensor:
    M, K = q_a.shape
    N = q_w.shape[0]
    r, nr = _rows(rows, M)
    y = torch.empty((nr, N), dtype=torch.bfloat16)
    _check(lib().oracle_gs128_mm(_p(q_a), _p(s_tok), _p(q_w), _p(s_blk.contiguous()), M, N, K,
                                 _p(r), nr, _p(y)), "gs128_mm")
    return y


def w8a16_mm(x, q_w, s_ch, rows=None, with_bound: bool = False):
    """y bf16 [rows, N]; with_bound also returns s_ch * sum|x q| (fp64)."""
    M, K = x.shape
    N = q_w.shape[0]
    r, nr = _rows(rows, M)
    y = torch.empty((nr, N), dtype=torch.bfloat16)
    mag = torch.empty((nr, N), dtype=torch.float64) if with_bound else None
    _check(lib().oracle_w8a16_mm(_p(x.contiguous()), _p(q_w), _p(s_ch), M, N, K, _p(r), nr,
                                 _p(y), _p(mag)), "w8a16_mm")
    return (y, mag) if with_bound else y


# ------------------------------------------------------------ next rows

def fold_norm_weight(w_norm: torch.Tensor, inv_s: Optional[torch.Tensor],
                     zero_centered: bool = True) -> torch.Tensor:
    """gamma fp32 [K] = (1 + w or w) * inv_s: the norm weight with 1/s folded in."""
    K = w_norm.numel()
    g = torch.empty(K, dtype=torch.float32)
    _check(lib().oracle_fold_norm_weight(_p(w_norm.contiguous()), K, 1 if zero_centered else 0,
                                         _p(inv_s), _p(g)), "fold_norm_weight")
    return g


def sumsq_f32(h: torch.Tensor) -> float:
    """Exact sum of squares of a bf16 vector, rounded once to fp32."""
    h = h.contiguous()
    return lib().oracle_sumsq_f32(_p(h), h.numel())


def rmsnorm_quant(h: torch.Tensor, gamma: torch.Tensor, eps: float, group: int = 0,
                  r_in: Optional[torch.Tensor] = None):
    """(q int8 [M,K], scales fp32 [M] or [M, K/128], r fp32 [M]); group 0 = per token."""
    M, K = h.shape
    g = K if group == 0 else group
    q = torch.empty((M, K), dtype=torch.int8)
    sc = torch.empty((M,) if g == K else (M, K // g), dtype=torch.float32)
    r = torch.empty(M, dtype=torch.float32)
    _check(lib().oracle_rmsnorm_quant(_p(h.contiguous()), M, K, _p(gamma.contiguous()), eps, g,
                                      _p(r_in), _p(q), _p(sc), _p(r)), "rmsnorm_quant")
    return q, sc, r


def quant_per_group(x: torch.Tensor, inv_s: Optional[torch.Tensor] = None):
    """(q int8 [M,K], s_a fp32 [M, K/128])."""
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8)
    s = torch.empty((M, K // 128), dtype=torch.float32)
    _check(lib().oracle_quant_per_group(_p(x.contiguous()), M, K, _p(inv_s), _p(q), _p(s)),
           "quant_per_group")
    return q, s


def pg128_mm(q_a, s_a, q_w, s_blk, rows=None) -> torch.Tensor:
    M, K = q_a.shape
    N = q_w.shape[0]
    r, nr = _rows(rows, M)
    y = torch.empty((nr, N), dtype=torch.bfloat16)
    _check(lib().oracle_pg128_mm(_p(q_a), _p(s_a.contiguous()), _p(q_w), _p(s_blk.contiguous()),
                                 M, N, K, _p(r), nr, _p(y)), "pg128_mm")
    return y


def dequant_weight_group(q_w: torch.Tensor, s_grp: torch.Tensor) -> torch.Tensor:
    N, K = q_w.shape
    w = torch.empty((N, K), dtype=torch.bfloat16)
    _check(lib().oracle_dequant_weight_group(_p(q_w), _p(s_grp.contiguous()), N, K, _p(w)),
           "dequant_weight_group")
    return w


def w8a16_group_mm(x, q_w, s_grp, rows=None, with_bound: bool = False):
    """y bf16 [rows, N]; with_bound also returns sum|x w_hat| (fp64)."""
    M, K = x.shape
    N = q_w.shape[0]
    r, nr = _rows(rows, M)
    y = torch.empty((nr, N), dtype=torch.bfloat16)
    mag = torch.empty((nr, N), dtype=torch.float64) if with_bound else None
    _check(lib().oracle_w8a16_group_mm(_p(x.contiguous()), _p(q_w), _p(s_grp.contiguous()),
                                       M, N, K, _p(r), nr, _p(y), _p(mag)), "w8a16_group_mm")
    return (y, mag) if with_bound else y


def f32_to_e4m3_bits(v: float) -> int:
    return lib().oracle_f32_to_e4m3(v)


def e4m3_bits_to_f32(b: int) -> float:
    return lib().oracle_e4m3_to_f32(b)


def quant_fp8_per_group(x: torch.Tensor, inv_s: Optional[torch.Tensor] = None):
    """(q e4m3 bits uint8 [M,K], s_a fp32 [M, K/128])."""
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8)
    s = torch.empty((M, K // 128), dtype=torch.float32)
    _check(lib().oracle_quant_fp8_per_group(_p(x.contiguous()), M, K, _p(inv_s), _p(q), _p(s)),
           "quant_fp8_per_group")
    return q, s


def quant_fp8_block(w: torch.Tensor, smooth: Optional[torch.Tensor] = None):
    """(q e4m3 bits uint8 [N,K], s_w fp32 [N/128, K/128])."""
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8)
    s = torch.empty((N // 128, K // 128), dtype=torch.float32)
    _check(lib().oracle_quant_fp8_block(_p(w.contiguous()), N, K, _p(smooth), _p(q), _p(s)),
           "quant_fp8_block")
    return q, s


def fp8_block_mm(q_a, s_a, q_w, s_w, rows=None, with_bound: bool = False):
    """y bf16 [rows, N]; with_bound also returns sum_kb |scale| sum|a w| (fp64)."""
    M, K = q_a.shape
    N = q_w.shape[0]
    r, nr = _rows(rows, M)
    y = torch.empty((nr, N), dtype=torch.bfloat16)
    mag = torch.empty((nr, N), dtype=torch.float64) if with_bound else None
    _check(lib().oracle_fp8_block_mm(_p(q_a.contiguous()), _p(s_a.contiguous()),
                                     _p(q_w.contiguous()), _p(s_w.contiguous()), M, N, K,
                                     _p(r), nr, _p(y), _p(mag)), "fp8_block_mm")
    return (y, mag) if with_bound else y
