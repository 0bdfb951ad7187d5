"""Seeded synthetic inputs for the W8A8 / W8A16 linear layer.

This module draws the raw BF16 activations X [M, K] and raw BF16 weights
W [N, K] that every test and benchmark uses, plus the outlier structure the
workloads call for. It holds no quantisation, smoothing or GEMM arithmetic:
only a counter-based random generator, a normal transform and the
outlier multipliers.  Both the CUDA path and the CPU oracle consume the same
bytes produced here.

Generator (our own definition, stated so anyone can re-implement it):

* ``mix64`` is the SplitMix64 finaliser (Steele, Lea, Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014; constants as published by
  Vigna).  Output ``i`` of sub-stream ``t`` of seed ``S`` is
  ``mix64(key + (i + 1) * 0x9E3779B97F4A7C15)`` with
  ``key = mix64((S << 8) | t)``, all arithmetic mod 2**64.
* Normals use Box–Muller in fp64 on pairs of outputs:
  ``u1 = ((r[2p] >> 11) + 1) * 2**-53`` (in (0, 1]),
  ``u2 = (r[2p+1] >> 11) * 2**-53`` (in [0, 1)),
  ``z[2p] = sqrt(-2 ln u1) cos(2 pi u2)``, ``z[2p+1] = sqrt(-2 ln u1) sin(2 pi u2)``.
* Values are rounded fp64 -> fp32, the outlier multipliers are applied in fp32,
  and the result is rounded to BF16 with round-to-nearest-even.

Workload shapes follow the model the quantisation pages describe
(hidden 5120, intermediate 17408 on the INT8 W8A16 page, "Architecture audit";
prefill chunks of 8192 tokens on the same page's deployment notes).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Sub-stream ids.
STREAM_X = 1
STREAM_W = 2
STREAM_OUTLIER_COLS = 3

SEED_BASE = 0x5EED0000


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    v = np.array([((seed & ((1 << 56) - 1)) << 8) | (stream & 0xFF)], dtype=np.uint64)
    return mix64(v)[0]


def uniform_bits(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of sub-stream ``stream``."""
    key = stream_key(seed, stream)
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(key + idx * GAMMA)


def normals_f64(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Standard normals ``start .. start+count-1`` (start must be even)."""
    assert start % 2 == 0
    npairs = (count + 1) // 2
    r = uniform_bits(seed, stream, start, 2 * npairs)
    u1 = ((r[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (r[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = rad * np.cos(ang)
    out[1::2] = rad * np.sin(ang)
    return out[:count]


def pick_columns(seed: int, K: int, count: int) -> np.ndarray:
    """``count`` distinct column indices of ``range(K)``, sorted (seeded)."""
    if count <= 0:
        return np.zeros(0, dtype=np.int64)
    keys = uniform_bits(seed, STREAM_OUTLIER_COLS, 0, K)
    order = np.argsort(keys, kind="stable")
    return np.sort(order[:count]).astype(np.int64)


@dataclasses.dataclass(frozen=True)
class XRecipe:
    """How the activation matrix of one workload is drawn."""
    col_count: int = 0          # number of seeded outlier columns
    col_factor: float = 1.0     # their multiplier
    row_period: int = 0         # rows with (m % row_period) < row_width are scaled
    row_width: int = 0
    row_factor: float = 1.0


def gen_x(M: int, K: int, seed: int, recipe: XRecipe = XRecipe(),
          chunk_rows: Optional[int] = None) -> torch.Tensor:
    """BF16 activations [M, K] ~ N(0, 1) with the recipe's outliers (CPU)."""
    out = torch.empty((M, K), dtype=torch.bfloat16)
    if M == 0 or K == 0:
        return out
    colmul = np.ones(K, dtype=np.float32)
    if recipe.col_count:
        colmul[pick_columns(seed, K, recipe.col_count)] = np.float32(recipe.col_factor)
    rows = chunk_rows or max(1, (1 << 22) // K)
    for r0 in range(0, M, rows):
        r1 = min(M, r0 + rows)
        z = normals_f64(seed, STREAM_X, r0 * K, (r1 - r0) * K).astype(np.float32)
        z = z.reshape(r1 - r0, K)
        z *= colmul[None, :]
        if recipe.row_period:
            m = np.arange(r0, r1)
            sel = (m % recipe.row_period) < recipe.row_width
            z[sel] *= np.float32(recipe.row_factor)
        out[r0:r1] = torch.from_numpy(z).to(torch.bfloat16)
    return out


def gen_w(N: int, K: int, seed: int, sigma: float = 0.02,
          chunk_rows: Optional[int] = None) -> torch.Tensor:
    """BF16 weights [N, K] ~ N(0, sigma^2) (CPU)."""
    out = torch.empty((N, K), dtype=torch.bfloat16)
    if N == 0 or K == 0:
        return out
    rows = chunk_rows or max(1, (1 << 22) // K)
    for r0 in range(0, N, rows):
        r1 = min(N, r0 + rows)
        z = normals_f64(seed, STREAM_W, r0 * K, (r1 - r0) * K).astype(np.float32)
        z *= np.float32(sigma)
        out[r0:r1] = torch.from_numpy(z.reshape(r1 - r0, K)).to(torch.bfloat16)
    return out


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, distributions and the layer variant."""
    name: str
    M: int
    K: int
    N: int
    variant: str                # "w8a8", "gs128" or "w8a16"
    x: XRecipe
    smooth: bool                # SmoothQuant factors from the max|X|/max|W| rule
    seed: int

    def make_x(self, M: Optional[int] = None) -> torch.Tensor:
        return gen_x(self.M if M is None else M, self.K, self.seed, self.x)

    def make_w(self) -> torch.Tensor:
        return gen_w(self.N, self.K, self.seed)


OUTLIER_COLS_1PCT = 51  # 1% of 5120 columns

WORKLOADS: Sequence[Workload] = (
    Workload("tiny_w8a8_M16_K256_N128", 16, 256, 128, "w8a8",
             XRecipe(col_count=4, col_factor=20.0), True, SEED_BASE + 0),
    Workload("decode_w8a8_M8_K5120_N5120", 8, 5120, 5120, "w8a8",
             XRecipe(col_count=OUTLIER_COLS_1PCT, col_factor=30.0), True, SEED_BASE + 1),
    Workload("prefill_w8a8_M8192_K5120_N34816", 8192, 5120, 34816, "w8a8",
             XRecipe(col_count=OUTLIER_COLS_1PCT, col_factor=30.0,
                     row_period=512, row_width=4, row_factor=50.0), True, SEED_BASE + 2),
    Workload("gs128_w8a8_M2048_K5120_N5120", 2048, 5120, 5120, "gs128",
             XRecipe(), False, SEED_BASE + 3),
    Workload("w8a16_down_proj_K17408_N5120", 16, 17408, 5120, "w8a16",
             XRecipe(row_period=512, row_width=1, row_factor=50.0), False, SEED_BASE + 4),
)

W8A16_M_VALUES = (1, 16, 8192)


def workload(i: int) -> Workload:
    return WORKLOADS[i]
