"""Parity of the next rows' CUDA path (through the C ABI) with the CPU oracle:
fused RMSNorm + fold + quantisation, per-group activations with gs128
weights, group-wise W8A16, and FP8 block-scaled weights with per-group
activations.

Bars: bit-exact on every code and scale and on the per-group GEMM output;
the RMSNorm factor r equal to the oracle's (the kernel sums squares in fp64
and rounds once; the oracle rounds the exact sum: they can differ only when
the sum sits within about K * 2^-53 of an fp32 rounding boundary, so the test
reports such rows, allows one ulp there, and checks the codes of every row
against the oracle given the kernel's r); group-wise W8A16 and FP8 outputs
within one bf16 ulp plus the fp32 accumulation bound stated in each check.
"""
from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import oracle
import w8a8_int8_quantized_sq_b200 as sq
from w8a8_int8_quantized_sq_b200 import inputs
from tests.prep import bf16_ulp, workload

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _bits(t: torch.Tensor) -> torch.Tensor:
    t = t.cpu()
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def assert_same(gpu: torch.Tensor, ref: torch.Tensor, what: str):
    g, r = _bits(gpu), _bits(ref)
    if not torch.equal(g, r):
        bad = (g != r).nonzero()
        raise AssertionError(f"{what}: {bad.shape[0]} of {r.numel()} differ; first at "
                             f"{bad[0].tolist()}: gpu {g[tuple(bad[0])]} ref {r[tuple(bad[0])]}")


@functools.lru_cache(maxsize=4)
def norm_weight(K: int, seed: int = 77) -> torch.Tensor:
    """Zero-centred norm weight w ~ N(0, 0.1) (bf16 [K]); the norm scales by 1 + w."""
    return inputs.gen_w(1, K, inputs.SEED_BASE + seed, sigma=0.1)[0].contiguous()


# ============================================================ fused RMSNorm

def _check_rmsnorm(h, gamma, group):
    q, sc, r = sq.rmsnorm_quant(h.cuda(), gamma.cuda(), EPS, group=group)
    r = r.cpu()
    _, _, r_ref = oracle.rmsnorm_quant(h, gamma, EPS, group=group)
    diff = (r != r_ref).nonzero().flatten()
    if diff.numel():
        ulp = torch.abs(r_ref.view(torch.int32).long() - r.view(torch.int32).long())
        assert int(ulp.max()) <= 1, f"inv_rms off by {int(ulp.max())} ulp"
        print(f"\nRMSNorm M={h.shape[0]} K={h.shape[1]}: {diff.numel()} rows with r one ulp "
              "from the exact-sum value")
    assert diff.numel() <= max(1, h.shape[0] // 1000)
    # every code and scale, given the kernel's r
    q_ref, sc_ref, _ = oracle.rmsnorm_quant(h, gamma, EPS, group=group, r_in=r)
    assert_same(q, q_ref, "codes")
    assert_same(sc, sc_ref, "scales")


@pytest.mark.parametrize("group", [0, 128])
def test_rmsnorm_quant_prefill(group):
    """Hidden state of the prefill workload (M=8192, K=5120), zero-centred norm
    weight with the workload's 1/s folded in."""
    d = workload(2)
    w = norm_weight(5120)
    gamma = oracle.fold_norm_weight(w, d["inv_s"], zero_centered=True)
    g_gpu = sq.fold_norm_weight(w.cuda(), d["inv_s"].cuda(), zero_centered=True)
    assert_same(g_gpu, gamma, "folded norm weight")
    _check_rmsnorm(d["x"], gamma, group)


@pytest.mark.parametrize("M,K", [(1, 128), (7, 256), (129, 384), (300, 2048), (33, 6272),
                                 (16, 17408), (5, 24576)])
@pytest.mark.parametrize("group", [0, 128])
def test_rmsnorm_quant_shapes(M, K, group):
    h = inputs.gen_x(M, K, 91, inputs.XRecipe(col_count=3, col_factor=40.0, row_period=5,
                                               row_width=1, row_factor=50.0))
    h[M // 2] = 0  # an all-zero row: r = 1/sqrt(eps), zero codes and scales
    gamma = oracle.fold_norm_weight(norm_weight(K), torch.rand(K) + 0.25, zero_centered=True)
    _check_rmsnorm(h, gamma, group)


def test_rmsnorm_quant_errors():
    h = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(256, device="cuda")
    with pytest.raises(sq.SqError) as e:
        sq.rmsnorm_quant(h, g, 0.0)
    assert e.value.code == 2
    with pytest.raises(sq.SqError) as e:
        sq.rmsnorm_quant(h, g, EPS, group=64)
    assert e.value.code == 2


# ======================================================== per-group (1x128)

@pytest.mark.parametrize("smooth", [False, True])
def test_quant_per_group_config3(smooth):
    d = workload(3)
    inv = (torch.rand(5120, generator=torch.Generator().manual_seed(3)) + 0.25) if smooth else None
    q_ref, s_ref = oracle.quant_per_group(d["x"], inv)
    q, s = sq.quant_per_group(d["x"].cuda(), inv.cuda() if smooth else None)
    assert_same(q, q_ref, "q_a")
    assert_same(s, s_ref, "s_a")


@pytest.mark.parametrize("M,K", [(1, 128), (9, 17408), (3, 25600)])
def test_quant_per_group_shapes(M, K):
    x = inputs.gen_x(M, K, 92, inputs.XRecipe(col_count=5, col_factor=40.0))
    x[0, 128:256] = 0
    inv = torch.rand(K) + 0.25
    q_ref, s_ref = oracle.quant_per_group(x, inv)
    q, s = sq.quant_per_group(x.cuda(), inv.cuda())
    assert_same(q, q_ref, "q_a")
    assert_same(s, s_ref, "s_a")


def test_pg128_config3_shape():
    """Per-group activations of the gs128 workload (M=2048, K=5120, N=5120)."""
    d = workload(3)
    q_a, s_a = oracle.quant_per_group(d["x"])
    ref = oracle.pg128_mm(q_a, s_a, d["q_w"], d["s_blk"])
    y = sq.w8a8_pg128_mm(q_a.cuda(), s_a.cuda(), d["q_w"].cuda(), d["s_blk"].cuda())
    assert_same(y, ref, "y pg128")


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (100, 256, 1024), (130, 384, 17408)])
def test_pg128_shapes(M, N, K):
    g = torch.Generator().manual_seed(M + N + K + 1)
    q_a = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    q_w = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    s_a = torch.rand(M, K // 128, generator=g) * 0.1 + 1e-3
    s_blk = torch.rand(N, K // 128, generator=g) * 1e-3 + 1e-5
    y = sq.w8a8_pg128_mm(q_a.cuda(), s_a.cuda(), q_w.cuda(), s_blk.cuda())
    assert_same(y, oracle.pg128_mm(q_a, s_a, q_w, s_blk), "y pg128")


# ===================================================== group-wise W8A16

def _check_within(y, ref, mag, K, terms_per_step, what):
    """|y - ref| <= ulp(ref) + gamma * mag with gamma covering an fp32
    accumulation of K exact products in steps of `terms_per_step`, plus the
    split-K combination."""
    gamma = (K / terms_per_step + 8) * 2.0 ** -22
    diff = (y.double() - ref.double()).abs()
    ulp = bf16_ulp(ref)
    assert torch.all(diff <= ulp + gamma * mag), (what, float((diff - ulp - gamma * mag).max()))
    beyond = int((diff > ulp).sum())
    print(f"\n{what}: {beyond} of {diff.numel()} outputs beyond 1 bf16 ulp, max "
          f"{float((diff / ulp).max()):.3f} ulp")
    assert beyond <= max(1, diff.numel() // 1000)


def _w8a16g(x, q_w, s_grp, rows=None, what="W8A16 group"):
    y = sq.w8a16_group_mm(x.cuda(), q_w.cuda(), s_grp.cuda()).cpu()
    if rows is not None:
        y = y[rows]
    ref, mag = oracle.w8a16_group_mm(x, q_w, s_grp, rows=rows, with_bound=True)
    _check_within(y, ref, mag, x.shape[1], 16, what)


@functools.lru_cache(maxsize=1)
def w8a16_group_weights():
    wl = inputs.workload(4)
    w = wl.make_w()
    return oracle.quant_weight(w, None, group=128)


@pytest.mark.parametrize("M", [1, 16])
def test_w8a16_group_decode(M):
    q_w, s_grp = w8a16_group_weights()
    x = inputs.workload(4).make_x(M)
    _w8a16g(x, q_w, s_grp, what=f"W8A16 group M={M} K=17408 N=5120")


def test_w8a16_group_prefill_every_row_tile():
    q_w, s_grp = w8a16_group_weights()
    x = workload(4, 8192)["x"]
    rng = np.random.default_rng(8193)
    rows = sorted({0, 511, 512, 8191} | {t * 128 + int(rng.integers(0, 128)) for t in range(64)})
    _w8a16g(x, q_w, s_grp, rows=rows, what="W8A16 group M=8192 K=17408 N=5120 (sampled rows)")


@pytest.mark.parametrize("M,N,K", [(3, 144, 256), (17, 144, 384), (32, 256, 1280),
                                   (8, 5120, 5120), (33, 256, 640)])
def test_w8a16_group_shapes(M, N, K):
    x = inputs.gen_x(M, K, 6)
    w = inputs.gen_w(N, K, 6)
    q_w, s_grp = oracle.quant_weight(w, None, group=128)
    _w8a16g(x, q_w, s_grp, what=f"W8A16 group M={M} K={K} N={N}")


# ===================================================================== FP8

@pytest.mark.parametrize("smooth", [False, True])
def test_quant_fp8_config3_shape(smooth):
    d = workload(3)
    inv = (torch.rand(5120, generator=torch.Generator().manual_seed(4)) + 0.25) if smooth else None
    q_ref, s_ref = oracle.quant_fp8_per_group(d["x"], inv)
    q, s = sq.quant_fp8_per_group(d["x"].cuda(), inv.cuda() if smooth else None)
    assert_same(q, q_ref, "fp8 q_a")
    assert_same(s, s_ref, "fp8 s_a")
    sm = (torch.rand(5120, generator=torch.Generator().manual_seed(5)) + 0.5) if smooth else None
    wq_ref, ws_ref = oracle.quant_fp8_block(d["w"], sm)
    wq, ws = sq.quant_fp8_block(d["w"].cuda(), sm.cuda() if smooth else None)
    assert_same(wq, wq_ref, "fp8 q_w")
    assert_same(ws, ws_ref, "fp8 s_w")


def test_quant_fp8_edges():
    x = inputs.gen_x(5, 384, 93, inputs.XRecipe(col_count=2, col_factor=40.0))
    x[1, :128] = 0                       # an all-zero group
    x[2, 5] = -1e-30                     # rounds to -0 in its group
    q_ref, s_ref = oracle.quant_fp8_per_group(x)
    q, s = sq.quant_fp8_per_group(x.cuda())
    assert_same(q, q_ref, "fp8 q_a edges")
    assert_same(s, s_ref, "fp8 s_a edges")
    w = inputs.gen_w(256, 256, 94)
    w[:128, :128] = 0                    # an all-zero block
    wq_ref, ws_ref = oracle.quant_fp8_block(w)
    wq, ws = sq.quant_fp8_block(w.cuda())
    assert_same(wq, wq_ref, "fp8 q_w edges")
    assert_same(ws, ws_ref, "fp8 s_w edges")


def _fp8_gemm_check(q_a, s_a, q_w, s_w, rows=None, what="FP8 block"):
    y = sq.fp8_block_mm(q_a.cuda(), s_a.cuda(), q_w.cuda(), s_w.cuda()).cpu()
    if rows is not None:
        y = y[rows]
    ref, mag = oracle.fp8_block_mm(q_a, s_a, q_w, s_w, rows=rows, with_bound=True)
    # inside a K block the tensor core accumulates 128 exact products in fp32
    # (steps of 32); the block partials then go through the fp32 fmaf chain
    _check_within(y, ref, mag, q_a.shape[1], 32, what)


def test_fp8_block_config3_shape():
    d = workload(3)
    q_a, s_a = oracle.quant_fp8_per_group(d["x"])
    q_w, s_w = oracle.quant_fp8_block(d["w"])
    _fp8_gemm_check(q_a, s_a, q_w, s_w, what="FP8 block M=2048 K=5120 N=5120")


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (100, 256, 1024), (130, 384, 17408)])
def test_fp8_block_shapes(M, N, K):
    x = inputs.gen_x(M, K, 95, inputs.XRecipe(col_count=3, col_factor=30.0))
    w = inputs.gen_w(N, K, 95)
    q_a, s_a = oracle.quant_fp8_per_group(x)
    q_w, s_w = oracle.quant_fp8_block(w)
    _fp8_gemm_check(q_a, s_a, q_w, s_w, what=f"FP8 block M={M} K={K} N={N}")
    sq.check_device_error()


# ------------------------------------------- 256-wide block-scaled pair tiles

def test_block_scaled_wide_tiles_with_a_ragged_last_tile():
    """M=8192, N=1920, K=256: enough tiles that the pair kernels take 256-wide
    B tiles, and N % 256 = 128 leaves the last tile half filled (zero-filled
    weight rows, guarded scales and stores).  gs128 bit-exact, FP8 within
    its bound, on a row sample."""
    M, N, K = 8192, 1920, 256
    assert sq.describe_plan(sq.OP_GS128, M, N, K, 148)["tile_n"] == 256
    assert sq.describe_plan(sq.OP_FP8BLK, M, N, K, 148)["tile_n"] == 256
    x = inputs.gen_x(M, K, 96, inputs.XRecipe(col_count=3, col_factor=30.0, row_period=512,
                                               row_width=4, row_factor=50.0))
    w = inputs.gen_w(N, K, 96)
    rng = np.random.default_rng(96)
    rows = sorted({0, 255, 256, 8191} | set(rng.integers(0, M, 60).tolist()))
    # gs128 (weights as the MMA's A operand)
    q_a, s_tok = oracle.quant_per_token(x)
    q_w, s_blk = oracle.quant_weight(w, None, group=128)
    y = sq.w8a8_gs128_mm(q_a.cuda(), s_tok.cuda(), q_w.cuda(), s_blk.cuda()).cpu()
    assert_same(y[rows], oracle.gs128_mm(q_a, s_tok, q_w, s_blk, rows=rows), "gs128 wide tiles")
    # FP8 blocks (tokens as the MMA's A operand)
    qf_a, sf_a = oracle.quant_fp8_per_group(x)
    qf_w, sf_w = oracle.quant_fp8_block(w)
    _fp8_gemm_check(qf_a, sf_a, qf_w, sf_w, rows=rows, what="FP8 block M=8192 K=256 N=1920 (rows)")
    sq.check_device_error()


def test_mma_peak_probe_is_plausible():
    """The issue-rate probe behind the roofline denominators: dense INT8 and
    FP8 rates between 1 and 6 POPS on a B200 (4.5 nominal), BF16 about half."""
    i8 = sq.mma_peak(sq.PEAK_I8)
    f8 = sq.mma_peak(sq.PEAK_F8)
    bf = sq.mma_peak(sq.PEAK_BF16)
    print(f"\nmeasured dense rates: INT8 {i8:.0f}, FP8 {f8:.0f}, BF16 {bf:.0f} TOPS")
    assert 1000 < i8 < 6000 and 1000 < f8 < 6000
    assert 0.35 < bf / i8 < 0.65
    sq.check_device_error()
