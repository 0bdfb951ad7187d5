"""Pins of the oracle functions for the layer's next rows: fused RMSNorm +
fold + quantisation, per-group (1 x 128) activations with gs128 weights,
group-wise W8A16, and FP8 block-scaled weights with per-group activations.

As in test_oracle_pins.py, every check compares the oracle with something it
does not compute itself: exact rational arithmetic, closed forms, invariants,
reductions to the already pinned per-token / per-channel / gs128 functions,
and torch's float8_e4m3fn conversion.
"""
from __future__ import annotations

import math
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from w8a8_int8_quantized_sq_b200 import inputs


def bf16_from_bits(bits):
    return torch.tensor(np.array(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def exact_f32_round(fr: Fraction) -> float:
    """A non-negative rational rounded to the nearest fp32, ties to even."""
    if fr == 0:
        return 0.0
    e = math.floor(math.log2(fr))
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    q = Fraction(2) ** max(e - 23, -149)
    n = fr / q
    lo = math.floor(n)
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    v = lo * q
    return math.inf if v >= Fraction(2) ** 128 else float(v)


# ============================================================ fused RMSNorm

def test_sumsq_exact_then_one_rounding():
    rng = np.random.default_rng(11)
    rows = []
    for _ in range(40):
        n = int(rng.integers(1, 600))
        v = rng.standard_normal(n) * 10.0 ** rng.integers(-20, 20, n)
        rows.append(torch.tensor(v, dtype=torch.float32).to(torch.bfloat16))
    # ties and sticky bits: 4096^2 + 1 = 2^24 + 1 is halfway between two fp32
    # numbers (ties to even: 2^24); any further positive term rounds it up
    rows.append(torch.tensor([4096.0, 1.0]).to(torch.bfloat16))
    rows.append(torch.tensor([4096.0, 1.0, 2.0 ** -60]).to(torch.bfloat16))
    rows.append(torch.tensor([4096.0, 3.0]).to(torch.bfloat16))   # 2^24 + 9 -> 2^24 + 8
    rows.append(bf16_from_bits([0x0001, 0x0003, 0x8001]))            # bf16 subnormals
    rows.append(torch.zeros(7, dtype=torch.bfloat16))
    for r in rows:
        exact = sum((Fraction(float(v)) ** 2 for v in r.float().tolist()), Fraction(0))
        assert oracle.sumsq_f32(r) == exact_f32_round(exact), r[:8]
    assert oracle.sumsq_f32(rows[-5]) == 2.0 ** 24
    assert oracle.sumsq_f32(rows[-4]) == 2.0 ** 24 + 2


def _gamma_ones(K):
    return torch.ones(K, dtype=torch.float32)


def test_rmsnorm_closed_form_constant_magnitude():
    # |h| = 2^j everywhere: ms = 4^j, r = 2^-j exactly (eps far below the
    # fp32 spacing of ms), x' = +-1, so every code is +-127 and s = f32(1/127)
    K = 256
    for j in (-3, 0, 5):
        signs = torch.where(torch.arange(K) % 3 == 0, -1.0, 1.0)
        h = (signs * 2.0 ** j).to(torch.bfloat16)[None, :]
        q, s, r = oracle.rmsnorm_quant(h, _gamma_ones(K), 1e-30)
        assert r.item() == 2.0 ** -j
        assert torch.equal(q[0].long(), (signs * 127).long())
        assert s.item() == f32(1.0 / 127.0)


def test_rmsnorm_scale_invariance():
    # scaling h by a power of two leaves r*h, hence codes and scales, unchanged
    x = inputs.gen_x(9, 384, 5, inputs.XRecipe(col_count=3, col_factor=30.0))
    g = torch.rand(384, dtype=torch.float32) + 0.5
    q0, s0, r0 = oracle.rmsnorm_quant(x, g, 1e-30)
    for j in (-7, 4):
        q1, s1, r1 = oracle.rmsnorm_quant((x.float() * 2.0 ** j).to(torch.bfloat16), g, 1e-30)
        assert torch.equal(q0, q1) and torch.equal(s0, s1)
        assert torch.equal(r1, r0 * 2.0 ** -j)


def test_rmsnorm_reconstruction_bound_fp64():
    # q * s reconstructs (h / rms) * gamma (computed in fp64 from the exact
    # mean square) within half a quantisation step plus a few fp32 roundings:
    # a dropped r, gamma, eps or 1/s fold fails this
    M, K = 24, 640
    x = inputs.gen_x(M, K, 21, inputs.XRecipe(col_count=5, col_factor=30.0, row_period=7,
                                               row_width=1, row_factor=50.0))
    w = inputs.gen_w(1, K, 22, sigma=0.1)[0]
    inv_s = (torch.rand(K, dtype=torch.float32) * 0.9 + 0.1)
    gamma = oracle.fold_norm_weight(w, inv_s, zero_centered=True)
    eps = 1e-6
    for group in (0, 128):
        q, s, r = oracle.rmsnorm_quant(x, gamma, eps, group=group)
        h = x.double()
        rms = torch.sqrt((h * h).mean(dim=1, keepdim=True) + eps)
        g64 = (1.0 + w.double()) * inv_s.double()
        want = h / rms * g64[None, :]
        sc = s.double()[:, None] if group == 0 else s.double().repeat_interleave(128, dim=1)
        err = (q.double() * sc - want).abs()
        assert torch.all(err <= 0.5 * sc * (1 + 2.0 ** -20) + 1e-6 * want.abs() + 1e-30)
        assert torch.all(q.abs() <= 127)


def test_rmsnorm_group_scales_and_token_scale_agree():
    # the row's amax is the largest block amax, and amax/127 is monotonic:
    # the per-token scale equals the largest per-group scale, exactly
    x = inputs.gen_x(16, 1024, 31, inputs.XRecipe(col_count=4, col_factor=20.0))
    g = torch.rand(1024, dtype=torch.float32) + 0.5
    _, s_tok, r0 = oracle.rmsnorm_quant(x, g, 1e-6, group=0)
    _, s_grp, r1 = oracle.rmsnorm_quant(x, g, 1e-6, group=128)
    assert torch.equal(r0, r1)
    assert torch.equal(s_grp.max(dim=1).values, s_tok)


def test_rmsnorm_zero_row_and_r_hook():
    x = inputs.gen_x(4, 256, 41)
    x[2] = 0
    g = torch.rand(256, dtype=torch.float32) + 0.5
    q, s, r = oracle.rmsnorm_quant(x, g, 1e-6)
    assert s[2].item() == 0.0 and torch.all(q[2] == 0)
    assert r[2].item() == f32(1.0 / f32(math.sqrt(f32(1e-6))))
    q2, s2, r2 = oracle.rmsnorm_quant(x, g, 1e-6, r_in=r)
    assert torch.equal(q, q2) and torch.equal(s, s2) and torch.equal(r, r2)


def test_fold_norm_weight_golden():
    # hand-worked: g = 1 + w (zero-centred), gamma = g * inv_s, all exact
    w = torch.tensor([0.0, 0.5, -1.0, 2.0]).to(torch.bfloat16)
    inv = torch.tensor([1.0, 0.5, 2.0, 0.25])
    assert oracle.fold_norm_weight(w, inv, True).tolist() == [1.0, 0.75, 0.0, 0.75]
    assert oracle.fold_norm_weight(w, inv, False).tolist() == [0.0, 0.25, -2.0, 0.5]
    assert oracle.fold_norm_weight(w, None, True).tolist() == [1.0, 1.5, 0.0, 3.0]


def test_rmsnorm_rejects_bad_arguments():
    x = torch.zeros((2, 256), dtype=torch.bfloat16)
    g = torch.ones(256)
    with pytest.raises(ValueError):
        oracle.rmsnorm_quant(x, g, 0.0)
    with pytest.raises(ValueError):
        oracle.rmsnorm_quant(x, g, 1e-6, group=64)


# ======================================================== per-group (1x128)

def test_quant_per_group_is_per_token_on_each_block():
    x = inputs.gen_x(12, 640, 51, inputs.XRecipe(col_count=6, col_factor=40.0))
    x[3, 128:256] = 0
    inv = torch.rand(640, dtype=torch.float32) + 0.25
    q, s = oracle.quant_per_group(x, inv)
    xb = x.reshape(12 * 5, 128)
    ib = inv.reshape(5, 128)
    for b in range(5):
        qb, sb = oracle.quant_per_token(xb[b::5].contiguous(), ib[b].contiguous())
        assert torch.equal(q.reshape(60, 128)[b::5], qb)
        assert torch.equal(s[:, b], sb)
    assert s[3, 1].item() == 0.0


def _rand_gs(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    q_a = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    q_w = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    s_blk = torch.rand(N, K // 128, generator=g) * 1e-3 + 1e-5
    return q_a, q_w, s_blk, g


def test_pg128_reduces_to_gs128_for_power_of_two_row_scales():
    # s_a[m, kb] = 2^j_m for every block: the scale products are exact, the
    # accumulator is 2^j_m times gs128's, and y equals gs128 with s_tok = 2^j_m
    M, N, K = 9, 64, 640
    q_a, q_w, s_blk, g = _rand_gs(M, N, K, 3)
    j = torch.randint(-12, 4, (M,), generator=g).double()
    s_tok = torch.exp2(j).float()
    s_a = s_tok[:, None].repeat(1, K // 128).contiguous()
    assert torch.equal(oracle.pg128_mm(q_a, s_a, q_w, s_blk).view(torch.int16),
                       oracle.gs128_mm(q_a, s_tok, q_w, s_blk).view(torch.int16))


def test_pg128_matches_fp64_within_the_chain_bound():
    M, N, K = 7, 96, 1280
    q_a, q_w, s_blk, g = _rand_gs(M, N, K, 4)
    s_a = torch.rand(M, K // 128, generator=g) * 0.1 + 1e-3
    y = oracle.pg128_mm(q_a, s_a, q_w, s_blk).double()
    P = torch.einsum("mbk,nbk->mnb", q_a.double().reshape(M, -1, 128),
                     q_w.double().reshape(N, -1, 128))
    sc = (s_a[:, None, :] * s_blk[None, :, :]).double()      # fp32 products, as defined
    exact = (P * sc).sum(-1)
    mag = (P.abs() * sc).sum(-1)
    nkb = K // 128
    ulp = torch.exp2(torch.floor(torch.log2(exact.abs().clamp_min(2.0 ** -126))) - 7)
    assert torch.all((y - exact).abs() <= ulp + (nkb + 2) * 2.0 ** -24 * mag)


def test_pg128_golden_small():
    # one row, one column, two K blocks of integers: P0 = 128 * 2 * 3 = 768,
    # P1 = 128 * (-1) * 5 = -640; scales 0.5*0.25 and 2*0.125 are exact:
    # acc = 768 * 0.125 - 640 * 0.25 = 96 - 160 = -64
    q_a = torch.cat([torch.full((1, 128), 2), torch.full((1, 128), -1)], 1).to(torch.int8)
    q_w = torch.cat([torch.full((1, 128), 3), torch.full((1, 128), 5)], 1).to(torch.int8)
    s_a = torch.tensor([[0.5, 2.0]])
    s_blk = torch.tensor([[0.25, 0.125]])
    assert oracle.pg128_mm(q_a, s_a, q_w, s_blk).float().item() == -64.0


# ===================================================== group-wise W8A16

def test_dequant_group_exact_for_power_of_two_scales():
    g = torch.Generator().manual_seed(5)
    q = torch.randint(-127, 128, (32, 384), generator=g, dtype=torch.int8)
    e = torch.randint(-20, 3, (32, 3), generator=g).double()
    s = torch.exp2(e).float()
    w_hat = oracle.dequant_weight_group(q, s)
    want = q.double() * s.double().repeat_interleave(128, dim=1)   # exact in bf16
    assert torch.equal(w_hat.double(), want)


def test_dequant_group_rounds_once_per_step():
    # |w_hat - q*s| is at most half a bf16 step of f32(q*s) plus the fp32
    # rounding before it (the two roundings the reading names)
    g = torch.Generator().manual_seed(6)
    q = torch.randint(-127, 128, (16, 256), generator=g, dtype=torch.int8)
    s = torch.rand(16, 2, generator=g) * 1e-2 + 1e-6
    w_hat = oracle.dequant_weight_group(q, s).double()
    exact = q.double() * s.double().repeat_interleave(128, dim=1)
    ulp = torch.exp2(torch.floor(torch.log2(exact.abs().clamp_min(2.0 ** -126))) - 7)
    assert torch.all((w_hat - exact).abs() <= 0.5 * ulp * (1 + 2.0 ** -15) + 2.0 ** -149)


def test_w8a16_group_reduces_to_per_channel_for_power_of_two_scales():
    # constant power-of-two scales per row: w_hat = q * s exactly and the
    # exact sum s * sum(x q) is the per-channel W8A16 oracle's
    M, N, K = 3, 48, 512
    x = inputs.gen_x(M, K, 7)
    g = torch.Generator().manual_seed(7)
    q = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    s_ch = torch.exp2(torch.randint(-14, -4, (N,), generator=g).double()).float()
    s_grp = s_ch[:, None].repeat(1, K // 128).contiguous()
    assert torch.equal(oracle.w8a16_group_mm(x, q, s_grp).view(torch.int16),
                       oracle.w8a16_mm(x, q, s_ch).view(torch.int16))


def test_w8a16_group_matches_exact_rational_rounding():
    M, N, K = 2, 8, 256
    x = inputs.gen_x(M, K, 8)
    g = torch.Generator().manual_seed(8)
    q = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    s = torch.rand(N, 2, generator=g) * 1e-2 + 1e-5
    y, mag = oracle.w8a16_group_mm(x, q, s, with_bound=True)
    w_hat = oracle.dequant_weight_group(q, s).float().tolist()
    xs = x.float().tolist()
    for m in range(M):
        for n in range(N):
            exact = sum((Fraction(a) * Fraction(b) for a, b in zip(xs[m], w_hat[n])), Fraction(0))
            mag_exact = sum((abs(Fraction(a) * Fraction(b)) for a, b in zip(xs[m], w_hat[n])),
                            Fraction(0))
            sign = -1 if exact < 0 else 1
            want = sign * _bf16_round_fraction(abs(exact))
            assert y[m, n].float().item() == want
            assert abs(mag[m, n].item() - float(mag_exact)) <= 1e-12 * float(mag_exact)


def _bf16_round_fraction(fr: Fraction) -> float:
    if fr == 0:
        return 0.0
    e = math.floor(math.log2(fr))
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    qq = Fraction(2) ** max(e - 7, -133)
    n = fr / qq
    lo = math.floor(n)
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return float(lo * qq)


# ===================================================================== FP8

def _torch_e4m3(vals: np.ndarray) -> np.ndarray:
    return torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_conversion_matches_torch():
    rng = np.random.default_rng(9)
    vals = list(rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-4, 3, 4000))
    # every code's value, and the halfway points between neighbouring codes
    finite = [oracle.e4m3_bits_to_f32(b) for b in range(256) if (b & 0x7F) != 0x7F]
    pos = sorted({abs(v) for v in finite})
    vals += finite
    vals += [(a + b) / 2 for a, b in zip(pos, pos[1:])]
    vals += [-(a + b) / 2 for a, b in zip(pos, pos[1:])]
    vals = np.array([v for v in vals if abs(v) <= 448.0], dtype=np.float32)
    want = _torch_e4m3(vals)
    got = np.array([oracle.f32_to_e4m3_bits(float(v)) for v in vals], dtype=np.uint8)
    # torch keeps -0 as 0x80 like the oracle; compare bit patterns
    assert np.array_equal(got, want)
    # saturation beyond the largest finite value (torch's conversion does not saturate)
    assert oracle.f32_to_e4m3_bits(449.0) == 0x7E and oracle.f32_to_e4m3_bits(-1e6) == 0xFE


def test_e4m3_decode_matches_torch():
    bits = np.arange(256, dtype=np.uint8)
    want = torch.tensor(bits).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_bits_to_f32(int(b)) for b in bits], dtype=np.float32)
    both_nan = np.isnan(want) & np.isnan(got)
    assert np.array_equal(got[~both_nan], want[~both_nan]) and np.isnan(got).sum() == 2


def test_fp8_quant_closed_form_identity():
    # a group whose values are e4m3 numbers with amax 448: scale 1, codes = values
    finite = [oracle.e4m3_bits_to_f32(b) for b in range(256) if (b & 0x7F) != 0x7F]
    rng = np.random.default_rng(10)
    row = np.array(rng.choice(finite, 256), dtype=np.float32)
    row[5] = 448.0
    row[200] = -448.0
    x = torch.tensor(row)[None, :].to(torch.bfloat16)   # e4m3 values are exact in bf16
    q, s = oracle.quant_fp8_per_group(x)
    assert torch.equal(s, torch.ones(1, 2))
    assert np.array_equal(q.numpy()[0], _torch_e4m3(row))
    wq, ws = oracle.quant_fp8_block(x.repeat(128, 1))
    assert torch.equal(ws, torch.ones(1, 2)) and torch.equal(wq[7], q[0])


def test_fp8_block_scale_is_block_amax():
    w = inputs.gen_w(256, 384, 12)
    w[130, 200] = 3.0   # one outlier: only block (1, 1) changes scale
    q, s = oracle.quant_fp8_block(w)
    wf = w.float().reshape(2, 128, 3, 128).abs().amax(dim=(1, 3))
    assert torch.equal(s, (wf / 448.0).float())
    assert s[1, 1].item() == f32(3.0 / 448.0)
    # reconstruction within half an e4m3 step (3 mantissa bits) of each value
    deq = torch.tensor(q.numpy()).view(torch.float8_e4m3fn).float()
    sc = s.repeat_interleave(128, 0).repeat_interleave(128, 1)
    err = (deq * sc - w.float()).abs()
    assert torch.all(err <= 2.0 ** -4 * w.float().abs() + 2.0 ** -10 * sc + 1e-30)


def test_fp8_block_mm_matches_exact_rational_rounding():
    M, N, K = 2, 128, 256
    x = inputs.gen_x(M, K, 13, inputs.XRecipe(col_count=2, col_factor=20.0))
    w = inputs.gen_w(N, K, 13)
    q_a, s_a = oracle.quant_fp8_per_group(x)
    q_w, s_w = oracle.quant_fp8_block(w)
    y, mag = oracle.fp8_block_mm(q_a, s_a, q_w, s_w, with_bound=True)
    a = torch.tensor(q_a.numpy()).view(torch.float8_e4m3fn).float().tolist()
    b = torch.tensor(q_w.numpy()).view(torch.float8_e4m3fn).float().tolist()
    for m in range(M):
        for n in range(0, N, 9):
            exact = Fraction(0)
            for kb in range(K // 128):
                part = sum((Fraction(a[m][k]) * Fraction(b[n][k])
                            for k in range(kb * 128, (kb + 1) * 128)), Fraction(0))
                sc = f32(s_a[m, kb].item() * s_w[n // 128, kb].item())
                exact += part * Fraction(sc)
            sign = -1 if exact < 0 else 1
            assert y[m, n].float().item() == sign * _bf16_round_fraction(abs(exact))
            assert mag[m, n].item() >= abs(float(exact)) * (1 - 1e-12)
