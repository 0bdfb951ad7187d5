"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute itself:
hand-worked examples (tests/golden), closed forms, invariants the pages
state (the SmoothQuant fold is function preserving, the weight ratio is a
separable per-row x per-column scale), brute force on tiny inputs, and
library routines (numpy integer matmul, exact rational rounding).
"""
from __future__ import annotations

import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from w8a8_int8_quantized_sq_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def bits_to_f32(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (b & 0xFFFF) << 16))[0]


# ---------------------------------------------------------------- conversions

def test_f32_to_bf16_matches_torch_rne():
    rng = np.random.default_rng(1)
    vals = list(rng.standard_normal(2000).astype(np.float32) * 1000)
    # exact ties: bf16 value plus half a spacing
    for base in (1.0, 3.0, 255.0, -7.0, 1e-3):
        b = np.float32(base)
        u = np.frombuffer(b.tobytes(), dtype=np.uint32)[0]
        vals.append(np.frombuffer(np.uint32(u + 0x8000).tobytes(), dtype=np.float32)[0])
        vals.append(np.frombuffer(np.uint32(u + 0x18000).tobytes(), dtype=np.float32)[0])
    ref = torch.tensor(np.array(vals, dtype=np.float32)).to(torch.bfloat16).view(torch.int16)
    got = [oracle.f32_to_bf16_bits(float(v)) for v in vals]
    assert [int(r) & 0xFFFF for r in ref.tolist()] == got


def _exact_bf16_round(d: float) -> float:
    """Round a double to 8 significant bits, ties to even, with rationals."""
    if d == 0:
        return 0.0
    f = Fraction(d)
    s = -1 if f < 0 else 1
    a = abs(f)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (e - 7)
    n = a / q
    lo = math.floor(n)
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return float(s * lo * q)


def test_f64_to_bf16_single_rounding():
    rng = np.random.default_rng(2)
    vals = list(rng.standard_normal(500) * 10.0 ** rng.integers(-6, 6, 500))
    # values just above a tie: a double-rounding implementation (f64 -> f32
    # -> bf16) gets these wrong
    vals += [1.0 + 2.0 ** -8 + 2.0 ** -40, 3.0 + 2.0 ** -7 + 2.0 ** -45,
             -(1.0 + 2.0 ** -8 + 2.0 ** -30), 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]
    for v in vals:
        want = _exact_bf16_round(float(v))
        got = bits_to_f32(oracle.f64_to_bf16_bits(float(v)))
        assert got == want, (v, got, want)


# --------------------------------------------------------------- golden files

def _parse_rows(path):
    rows = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append(line)
    return rows


def test_golden_quant_per_token():
    for line in _parse_rows(os.path.join(GOLDEN, "quant_per_token.txt")):
        xs, inv, q, s = [p.split() for p in line.split("|")]
        x = bf16([float(v) for v in xs])[None, :]
        inv_s = torch.tensor([float(v) for v in inv], dtype=torch.float32)
        qa, st = oracle.quant_per_token(x, inv_s)
        assert qa[0].tolist() == [int(v) for v in q], line
        assert st[0].item() == float(s[0]), line


def _golden_kv(name):
    out = {}
    for line in _parse_rows(os.path.join(GOLDEN, name)):
        k, v = line.split(":", 1)
        out[k.strip()] = v.strip()
    return out


def _mat(s, dtype):
    return torch.tensor([[float(v) for v in r.split()] for r in s.split(";")]).to(dtype)


def test_golden_scaled_mm():
    g = _golden_kv("scaled_mm.txt")
    qa = _mat(g["q_a"], torch.int8)
    qw = _mat(g["q_w"], torch.int8)
    acc = oracle.mm_i32(qa, qw)
    assert acc.tolist() == _mat(g["acc"], torch.int32).tolist()
    s_tok = torch.tensor([float(v) for v in g["s_tok"].split()], dtype=torch.float32)
    s_ch = torch.tensor([float(v) for v in g["s_ch"].split()], dtype=torch.float32)
    y = oracle.w8a8_scaled_mm(qa, s_tok, qw, s_ch)
    assert y.float().tolist() == _mat(g["y"], torch.float32).tolist()
    assert torch.equal(oracle.epilogue_ch(acc, s_tok, s_ch), y)
    racc = torch.tensor([[int(v) for v in g["round_acc"].split()]], dtype=torch.int32)
    n = racc.shape[1]
    yr = oracle.epilogue_ch(racc, torch.ones(1), torch.ones(n))
    assert yr.float()[0].tolist() == [float(v) for v in g["round_y"].split()]


def test_golden_gs128_and_smooth():
    g = _golden_kv("gs128_and_smooth.txt")
    f = dict(kv.split("=") for kv in g["gs128"].split())
    K = 256
    qa = torch.ones((1, K), dtype=torch.int8)
    qw = torch.cat([torch.full((1, 128), int(f["w_blk0"])), torch.full((1, 128), int(f["w_blk1"]))],
                   dim=1).to(torch.int8)
    s_blk = torch.tensor([[float(v) for v in f["s_blk"].split(",")]], dtype=torch.float32)
    y = oracle.gs128_mm(qa, torch.tensor([float(f["s_tok"])]), qw, s_blk)
    assert y.float().item() == float(f["y"])
    # smoothing factors: build X, W whose column maxima are the listed values
    xm = [float(v) for v in g["smooth_xmax"].split()]
    wm = [float(v) for v in g["smooth_wmax"].split()]
    want = [float(v) for v in g["smooth_s"].split()]
    x = bf16([xm, [-v / 2 for v in xm]])
    w = bf16([[-v for v in wm], [v / 4 for v in wm]])
    s, inv = oracle.smooth_factors(x, w)
    assert s.tolist() == want
    assert inv.tolist() == [np.float32(1.0 / np.float64(np.float32(v))).item() for v in want]


# ------------------------------------------------------------------ quant

def _brute_code(v: np.float32, mult: np.float32) -> int:
    """Nearest integer in [-127, 127] to fp32(v*mult), ties to even, by search."""
    t = float(np.float32(v) * np.float32(mult))
    best, bd = None, None
    for c in range(-127, 128):
        d = abs(t - c)
        if bd is None or d < bd or (d == bd and c % 2 == 0):
            best, bd = c, d
    return best


def test_quant_brute_force_tiny():
    rng = np.random.default_rng(3)
    for trial in range(40):
        K = int(rng.integers(1, 9))
        x = bf16((rng.standard_normal((2, K)) * 10 ** rng.uniform(-2, 2)).tolist())
        inv = torch.tensor(rng.uniform(0.1, 3.0, K).astype(np.float32))
        q, s = oracle.quant_per_token(x, inv)
        xf = x.float().numpy() * inv.numpy()[None, :]        # fp32 products
        for m in range(2):
            amax = np.float32(np.abs(xf[m]).max())
            assert s[m].item() == np.float32(amax / np.float32(127)).item()
            mult = np.float32(np.float32(127) / amax)
            assert q[m].tolist() == [_brute_code(v, mult) for v in xf[m]]


def test_quant_closed_forms():
    # integer rows with amax = 127: scale 1 and the codes equal the values
    rng = np.random.default_rng(4)
    ints = rng.integers(-127, 128, (8, 64))
    ints[:, 5] = 127
    x = bf16(ints.astype(np.float32).tolist())
    q, s = oracle.quant_per_token(x)
    assert torch.equal(q.to(torch.int64), torch.tensor(ints))
    assert torch.all(s == 1.0)
    # odd symmetry q(-x) = -q(x), same scale
    xr = bf16(rng.standard_normal((4, 300)).tolist())
    q1, s1 = oracle.quant_per_token(xr)
    q2, s2 = oracle.quant_per_token(-xr)
    assert torch.equal(q1, -q2) and torch.equal(s1, s2)
    # reconstruction error at most half a step, plus the fp32 roundings of
    # the multiplier 127/amax and of the products (127 * 2^-22 steps at most)
    xf = xr.float()
    err = (xf - q1.float() * s1[:, None]).abs()
    assert torch.all(err <= s1[:, None] * (0.5 + 2.0 ** -14))
    assert int(q1.abs().max()) == 127 and int(q1.min()) >= -127


def test_quant_weight_per_channel_and_gs128():
    w = inputs.gen_w(32, 512, seed=7)
    q, sc = oracle.quant_weight(w)
    wf = w.float()
    amax = wf.abs().amax(dim=1)
    assert torch.equal(sc, amax / 127.0)
    assert torch.all((q.float() * sc[:, None] - wf).abs() <= sc[:, None] * (0.5 + 2.0 ** -14))
    q2, sb = oracle.quant_weight(w, group=128)
    assert sb.shape == (32, 4)
    for b in range(4):
        blk = wf[:, b * 128:(b + 1) * 128]
        assert torch.equal(sb[:, b], blk.abs().amax(dim=1) / 127.0)
        qq, _ = oracle.quant_per_token(w[:, b * 128:(b + 1) * 128].contiguous())
        assert torch.equal(q2[:, b * 128:(b + 1) * 128], qq)
    # a constant row: every group scale equals the channel scale
    wc = bf16([[0.5] * 256, [-0.25] * 256])
    _, sc_c = oracle.quant_weight(wc)
    _, sb_c = oracle.quant_weight(wc, group=128)
    assert torch.equal(sb_c, sc_c[:, None].expand(2, 2).contiguous())


# ------------------------------------------------------------- smoothing fold

def test_fold_is_function_preserving_fp64():
    M, K, N = 16, 256, 128
    x = inputs.gen_x(M, K, 11, inputs.XRecipe(col_count=4, col_factor=20.0))
    w = inputs.gen_w(N, K, 11)
    s, inv = oracle.smooth_factors(x, w)
    assert torch.all(s <= 16.0) and torch.all(s > 0)
    xs = (x.double() * inv.double()[None, :]).float().double()      # X diag(s)^-1, f32
    ws = oracle.fold_weight(w, s).double()                           # diag(s) W, f32
    ref = x.double() @ w.double().T
    got = xs @ ws.T
    rel = (got - ref).norm() / ref.norm()
    assert rel < 1e-5
    # the ratio to the original weights is one per-column factor for every row
    nz = w.float() != 0
    ratio = ws / w.double()                  # exact quotient up to fp64 rounding
    col = s.double()
    dev = ((ratio - col[None, :]).abs() / col[None, :])[nz]
    assert float(dev.max()) <= 2.0 ** -24
    # after INT8 quantisation: q*s_ch/W ~ s_k times a per-row factor 1, within
    # the quantisation step 0.5*s_ch/|W| (plus fp32 slack)
    q, sc = oracle.quant_weight(w, s)
    big = w.float().abs() > 0.01
    deq = q.float() * sc[:, None]
    r = deq / w.float() / s[None, :]
    bound = 0.5 * sc[:, None] / (w.float().abs() * s[None, :]) + 1e-5
    assert torch.all(((r - 1).abs() <= bound)[big])


def test_smooth_factors_cap_and_degenerate():
    x = bf16([[1.0, 0.0, 0.0, 400.0]])
    w = bf16([[1.0, 0.0, 2.0, 0.01]])
    s, inv = oracle.smooth_factors(x, w)
    # col0: 1/1 = 1; col1: both zero -> 1; col2: 0 -> floor 1e-5; col3: capped
    assert s[0] == 1.0 and s[1] == 1.0 and s[3] == 16.0
    assert s[2].item() == np.float32(1e-5).item()
    assert inv[3] == 1.0 / 16.0


# ------------------------------------------------------------------- GEMMs

@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (16, 128, 256), (2, 17, 1000)])
def test_mm_i32_vs_numpy(M, N, K):
    rng = np.random.default_rng(M * 1000 + N + K)
    qa = rng.integers(-127, 128, (M, K)).astype(np.int8)
    qw = rng.integers(-127, 128, (N, K)).astype(np.int8)
    want = qa.astype(np.int64) @ qw.astype(np.int64).T
    got = oracle.mm_i32(torch.from_numpy(qa), torch.from_numpy(qw))
    assert np.array_equal(got.numpy().astype(np.int64), want)
    rows = [M - 1, 0]
    assert np.array_equal(oracle.mm_i32(torch.from_numpy(qa), torch.from_numpy(qw), rows).numpy(),
                          want[rows])


def test_mm_i32_extremes_no_overflow():
    K = 17408
    qa = torch.full((2, K), 127, dtype=torch.int8)
    qa[1] = -127
    qw = torch.full((1, K), 127, dtype=torch.int8)
    acc = oracle.mm_i32(qa, qw)
    assert acc[:, 0].tolist() == [K * 127 * 127, -K * 127 * 127]


def test_epilogue_vs_torch_ops_and_unit_scales():
    rng = np.random.default_rng(5)
    acc = torch.from_numpy(rng.integers(-2 ** 27, 2 ** 27, (7, 9)).astype(np.int32))
    s_tok = torch.from_numpy(rng.uniform(0.001, 2, 7).astype(np.float32))
    s_ch = torch.from_numpy(rng.uniform(0.0001, 0.01, 9).astype(np.float32))
    want = ((acc.float() * s_tok[:, None]) * s_ch[None, :]).to(torch.bfloat16)
    assert torch.equal(oracle.epilogue_ch(acc, s_tok, s_ch), want)
    small = torch.from_numpy(rng.integers(-256, 257, (5, 6)).astype(np.int32))
    y = oracle.epilogue_ch(small, torch.ones(5), torch.ones(6))
    assert torch.equal(y.float(), small.float())


def test_w8a8_scaled_mm_composes():
    rng = np.random.default_rng(6)
    qa = torch.from_numpy(rng.integers(-127, 128, (9, 384)).astype(np.int8))
    qw = torch.from_numpy(rng.integers(-127, 128, (40, 384)).astype(np.int8))
    s_tok = torch.from_numpy(rng.uniform(0.01, 1, 9).astype(np.float32))
    s_ch = torch.from_numpy(rng.uniform(1e-4, 1e-3, 40).astype(np.float32))
    y = oracle.w8a8_scaled_mm(qa, s_tok, qw, s_ch)
    assert torch.equal(y, oracle.epilogue_ch(oracle.mm_i32(qa, qw), s_tok, s_ch))
    # the transposed operand order gives a different answer (guards the index order)
    yt = oracle.w8a8_scaled_mm(qw[:9].contiguous(), s_tok, qa, s_ch[:9].contiguous())
    assert not torch.equal(y[:, :9], yt[:, :9])


def test_gs128_reduces_to_per_channel_and_fp64():
    rng = np.random.default_rng(7)
    M, N, K = 6, 24, 512
    qa = torch.from_numpy(rng.integers(-127, 128, (M, K)).astype(np.int8))
    qw = torch.from_numpy(rng.integers(-127, 128, (N, K)).astype(np.int8))
    s_tok = torch.from_numpy(rng.uniform(0.01, 1, M).astype(np.float32))
    s_ch = torch.from_numpy(rng.uniform(1e-4, 1e-3, N).astype(np.float32))
    y_gs = oracle.gs128_mm(qa, s_tok, qw, s_ch[:, None].expand(N, K // 128).contiguous())
    y_ch = oracle.w8a8_scaled_mm(qa, s_tok, qw, s_ch)
    ulp = _bf16_ulp(y_ch.float())
    assert torch.all((y_gs.float() - y_ch.float()).abs() <= ulp)
    s_blk = torch.from_numpy(rng.uniform(1e-4, 1e-3, (N, K // 128)).astype(np.float32))
    y = oracle.gs128_mm(qa, s_tok, qw, s_blk)
    a = qa.numpy().astype(np.float64).reshape(M, K // 128, 128)
    b = qw.numpy().astype(np.float64).reshape(N, K // 128, 128)
    parts = np.einsum("mbk,nbk->mnb", a, b)
    exact = (parts * s_blk.numpy().astype(np.float64)[None]).sum(-1) * s_tok.numpy()[:, None]
    assert np.all(np.abs(y.float().numpy() - exact) <= _bf16_ulp(torch.from_numpy(exact)).numpy())


def _bf16_ulp(y: torch.Tensor) -> torch.Tensor:
    a = y.double().abs().clamp_min(2.0 ** -126)
    return torch.exp2(torch.floor(torch.log2(a)) - 7)


def test_w8a16_vs_fp64_matmul():
    rng = np.random.default_rng(8)
    M, N, K = 3, 20, 1000
    x = bf16(rng.standard_normal((M, K)).tolist())
    qw = torch.from_numpy(rng.integers(-127, 128, (N, K)).astype(np.int8))
    s_ch = torch.from_numpy(rng.uniform(1e-4, 1e-3, N).astype(np.float32))
    y, mag = oracle.w8a16_mm(x, qw, s_ch, with_bound=True)
    exact = (x.double().numpy() @ qw.numpy().astype(np.float64).T) * s_ch.numpy()[None, :]
    ref = torch.tensor([[bits_to_f32(oracle.f64_to_bf16_bits(float(v))) for v in r] for r in exact])
    assert torch.equal(y.float(), ref)
    assert np.allclose(mag.numpy(), np.abs(x.double().numpy())
                       @ np.abs(qw.numpy().astype(np.float64)).T * s_ch.numpy()[None, :])
    # M = 1, unit scales: a plain dot product of small integers is exact
    xi = bf16([[1.0, 2.0, -3.0, 4.0]])
    qi = torch.tensor([[1, 1, 1, 1], [2, 0, 1, -1]], dtype=torch.int8)
    assert oracle.w8a16_mm(xi, qi, torch.ones(2)).float()[0].tolist() == [4.0, -5.0]


def test_oracle_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.quant_weight(torch.zeros((2, 100), dtype=torch.bfloat16), group=128)
    with pytest.raises(ValueError):
        oracle.mm_i32(torch.zeros((2, 4), dtype=torch.int8), torch.zeros((3, 4), dtype=torch.int8),
                      rows=[5])


# -------------------------------------------------------- seeded generator

def test_generator_is_deterministic_and_shaped():
    w0 = inputs.workload(0)
    x1, x2 = w0.make_x(), w0.make_x()
    assert torch.equal(x1.view(torch.int16), x2.view(torch.int16))
    assert x1.shape == (16, 256) and x1.dtype == torch.bfloat16
    z = inputs.normals_f64(123, 1, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    cols = inputs.pick_columns(w0.seed, 256, 4)
    assert len(set(cols.tolist())) == 4
    big = x1.float().abs().amax(dim=0)
    assert set(torch.topk(big, 4).indices.tolist()) == set(cols.tolist())
    # chunking does not change the values
    xa = inputs.gen_x(37, 64, 5, inputs.XRecipe(row_period=8, row_width=2, row_factor=50.0))
    xb = inputs.gen_x(37, 64, 5, inputs.XRecipe(row_period=8, row_width=2, row_factor=50.0),
                      chunk_rows=5)
    assert torch.equal(xa.view(torch.int16), xb.view(torch.int16))


def test_generator_is_splitmix64():
    """The input generator's per-stream sequence is SplitMix64 started at the
    stream key: its finaliser stepped by the golden-ratio increment
    reproduces the published reference outputs for state 1234567."""
    published = [6457827717110365317, 3203168211198807973, 9817491932198370423,
                 4593380528125082431, 16408922859458223821]
    idx = np.arange(1, 6, dtype=np.uint64)
    with np.errstate(over="ignore"):
        got = inputs.mix64(np.uint64(1234567) + idx * inputs.GAMMA)
    assert [int(v) for v in got] == published
    # uniform_bits(seed, stream, ...) is the same sequence from stream_key
    key = inputs.stream_key(7, 3)
    with np.errstate(over="ignore"):
        ref = inputs.mix64(key + np.arange(11, 21, dtype=np.uint64) * inputs.GAMMA)
    assert np.array_equal(inputs.uniform_bits(7, 3, 10, 10), ref)
