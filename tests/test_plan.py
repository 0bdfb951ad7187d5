"""CPU checks of the host-side schedule (sq_describe_plan): which kernel,
grid, tile and split each workload gets, and the workspace it needs."""
from __future__ import annotations

import pytest

import w8a8_int8_quantized_sq_b200 as sq

B200_SMS = 148
W8A8, GS128, W8A16, I32 = sq.OP_W8A8, sq.OP_GS128, sq.OP_W8A16, sq.OP_W8A8_I32


def plan(op, M, N, K, sms=B200_SMS):
    return sq.describe_plan(op, M, N, K, sms)


def slots_bytes(grid, bn):
    # 64 KiB reserved region + two 128 x bn int32/fp32 slots per CTA
    return 65536 + grid * 2 * 128 * bn * 4


def test_prefill_uses_cta_pairs():
    p = plan(W8A8, 8192, 34816, 5120)
    assert (p["kernel"], p["tile_m"], p["tile_n"]) == (0, 256, 256)
    assert p["grid"] == B200_SMS and p["workspace_bytes"] == 0
    assert plan(I32, 33, 256, 256)["kernel"] == 0  # M > 32: no swapped schedule


def test_decode_whole_splits_in_clusters():
    # 40 weight tiles of 128 rows, 148 // 40 = 3 K parts each, 13 K blocks per part
    p = plan(W8A8, 8, 5120, 5120)
    assert (p["kernel"], p["grid"], p["tile_m"], p["tile_n"], p["splits"]) == (3, 120, 16, 128, 3)
    assert p["workspace_bytes"] == slots_bytes(120, 16)  # kept for the fallback
    # on a smaller part the same shape gets fewer splits
    assert plan(W8A8, 8, 5120, 5120, sms=100)["splits"] == 2


def test_cluster_size_limits():
    # 32 tokens: N = 32 tiles; a 128 x 32 int32 part is 16 KB, at most 5 per tile
    p = plan(W8A8, 24, 3712, 2560)
    assert (p["kernel"], p["splits"], p["tile_m"]) == (3, 5, 32)
    # one tile, 10 K blocks: 10 splits exceed a cluster, parts meet in the workspace
    p = plan(W8A8, 32, 128, 1280)
    assert (p["kernel"], p["splits"], p["grid"]) == (2, 10, 10)
    # 16 tokens, 18 tiles: 8 splits (the largest portable cluster)
    assert plan(W8A8, 8, 2304, 4096)["splits"] == 8


def test_long_k_small_m_uses_stream_k():
    # 272 K blocks per tile: whole splits would give 90 per CTA, so every SM
    # takes an equal range of the (tile, K block) space instead
    p = plan(W8A16, 16, 5120, 17408)
    assert (p["kernel"], p["grid"], p["splits"], p["tile_m"]) == (2, B200_SMS, 0, 16)
    assert p["workspace_bytes"] == slots_bytes(B200_SMS, 16)
    # group-wise scales keep the tensor-core schedule for one token as well
    p = plan(sq.OP_W8A16_GROUP, 1, 5120, 17408)
    assert (p["kernel"], p["grid"], p["splits"], p["tile_m"]) == (2, B200_SMS, 0, 16)
    assert plan(W8A8, 8, 5120, 17408)["kernel"] == 2


def test_block_scaled_pairs_and_large_m_w8a16():
    # gs128 on CTA pairs, weights as the MMA's A operand: 128 tokens x 256
    # channels per pair tile, 16 x 20 = 320 tiles over 74 pairs
    p = plan(GS128, 2048, 5120, 5120)
    assert (p["kernel"], p["tile_m"], p["tile_n"], p["grid"], p["workspace_bytes"]) == \
        (4, 128, 256, B200_SMS, 0)
    # FP8 blocks: tokens as A, 256 tokens x 128 channels (one weight block)
    p = plan(sq.OP_FP8BLK, 2048, 5120, 5120)
    assert (p["kernel"], p["tile_m"], p["tile_n"]) == (4, 256, 128)
    # enough tiles for three waves of SM pairs: 256-wide B tiles
    assert (plan(GS128, 8192, 34816, 5120)["tile_m"], plan(GS128, 8192, 34816, 5120)["tile_n"]) == (256, 256)
    assert plan(sq.OP_FP8BLK, 8192, 34816, 5120)["tile_n"] == 256
    # per-group activations x gs128 weights: one CTA per 128 x 128 tile
    p = plan(sq.OP_PG128, 2048, 5120, 5120)
    assert (p["kernel"], p["tile_m"], p["tile_n"], p["grid"]) == (1, 128, 128, B200_SMS)
    # group-wise W8A16 plans like per-channel W8A16 from two tokens on
    for M in (2, 16, 8192):
        assert plan(sq.OP_W8A16_GROUP, M, 5120, 17408) == plan(W8A16, M, 5120, 17408)
    # M > 32: the weights are converted into a bf16 copy in the workspace
    p = plan(W8A16, 8192, 5120, 17408)
    assert p["kernel"] == 0 and p["workspace_bytes"] >= 5120 * 17408 * 2


def test_swapped_grid_never_exceeds_the_sms():
    for sms in (1, 7, 132, 148):
        for M, N, K in [(1, 16, 128), (8, 5120, 5120), (16, 5120, 17408), (32, 272, 640),
                        (7, 144, 384)]:
            p = plan(W8A8, M, N, K, sms=sms)
            assert 1 <= p["grid"] <= sms
            if p["splits"]:
                assert p["grid"] == p["splits"] * ((N + 127) // 128)


def test_bad_arguments():
    with pytest.raises(sq.SqError):
        plan(W8A8, 8, 5120, 5120, sms=0)
    with pytest.raises(sq.SqError):
        plan(W8A8, 8, 5120, 200)  # K % 128
    with pytest.raises(sq.SqError):
        plan(9, 8, 5120, 5120)


def test_single_token_w8a16_runs_as_matrix_vector():
    # one token, per-channel scales: one contiguous run of rows per CTA on
    # the CUDA cores, whole K, K / 64 compute threads plus a producer warp
    p = plan(W8A16, 1, 5120, 17408)
    assert (p["kernel"], p["grid"], p["tile_m"], p["tile_n"], p["splits"]) == \
        (5, B200_SMS, 1, -(-5120 // B200_SMS), 1)
    # fewer rows than SMs: one row per CTA
    p = plan(W8A16, 1, 16, 128)
    assert (p["kernel"], p["grid"], p["tile_n"]) == (5, 16, 1)
    # the widest block (15 compute warps of 64 codes per thread + 1) still
    # fits; 16 compute warps do not
    assert plan(W8A16, 1, 144, 30720)["kernel"] == 5
    assert plan(W8A16, 1, 272, 30848)["kernel"] == 2
    # two tokens stay on the tensor cores
    assert plan(W8A16, 2, 5120, 17408)["kernel"] == 2
