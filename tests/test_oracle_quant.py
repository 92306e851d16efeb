"""Pins of the oracle's block-scaled FP8 quantiser ("RL at 1T scale: prime-rl
performance deep dive", §FP8 Training: block-scaled FP8 as in DeepSeek-V3).
No GPU."""
import json
import os

import ml_dtypes
import numpy as np
import pytest

from moe_expert_layer_replay_b200.inputs import to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_bf16(rng, shape, std=1.0):
    return to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def _blocks(rows, cols, br, bc):
    for bi in range(0, rows, br):
        for bj in range(0, cols, bc):
            yield bi // br, bj // bc, slice(bi, min(bi + br, rows)), slice(bj, min(bj + bc, cols))


@pytest.mark.parametrize("br,bc", [(1, 128), (128, 128), (128, 1)])
def test_scale_rule_and_codes(orc, br, bc):
    rng = np.random.default_rng(10)
    rows, cols = 300, 384
    x = _rand_bf16(rng, (rows, cols), 3.0)
    x[0:1, :] = 0  # an all-zero row: zero blocks for 1x128
    q, s = orc.quant_block(x, br, bc)
    xf = orc.bf16_to_f64(x).astype(np.float32)
    for bi, bj, rs, cs in _blocks(rows, cols, br, bc):
        blk = xf[rs, cs]
        amax = np.abs(blk).max()
        sc = s[bi, bj]
        # library IEEE division
        assert sc == np.float32(amax) / np.float32(448.0)
        # closed form: s * 448 within one fp32 ulp of amax
        assert abs(np.float64(sc) * 448 - amax) <= np.spacing(np.float32(amax)) or amax == 0
        if amax == 0:
            assert sc == 0 and np.all(q[rs, cs] == 0)
            continue
        codes = q[rs, cs]
        # the largest element maps to +-448
        im = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
        assert codes[im] & 0x7F == 0x7E
        # every code = ml_dtypes' nearest-even cast of fp32(x / s)
        ref = (blk / sc).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
        assert np.array_equal(codes, ref)


def test_roundtrip_bound(orc):
    rng = np.random.default_rng(11)
    x = _rand_bf16(rng, (256, 512), 1.0)
    x[:, :128] = _rand_bf16(rng, (256, 128), 1e-3)
    for br, bc in [(1, 128), (128, 128), (128, 1)]:
        q, s = orc.quant_block(x, br, bc)
        xf = orc.bf16_to_f64(x)
        deq = orc.dequant_block(q, s, br, bc)
        sf = np.repeat(np.repeat(s.astype(np.float64), br, 0)[:256], bc, 1)[:, :512]
        bound = np.maximum(2.0 ** -4 * np.abs(xf), 2.0 ** -10 * sf) * (1 + 1e-6)
        assert np.all(np.abs(xf - deq) <= bound)


def test_square_block_transpose_invariance(orc):
    rng = np.random.default_rng(12)
    W = _rand_bf16(rng, (384, 256), 0.02)
    q, s = orc.quant_block(W, 128, 128)
    qT, sT = orc.quant_block(np.ascontiguousarray(W.T), 128, 128)
    assert np.array_equal(q.T, qT) and np.array_equal(s.T, sT)


def test_rows128_is_transposed_1x128(orc):
    rng = np.random.default_rng(13)
    X = _rand_bf16(rng, (256, 384))
    q, s = orc.quant_block(X, 128, 1)
    qT, sT = orc.quant_block(np.ascontiguousarray(X.T), 1, 128)
    assert np.array_equal(q.T, qT) and np.array_equal(s.T, sT)


def test_ragged_edge_blocks(orc):
    rng = np.random.default_rng(14)
    X = _rand_bf16(rng, (200, 300))
    q, s = orc.quant_block(X, 128, 128)
    assert s.shape == (2, 3)
    qe, se = orc.quant_block(np.ascontiguousarray(X[128:, 256:]), 128, 128)
    assert se.shape == (1, 1) and se[0, 0] == s[1, 2]
    assert np.array_equal(qe, q[128:, 256:])


def test_negative_zero_keeps_sign(orc):
    x = np.zeros((1, 128), np.uint16)
    x[0, 0] = to_bf16_bits(np.array([2.0], np.float32))[0]
    x[0, 1] = 0x8000  # -0.0
    q, s = orc.quant_block(x, 1, 128)
    assert q[0, 0] == 0x7E and q[0, 1] == 0x80 and q[0, 2] == 0x00


def test_golden_block(orc):
    """Hand-worked block (derivation in the fixture)."""
    with open(os.path.join(GOLDEN, "quant_1x128_block.json")) as f:
        g = json.load(f)
    x = np.zeros((1, 128), np.float32)
    x[0, :len(g["x"])] = g["x"]
    q, s = orc.quant_block(to_bf16_bits(x), 1, 128)
    assert float(s[0, 0]) == g["scale"]
    assert [int(c) for c in q[0, :len(g["codes"])]] == g["codes"]
