"""Pins of the oracle's NVFP4 rule ("RL at 1T scale: prime-rl performance deep
dive", §Future work: NVFP4 on Blackwell; the format is NVIDIA's NVFP4: e2m1
elements in 16-element blocks with e4m3 block scales and an fp32 tensor
scale).  No GPU."""
import json
import os

import ml_dtypes
import numpy as np
import pytest

from moe_expert_layer_replay_b200.inputs import to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e2m1_encode_matches_ml_dtypes(orc):
    from oracle import nvfp4
    rng = np.random.default_rng(90)
    mags = np.array(nvfp4.E2M1_MAGNITUDES)
    mids = (mags[1:] + mags[:-1]) / 2
    grid = np.concatenate([mags, mids, np.nextafter(mids.astype(np.float32), 0), np.nextafter(mids.astype(np.float32), 10),
                           [6.5, 7, 1e6, 1e-30, 0.0], rng.uniform(0, 8, 5000)]).astype(np.float32)
    v = np.concatenate([grid, -grid])
    got = nvfp4.e2m1_encode(v)
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    assert np.array_equal(got, ref)
    assert np.array_equal(nvfp4.e2m1_decode(np.arange(16, dtype=np.uint8)),
                          np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64))


def test_scale_rule_and_codes(orc):
    from oracle import nvfp4
    rng = np.random.default_rng(91)
    rows, cols = 40, 256
    x = to_bf16_bits((rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-6, 6, (rows, 1)))).astype(np.float32))
    x[3, 16:32] = 0                                           # an all-zero block
    codes, S8, s_g = nvfp4.quant(x)
    xf = orc.bf16_to_f64(x).astype(np.float32)
    amax_t = np.abs(xf).max()
    assert s_g == np.float32(np.float32(2688.0) / amax_t)      # IEEE fp32 division
    blk = xf.reshape(rows, cols // 16, 16)
    s_b = np.abs(blk).max(-1) / np.float32(6.0)
    ref_S8 = (s_b * s_g).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(S8, ref_S8)
    S_b = S8.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(S_b > 0, np.float32(s_g) / S_b, 0).astype(np.float32)
    ref = ((blk * inv[..., None]).astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15)
    ref = np.where((S_b > 0)[..., None], ref, 0).reshape(rows, cols)
    assert np.array_equal(codes, ref)
    assert np.all(codes[3, 16:32] == 0) and S8[3, 1] == 0
    # the amax element of a block lands near the top of the e2m1 range
    top = np.abs(nvfp4.e2m1_decode(codes)).reshape(rows, cols // 16, 16).max(-1)
    assert np.all(top[S8 > 0] >= 4.0)


def test_round_trip_bound(orc):
    """Each value is the nearest e2m1 multiple of its block's step S_b / s_g
    (up to saturation at 6 steps of the block's largest magnitude)."""
    from oracle import nvfp4
    rng = np.random.default_rng(92)
    x = to_bf16_bits(rng.standard_normal((64, 512)).astype(np.float32))
    codes, S8, s_g = nvfp4.quant(x)
    xd = nvfp4.dequant(codes, S8, s_g)
    xf = orc.bf16_to_f64(x)
    step = (S8.view(ml_dtypes.float8_e4m3fn).astype(np.float64) / np.float64(s_g)).repeat(16, axis=1)
    err = np.abs(xd - xf)
    mag = np.abs(xf) / step
    half_gap = np.where(mag < 2, 0.25, np.where(mag < 4, 0.5, 1.0))   # half the e2m1 spacing
    assert np.all(err <= half_gap * step * (1 + 1e-6) + np.maximum(mag - 6, 0) * step)


def test_pack_unpack_and_gemm(orc):
    from oracle import nvfp4
    rng = np.random.default_rng(93)
    A = to_bf16_bits(rng.standard_normal((24, 320)).astype(np.float32))
    B = to_bf16_bits((rng.standard_normal((40, 320)) * 0.02).astype(np.float32))
    qa, sa, ga = nvfp4.quant(A)
    qb, sb, gb = nvfp4.quant(B)
    assert np.array_equal(nvfp4.unpack(nvfp4.pack(qa)), qa)
    assert nvfp4.pack(qa)[0, 0] == (qa[0, 0] | (qa[0, 1] << 4))
    C = nvfp4.gemm(qa, sa, ga, qb, sb, gb)
    ref = nvfp4.dequant(qa, sa, ga) @ nvfp4.dequant(qb, sb, gb).T
    np.testing.assert_allclose(C, ref, rtol=1e-12, atol=1e-12)
    # NVFP4 stays within its error of the exact product
    exact = orc.bf16_to_f64(A) @ orc.bf16_to_f64(B).T
    assert np.linalg.norm(C - exact) / np.linalg.norm(exact) < 0.15


def test_golden_block(orc):
    from oracle import nvfp4
    g = json.load(open(os.path.join(GOLDEN, "nvfp4_block.json")))
    x = to_bf16_bits(np.array([g["x"]], np.float32))
    codes, S8, s_g = nvfp4.quant(x)
    assert float(s_g) == g["s_g"]
    assert S8.tolist() == [g["S8"]]
    assert codes[0].tolist() == g["codes"]
