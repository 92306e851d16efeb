"""Pins of the oracle's scalar codecs (e4m3fn, bf16) against brute force and
library casts.  No GPU."""
import ml_dtypes
import numpy as np
import pytest
import torch


def _all_e4m3_values():
    codes = np.arange(256, dtype=np.uint8)
    vals = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return codes, vals


def test_e4m3_decode_matches_ml_dtypes(orc):
    codes, vals = _all_e4m3_values()
    mine = orc.e4m3_decode(codes)
    nan = np.isnan(vals)
    assert np.array_equal(np.isnan(mine), nan)
    assert nan.sum() == 2  # 0x7F, 0xFF
    assert np.array_equal(mine[~nan], vals[~nan])
    assert orc.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0
    assert orc.e4m3_decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9


def _brute_force_e4m3(v32):
    """Nearest finite e4m3 code by exhaustive search; ties -> even mantissa;
    a zero result keeps the sign of v."""
    codes, vals = _all_e4m3_values()
    fin = ~np.isnan(vals)
    codes, vals = codes[fin], vals[fin]
    v = v32.astype(np.float64)
    # beyond the largest finite value the nearest is 448; clipping keeps the
    # distances representable
    d = np.abs(np.clip(v, -1e4, 1e4)[:, None] - vals[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    out = np.empty(v.shape, np.uint8)
    for i in range(len(v)):
        c = codes[cand[i]]
        if len(c) > 1 and not np.all(vals[cand[i]] == 0):
            c = c[(c & 1) == 0]  # a tie between two values: even mantissa
        if len(c) > 1:  # +0 / -0: keep the sign of v
            c = c[(c & 0x80) == (0x80 if np.signbit(v[i]) else 0)]
        assert len(c) == 1
        out[i] = c[0]
    return out


def _interesting_fp32(rng, n=20000):
    _, vals = _all_e4m3_values()
    fin = vals[~np.isnan(vals)]
    pos = np.unique(np.abs(fin))
    mids = (pos[1:] + pos[:-1]) / 2  # exact ties
    pts = np.concatenate([pos, mids, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20),
                          [448.0, 449.0, 463.99, 464.0, 464.01, 480.0, 1e6, 3.4e38,
                           2.0 ** -10, 2.0 ** -11, 2.0 ** -12, 3 * 2.0 ** -11, 1e-30, 0.0]])
    r = np.exp(rng.uniform(np.log(1e-5), np.log(600.0), n))
    allv = np.concatenate([pts, r])
    allv = np.concatenate([allv, -allv]).astype(np.float32)
    return allv


def test_e4m3_encode_brute_force(orc):
    rng = np.random.default_rng(1)
    v = _interesting_fp32(rng, 4000)
    assert np.array_equal(orc.e4m3_encode(v), _brute_force_e4m3(v))


def test_e4m3_encode_matches_ml_dtypes_in_range(orc):
    rng = np.random.default_rng(2)
    v = _interesting_fp32(rng, 50000)
    v = v[np.abs(v) <= 448.0]
    ref = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(orc.e4m3_encode(v), ref)


def test_e4m3_saturation_and_zero_sign(orc):
    v = np.array([448.0, 500.0, 1e30, np.inf, -1e30, -np.inf, 0.0, -0.0, -1e-9, 1e-9],
                 np.float32)
    assert list(orc.e4m3_encode(v)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x00, 0x80, 0x80, 0x00]


def test_e4m3_exhaustive_bf16_quotients(orc):
    """Every bf16 value x, divided in fp32 by several scales, encodes to the
    brute-force nearest e4m3 code (the full domain of the quantiser's
    element step)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = orc.bf16_to_f64(bits).astype(np.float32)
    x = x[np.isfinite(x)]
    _, vals = _all_e4m3_values()
    fin = np.sort(np.unique(vals[~np.isnan(vals)]))
    for s in [1.0, 2.0 ** -30, 3.7, 0.0123, 1e-38]:
        q = (x / np.float32(s)).astype(np.float32)  # IEEE fp32 divide
        got = orc.e4m3_encode(q)
        # vectorised brute force: nearest of the sorted finite values
        a = np.abs(q.astype(np.float64))
        pos_vals = fin[fin >= 0]
        i = np.clip(np.searchsorted(pos_vals, a), 1, len(pos_vals) - 1)
        lo, hi = pos_vals[i - 1], pos_vals[i]
        pick_hi = (hi - a < a - lo)
        tie = (hi - a == a - lo)
        lo_code = np.abs(lo).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
        hi_code = np.abs(hi).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
        pick_hi |= tie & ((hi_code & 1) == 0)
        mag = np.where(pick_hi, hi_code, lo_code)
        mag = np.where(a >= pos_vals[-1], 0x7E, mag)
        ref = (mag | np.where(np.signbit(q), 0x80, 0)).astype(np.uint8)
        assert np.array_equal(got, ref), s


def test_bf16_round_matches_torch_on_fp32_values(orc):
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        (rng.standard_normal(1000) * 1e-39).astype(np.float32),
                        np.array([3.3e38, 3.4e38, -3.4e38, 0.0, -0.0], np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.bf16_round(v.astype(np.float64)), ref)


def test_bf16_round_double_brute_force(orc):
    """fp64 inputs just off the bf16 midpoints (where rounding through fp32
    first would go wrong) round to the nearest bf16, ties to even."""
    rng = np.random.default_rng(4)
    b = rng.integers(0x0080, 0x7F00, 2000).astype(np.uint16)
    lo = orc.bf16_to_f64(b)
    hi = orc.bf16_to_f64(b + 1)
    mid = (lo + hi) / 2
    for v, want in [(mid, np.where(b % 2 == 0, b, b + 1)),
                    (mid + (hi - lo) * 2.0 ** -40, b + 1),
                    (mid - (hi - lo) * 2.0 ** -40, b)]:
        assert np.array_equal(orc.bf16_round(v), want.astype(np.uint16))
        assert np.array_equal(orc.bf16_round(-v), (want | 0x8000).astype(np.uint16))
