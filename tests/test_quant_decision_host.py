"""The quantisers' divide-free e4m3 codes (the arithmetic of e4m3_codes() in
the CUDA kernels, restated step by step here in fp32 with an exact fp32 FMA)
equal the IEEE definition code = e4m3(RN(x / s)) that the oracle encodes, on
the whole domain the kernels feed them: bf16 values x with |x| <= amax, amax a
bf16 value, s = RN(amax / 448).  No GPU: this pins the method; the GPU tests
pin the kernels.

Method (Markstein's correction of a quotient by a correctly rounded
reciprocal; P. Markstein, "Computation of elementary functions on the IBM
RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990), with -r in
place of r as the kernels run it:
    r = RN(1/s);  a = RN(x * -r);  e = RN(a * s + x)  (one FMA);
    q' = RN(e * -r + a)  (one FMA);  code = e4m3(q') with its sign bit flipped.
Scales below 2^-90 take IEEE division (not restated here).

The checks are exhaustive: every non-negative finite bf16 x up to amax and its
negative, against every one of the 128 bf16 amax mantissas, at amax exponents
that cover the scale-invariant middle of the range and both of its ends (the
smallest scale on this path, just above 2^-90, and the largest finite bf16
amax).  Between the ends every step scales exactly by powers of two."""
import numpy as np
import pytest

f32 = np.float32


def _flt(u):
    return np.asarray(u, np.uint32).view(f32)


def _rn32_of_sum(hi, lo):
    """fp32 rounding (to nearest even) of the exact value hi + lo, where hi =
    RN64(hi + lo) and lo is its exact error (a TwoSum pair)."""
    f = hi.astype(f32)
    fd = f.astype(np.float64)
    other = np.where(fd < hi, np.nextafter(f, f32(np.inf)), np.nextafter(f, f32(-np.inf)))
    tie = (hi == (fd + other.astype(np.float64)) / 2) & (fd != hi)
    lo_f, hi_f = np.minimum(f, other), np.maximum(f, other)
    out = np.where(tie & (lo > 0), hi_f, f)
    return np.where(tie & (lo < 0), lo_f, out).astype(f32)


def fma32(a, b, c):
    """fp32 fma(a, b, c) = RN32(a*b + c) exactly: a*b is exact in fp64 (48
    significant bits), the sum is split by TwoSum, then rounded once."""
    a, b, c = (np.asarray(t, f32).astype(np.float64) for t in (a, b, c))
    p = a * b
    s = p + c
    bb = s - p
    lo = (p - (s - bb)) + (c - bb)
    return _rn32_of_sum(s, lo)


def kernel_codes(orc, x, s, correct=True, fused=True):
    x = np.asarray(x, f32)
    r = f32(1) / f32(s)                                  # RN(1/s)
    nr = -r
    a = (x * nr).astype(f32)                             # RN(x * -r) = -q0
    q = a
    if correct and fused:
        e = fma32(a, f32(s), x)                          # x - q0 s
        q = fma32(e, nr, a)                              # -(q0 + e r)
    elif correct:                                        # each product rounded before its sum
        e = ((a * f32(s)).astype(f32) + x).astype(f32)
        q = ((e * nr).astype(f32) + a).astype(f32)
    return orc.e4m3_encode(q) ^ np.uint8(0x80)           # flip the sign bits


def _domain_cases(exponents):
    xs = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(f32)    # every finite x >= 0 in bf16
    for e in exponents:
        for m in range(128):
            amax = _flt(np.uint32(((e << 7) | m) << 16))
            s = f32(amax / f32(448))
            x = xs[xs <= amax]
            yield np.concatenate([x, -x]), s


def _mismatches(orc, exponents, **kw):
    bad = tested = 0
    for x, s in _domain_cases(exponents):
        assert 2.0 ** -90 <= s < np.inf
        exact = orc.e4m3_encode((x / s).astype(f32))      # IEEE RN(x / s), then e4m3
        bad += int(np.count_nonzero(kernel_codes(orc, x, s, **kw) != exact))
        tested += x.size
    return bad, tested


# 0x2E: amax in [2^-81, 2^-80), the smallest scales on this path (s just above
# 2^-90); 0x40, 0x7F: the middle; 0xFE: amax up to the largest finite bf16
@pytest.mark.parametrize("exponents", [[0x2E], [0x40, 0x7F], [0xFE]])
def test_every_bf16_value_against_every_amax_mantissa(orc, exponents):
    bad, tested = _mismatches(orc, exponents)
    assert tested > 1_000_000 and bad == 0


def test_signed_zeros(orc):
    for s in (f32(1.0), f32(3.0e-20), f32(7.0e30)):
        codes = kernel_codes(orc, np.array([0.0, -0.0], f32), s)
        assert list(codes) == [0x00, 0x80]


@pytest.mark.parametrize("variant", [dict(correct=False), dict(fused=False)])
def test_broken_variants_are_caught(orc, variant):
    """Dropping the correction step (codes of RN(x * r) alone), or computing it
    with a rounded product before each sum instead of FMAs, must fail the same
    check."""
    bad, _ = _mismatches(orc, [0x40], **variant)
    assert bad > 0
