"""The quantisers' divide-free exact decision (the arithmetic of quotients()
in the CUDA kernels, restated here step by step in numpy fp32) gives the same
e4m3 code as the IEEE definition code = e4m3(RN(x / s)) that the oracle
encodes.  No GPU: this pins the method; the GPU tests pin the kernels.

Method: q' = RN(x * RN(1/s)); M = the e4m3 rounding midpoint of q''s bracket
(below 2^-6 found in [2^-6, 2^-5) after adding 2^-6 with rounding toward
zero); e = RN(|x| - M*s) (one fp32 FMA); the code is that of M, or of its fp32
neighbour on the side e > c or e < -c, c = s * ulp(M)/2."""
import numpy as np
import pytest

f32 = np.float32


def _bits(a):
    return np.asarray(a, f32).view(np.uint32)


def _flt(u):
    return np.asarray(u, np.uint32).view(f32)


def kernel_quotients(x, s, cmp_zero=False, rn_map=False):
    x = np.asarray(x, f32)
    r = f32(1) / f32(s)                                   # RN(1/s)
    qp = (x * r).astype(f32)                              # RN(x * r)
    b = _bits(qp) & np.uint32(0x7FFFFFFF)
    sub = b < 0x3C800000
    s64 = _flt(b).astype(np.float64) + 2.0 ** -6          # exact in fp64
    y32 = s64.astype(f32)
    if not rn_map:                                        # round toward zero
        y32 = np.where(np.abs(y32.astype(np.float64)) > s64, np.nextafter(y32, f32(0)), y32).astype(f32)
    y = np.where(sub, _bits(y32), b).astype(np.uint32)
    My = _flt((y & np.uint32(0xFFF00000)) | np.uint32(0x00080000))
    M = np.where(sub, (My - f32(2.0 ** -6)).astype(f32), My).astype(f32)
    c = (f32(s) * f32(2.0 ** -24) * _flt(_bits(M) & np.uint32(0x7F800000))).astype(f32)
    # one fp32 FMA: the exact |x| - M*s (fp64 holds it near M), rounded once to fp32
    e = (np.abs(x).astype(np.float64) - M.astype(np.float64) * np.float64(s)).astype(f32)
    if cmp_zero:
        c = np.zeros_like(c)
    mb = _bits(M).astype(np.int64) + (e > c) - (e < -c)
    return _flt(mb.astype(np.uint32) | (_bits(qp) & np.uint32(0x80000000)))


def _mismatches(orc, x, s, **kw):
    x = np.asarray(x, f32)
    exact = (x / f32(s)).astype(f32)                      # IEEE RN(x / s)
    return int(np.count_nonzero(orc.e4m3_encode(kernel_quotients(x, s, **kw)) != orc.e4m3_encode(exact)))


def _grid_and_midpoints():
    vals = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        vals.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))
    v = np.array(sorted(set(vals)))
    return np.concatenate([v, (v[1:] + v[:-1]) / 2])


def test_random_values_and_scales(orc):
    rng = np.random.default_rng(21)
    bad = 0
    for trial in range(60):
        n = 1 << 15
        kind = trial % 3
        if kind == 0:
            x = rng.standard_normal(n) * rng.standard_normal(n)
        elif kind == 1:
            x = rng.standard_t(2, n) * 10.0 ** rng.uniform(-20, 20)
        else:
            x = rng.uniform(-1, 1, n) * 2.0 ** rng.integers(-60, 60)
        x = x.astype(f32)
        if trial % 2 == 0:
            x = _flt(_bits(x) & np.uint32(0xFFFF0000))        # bf16-exact values
        s = f32(np.abs(x).max() / f32(448))
        if trial % 4 == 1:                                   # short-mantissa scale: exact midpoints abound
            s = _flt(np.array([_bits(np.array([s], f32))[0] & 0xFFC00000], np.uint32))[0]
        if not (2.0 ** -90 <= s < np.inf):
            continue
        bad += _mismatches(orc, x, s)
    assert bad == 0


def test_grid_points_midpoints_neighbours_and_zeros(orc):
    rng = np.random.default_rng(22)
    base = _grid_and_midpoints()
    bad = tested = 0
    for _ in range(300):
        s = f32(rng.uniform(0.5, 2.0) * 2.0 ** rng.integers(-88, 60))
        x = (np.concatenate([base, -base]) * np.float64(s)).astype(f32)
        x = np.concatenate([x, np.nextafter(x, f32(np.inf)), np.nextafter(x, f32(-np.inf)), np.array([0.0, -0.0], f32)])
        x = x[np.abs(x) <= f32(448) * s]
        bad += _mismatches(orc, x, s)
        tested += x.size
    assert tested > 400_000 and bad == 0


@pytest.mark.parametrize("variant", [dict(cmp_zero=True), dict(rn_map=True)])
def test_broken_variants_are_caught(orc, variant):
    """Comparing against 0 instead of +-c, or mapping the subnormal brackets with
    round-to-nearest, must fail the same checks."""
    rng = np.random.default_rng(23)
    base = _grid_and_midpoints()
    bad = 0
    for _ in range(60):
        s = f32(rng.uniform(0.5, 2.0) * 2.0 ** rng.integers(-60, 40))
        x = (np.concatenate([base, -base]) * np.float64(s)).astype(f32)
        x = np.concatenate([x, np.nextafter(x, f32(np.inf)), np.nextafter(x, f32(-np.inf))])
        x = x[np.abs(x) <= f32(448) * s]
        bad += _mismatches(orc, x, s, **variant)
    assert bad > 0
