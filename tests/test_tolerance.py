"""The parity tolerance helper itself (no GPU): the contract bounds, the
one-bf16-unit allowance for bf16 outputs, and the cap on how many elements
that allowance may forgive."""
import numpy as np
import pytest

from _util import MAX_FORGIVEN_SHARE, bf16_ulp, close


def _ref(n=20000, seed=70):
    rng = np.random.default_rng(seed)
    r = rng.standard_normal(n)
    r[:60] = np.sign(r[:60]) * rng.uniform(5.0, 7.5, 60)   # a tail whose bf16 unit exceeds 2e-2 * rms
    return (r.astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32).astype(np.float64)


def test_close_accepts_identical_and_small_errors():
    ref = _ref()
    assert close(ref, ref, bf16=True)[2] == 0
    close(ref * (1 + 1e-4), ref)


def test_close_rejects_bias_and_outliers():
    ref = _ref()
    with pytest.raises(AssertionError, match="Frobenius"):
        close(ref * 1.01, ref)
    bad = ref.copy()
    bad[7] += 0.2
    with pytest.raises(AssertionError, match="max-abs"):
        close(bad, ref)


def test_one_ulp_flips_are_counted_and_capped():
    ref = _ref()
    big = np.nonzero(bf16_ulp(ref) > 2e-2 * np.sqrt(np.mean(ref ** 2)))[0]   # the planted tail
    assert len(big) >= 50
    got = ref.copy()
    got[big[:2]] += bf16_ulp(ref[big[:2]])
    assert close(got, ref, bf16=True)[2] == 2
    n_allowed = int(MAX_FORGIVEN_SHARE * ref.size)
    got = ref.copy()
    got[big[:n_allowed + 1]] += bf16_ulp(ref[big[:n_allowed + 1]])
    with pytest.raises(AssertionError, match="allowance"):
        close(got, ref, bf16=True)
