"""Test helpers: host<->device marshalling and the parity tolerance.

Tolerance for floating-point outputs (from the parity contract of the layer):
relative Frobenius error <= 2e-3 and max-abs error <= 2e-2 * rms(reference).
"""
import numpy as np
import torch

REL_FRO = 2e-3
MAX_ABS_RMS = 2e-2
# End-to-end comparisons (oracle run from the raw inputs alone) of outputs that
# lie downstream of an FP8 re-quantisation of a float intermediate (h, d[g|u]):
# the two sides compute that intermediate in different precision (fp32 vs fp64
# accumulation), so an element can land on the neighbouring e4m3 code (a
# relative step of up to 2^-3 of that element).  The relative Frobenius bound
# stays; the max-abs bound is 5e-2 * rms there.  Per-step comparisons, on
# identical inputs, use the contract bounds above.
MAX_ABS_RMS_E2E = 5e-2


def dev(a, dtype=None):
    """numpy -> cuda tensor (uint16 arrays become bf16 tensors)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    t = torch.from_numpy(a).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    """cuda tensor -> numpy (bf16 -> uint16 bit patterns)."""
    t = t.detach().contiguous()
    if t.dtype == torch.bfloat16:
        return t.cpu().view(torch.int16).numpy().view(np.uint16)
    return t.cpu().numpy()


def bf(a):
    """bf16 bit patterns -> float64."""
    return (np.asarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp(v):
    """Spacing of the bf16 grid at |v| (2^(e-7) for v in [2^e, 2^(e+1)))."""
    a = np.abs(np.asarray(v, np.float64)).astype(np.float32)
    return np.spacing(a).astype(np.float64) * 2.0 ** 16


# Share of the elements that the one-bf16-unit allowance below may forgive:
# outside it, a drift of rounding flips (not only the odd neighbour) fails.
MAX_FORGIVEN_SHARE = 1e-3


def close(got, ref, rel_fro=REL_FRO, max_abs_rms=MAX_ABS_RMS, what="", bf16=False):
    """Relative Frobenius and max-abs bounds.  For bf16 outputs (bf16=True) an
    element one bf16 unit away from the reference passes the max-abs test:
    both sides round a value computed in different precision (fp32 vs fp64)
    to bf16, so they can land on neighbouring bf16 numbers; that step (2^-8
    relative) exceeds 2e-2 * rms for elements above about 5 rms.  Such
    forgiven elements are counted, and their share must stay at most
    MAX_FORGIVEN_SHARE (at least 2 elements are always allowed).  Returns
    (relative Frobenius error, max-abs error, forgiven count)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    nref = np.linalg.norm(ref)
    err = np.linalg.norm(got - ref)
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    rel = err / nref if nref > 0 else err
    diff = np.abs(got - ref)
    bound = max_abs_rms * rms + 1e-30
    forgiven = 0
    if bf16 and ref.size:
        within_ulp = diff <= bf16_ulp(ref) * (1 + 1e-9)
        forgiven = int(np.count_nonzero(within_ulp & (diff > bound)))
        diff = np.where(within_ulp, 0.0, diff)
    mx = np.max(diff) if ref.size else 0.0
    assert rel <= rel_fro, f"{what}: relative Frobenius error {rel:.3e} > {rel_fro}"
    assert mx <= bound, f"{what}: max-abs error {mx:.3e} > {max_abs_rms} * rms {rms:.3e}"
    assert forgiven <= max(2, MAX_FORGIVEN_SHARE * ref.size), \
        f"{what}: {forgiven} of {ref.size} elements passed only by the one-bf16-unit allowance"
    return rel, mx, forgiven


def same_bits(got, ref, what=""):
    got = np.ascontiguousarray(got)
    ref = np.ascontiguousarray(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if got.dtype == np.float32:
        got, ref = got.view(np.int32), ref.view(np.int32)
    bad = np.nonzero(got != ref)
    assert len(bad[0]) == 0, f"{what}: {len(bad[0])} mismatches, first at {tuple(b[0] for b in bad)}: " \
                             f"{got[tuple(b[0] for b in bad)]} vs {ref[tuple(b[0] for b in bad)]}"


def rand_bf16(rng, shape, std=1.0):
    from moe_expert_layer_replay_b200.inputs import to_bf16_bits
    return to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))
