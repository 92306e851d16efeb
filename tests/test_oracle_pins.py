"""Direct pins of the oracle's layer helpers that the full-size parity tests
and the CPU baseline rest on.  No GPU.

Each helper is compared with an independent construction from library
routines (numpy sorts and matmul, ml_dtypes casts, torch autograd and casts),
on inputs built so that a one-line slip (a wrong slice of the scale grid, a
repeat where a tile was meant, the wrong expert for a row, a dropped term)
changes the result by O(1):

* forward_tokens (the per-token forward used for sampled full-size parity)
  against the rows of the all-token forward, bit for bit;
* wgrad_expert against A^T B over operands dequantised independently, with
  row blocks of very different magnitude;
* scaled_rows against torch's fp32 product and bf16 cast;
* dispatch_rows and expert_of_rows against a stable argsort and the segment
  layout rebuilt from bincount;
* dequant_block, router_grads, swiglu_bwd and unpermute_reduce against
  library decodes, torch autograd and numpy sums.

The block rule these follow (1x128 activations, 128x128 weights, 128x1 along
rows for the weight gradient) is the DeepSeek-V3 block-scaled FP8 of "RL at
1T scale: prime-rl performance deep dive", §FP8 Training.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

from moe_expert_layer_replay_b200.inputs import to_bf16_bits


def _zipf_idx(rng, T, E, k, s, empty=0, bad=0):
    p = np.arange(1, E + 1, dtype=np.float64) ** -s
    if empty:
        p[E - empty:] = 0.0
    with np.errstate(divide="ignore"):
        keys = np.log(p / p.sum())[None, :] - np.log(-np.log(rng.random((T, E))))
    idx = np.argsort(-keys, axis=1, kind="stable")[:, :k].astype(np.int32)
    for i in range(bad):  # routing entries outside [0, E): dropped by the permute
        idx[rng.integers(0, T), rng.integers(0, k)] = E + i if i % 2 == 0 else -1 - i
    return idx


def _weights(rng, T, k):
    g = rng.standard_exponential((T, k))
    return (g / g.sum(1, keepdims=True)).astype(np.float32)


def _bf16(rng, shape, std=1.0):
    return to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def _deq(q, s, br, bc):
    """Independent dequantisation: ml_dtypes decode times the scale grid
    broadcast with np.repeat over whole blocks."""
    rows, cols = q.shape
    v = q.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    g = np.repeat(np.repeat(s.astype(np.float64), br, axis=0), bc, axis=1)[:rows, :cols]
    return v * g


# --------------------------------------------------------------------------
# forward_tokens == rows of forward
# --------------------------------------------------------------------------

@pytest.mark.parametrize("align", [128, 1])
@pytest.mark.parametrize("case", ["zipf_empty_bad", "uniform"])
def test_forward_tokens_equals_forward_rows(orc, align, case):
    from oracle import layer as OL
    rng = np.random.default_rng(50 + align)
    T, D, I, E, k = 160, 256, 256, 8, 3
    if case == "zipf_empty_bad":
        idx = _zipf_idx(rng, T, E, k, 1.5, empty=2, bad=3)
    else:
        idx = _zipf_idx(rng, T, E, k, 0.0)
    w = _weights(rng, T, k)
    x = _bf16(rng, (T, D))
    Wg, Wu, Wd = _bf16(rng, (E, I, D), 0.05), _bf16(rng, (E, I, D), 0.05), _bf16(rng, (E, D, I), 0.05)
    fw = OL.forward(x, idx, w, Wg, Wu, Wd, align=align)
    if case == "zipf_empty_bad":
        assert np.sum(fw["counts"] == 0) >= 2 and np.sum(fw["pos"] < 0) >= 1
    for tokens in (np.arange(T), np.sort(rng.choice(T, 23, replace=False)), np.array([T - 1, 0, 5])):
        ft = OL.forward_tokens(x, idx, w, fw["Wq"], tokens, align=align)
        rows = ft["rows"].reshape(-1)
        assert np.array_equal(ft["rows"], fw["pos"][tokens])
        ok = rows >= 0
        for name in ("h", "hq", "hs", "Y"):
            assert np.array_equal(ft[name][ok], fw[name][rows[ok]]), name
        # an entry outside [0, E) has no row: its FFN output is zero and the
        # combine skips it
        assert not np.any(ft["Y"][~ok])
        assert np.array_equal(ft["y"], fw["y"][tokens])


# --------------------------------------------------------------------------
# wgrad_expert against numpy over independently dequantised operands
# --------------------------------------------------------------------------

def test_wgrad_expert_matches_library(orc):
    from oracle import layer as OL
    rng = np.random.default_rng(60)
    rows, M, N = 640, 200, 136
    # five 128-row blocks of very different magnitude: a block offset in the
    # scale grid changes the result by O(1)
    mag = np.repeat(np.array([1.0, 37.0, 0.02, 5.0, 900.0]), 128)[:, None]
    A = to_bf16_bits((rng.standard_normal((rows, M)) * mag).astype(np.float32))
    B = to_bf16_bits((rng.standard_normal((rows, N)) * mag[::-1]).astype(np.float32))
    Aq, As = OL.quant_rows128(A)
    Bq, Bs = OL.quant_rows128(B)
    assert As.shape == (5, M) and Bs.shape == (5, N)
    Ad, Bd = _deq(Aq, As, 128, 1), _deq(Bq, Bs, 128, 1)
    for r0, r1 in [(0, 640), (128, 512), (384, 512), (256, 640)]:
        ref = Ad[r0:r1].T @ Bd[r0:r1]
        got = OL.wgrad_expert(Aq, As, Bq, Bs, r0, r1)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
        sub = OL.wgrad_expert(Aq, As, Bq, Bs, r0, r1, m0=70, M=40, n0=8, N=100)
        np.testing.assert_allclose(sub, ref[70:110, 8:108], rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # the planted magnitudes matter: shifting the scale blocks by one is far off
    wrong = _deq(Aq[128:512], As[0:3], 128, 1).T @ Bd[128:512]
    ref = Ad[128:512].T @ Bd[128:512]
    assert np.linalg.norm(wrong - ref) > 0.5 * np.linalg.norm(ref)


# --------------------------------------------------------------------------
# scaled_rows against torch
# --------------------------------------------------------------------------

def test_scaled_rows_matches_torch(orc):
    from oracle import layer as OL
    rng = np.random.default_rng(61)
    T, D, E, k = 200, 384, 6, 3
    idx = _zipf_idx(rng, T, E, k, 1.0, bad=2)
    w = _weights(rng, T, k)
    w[3, 1] = 1e-30   # products that leave bf16's normal range
    dy = _bf16(rng, (T, D), 0.01)
    # Token 0, slot 0: products whose fp32 rounding lands exactly on a bf16
    # midpoint while the exact product does not.  Rounding the fp32 product to
    # bf16 (the rule) and rounding the exact product differ there.
    dyv = orc.bf16_to_f64(np.arange(0x3f80, 0x4000, dtype=np.uint16))   # bf16 values in [1, 2)
    hits = []
    while not hits:
        w0 = np.float32(rng.uniform(0.5, 1.0))
        exact = np.float64(w0) * dyv                      # exact in fp64 (24 + 8 bits)
        p32 = (np.float32(w0) * dyv.astype(np.float32)).astype(np.float64)
        mid = (p32.view(np.uint64) & np.uint64((1 << 45) - 1)) == np.uint64(1 << 44)
        hits = [int(s) for s in np.nonzero(mid & (exact != p32))[0]]
    w[0, 0] = w0
    dy[0, :len(hits)] = np.arange(0x3f80, 0x4000, dtype=np.uint16)[hits]
    assert np.any(orc.bf16_round(np.float64(w[0, 0]) * orc.bf16_to_f64(dy[0, :len(hits)])) !=
                  orc.bf16_round((np.float32(w[0, 0]) * orc.bf16_to_f64(dy[0, :len(hits)]).astype(np.float32))
                                 .astype(np.float64)))
    counts, offsets, pos, src = orc.permute(idx, E, 128)
    R = int(offsets[E])
    got = OL.scaled_rows(dy, w, pos, R)
    dyt = torch.from_numpy(dy.view(np.int16)).view(torch.bfloat16).float()
    wt = torch.from_numpy(w)
    ref = np.zeros((R, D), np.uint16)
    for t in range(T):
        for j in range(k):
            if pos[t, j] >= 0:
                row = (wt[t, j] * dyt[t]).to(torch.bfloat16)   # fp32 product, then bf16 (RNE)
                ref[pos[t, j]] = row.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------------
# dispatch_rows / expert_of_rows against an independent segment layout
# --------------------------------------------------------------------------

@pytest.mark.parametrize("align", [128, 1])
def test_dispatch_rows_and_expert_of_rows(orc, align):
    from oracle import layer as OL
    rng = np.random.default_rng(62 + align)
    T, D, E, k = 300, 128, 10, 4
    idx = _zipf_idx(rng, T, E, k, 1.8, empty=3, bad=2)
    x = _bf16(rng, (T, D))
    flat = idx.ravel()
    valid = (flat >= 0) & (flat < E)
    cnt = np.bincount(flat[valid], minlength=E)
    padded = (cnt + align - 1) // align * align
    offs = np.concatenate([[0], np.cumsum(padded)])
    # rows of each segment in stable order of the flat entry index
    order = np.argsort(np.where(valid, flat, E), kind="stable")[:valid.sum()]
    src_ref = np.full(int(offs[E]) + 256, -1, np.int64)
    for e in range(E):
        ent = order[np.searchsorted(flat[order], e):np.searchsorted(flat[order], e, side="right")]
        src_ref[offs[e]:offs[e] + len(ent)] = ent
    counts, offsets, pos, src = orc.permute(idx, E, align, len(src_ref))
    assert np.array_equal(offsets, offs) and np.array_equal(src, src_ref)
    rows = np.arange(len(src_ref))
    Xp = OL.dispatch_rows(x, src, rows, k)
    ref = np.zeros((len(rows), D), np.uint16)
    ok = src_ref >= 0
    ref[ok] = x[src_ref[ok] // k]
    assert np.array_equal(Xp, ref)
    exp_ref = np.full(len(rows), -1, np.int32)
    exp_ref[:offs[E]] = np.repeat(np.arange(E), padded)
    assert np.array_equal(OL.expert_of_rows(offsets, rows), exp_ref)
    perm = rng.permutation(len(rows))
    assert np.array_equal(OL.expert_of_rows(offsets, rows[perm]), exp_ref[perm])


# --------------------------------------------------------------------------
# dequant_block, router_grads, swiglu_bwd, unpermute_reduce
# --------------------------------------------------------------------------

@pytest.mark.parametrize("br,bc", [(1, 128), (128, 1), (128, 128)])
def test_dequant_block_matches_ml_dtypes(orc, br, bc):
    rng = np.random.default_rng(63)
    rows, cols = 260, 400
    x = to_bf16_bits((rng.standard_normal((rows, cols)) *
                      np.exp(rng.uniform(-8, 8, (rows, 1)))).astype(np.float32))
    q, s = orc.quant_block(x, br, bc)
    got = orc.dequant_block(q, s, br, bc)
    assert np.array_equal(got, _deq(q, s, br, bc))


def test_router_grads_match_torch_autograd(orc):
    from oracle import layer as OL
    rng = np.random.default_rng(64)
    T, D, E, k = 40, 96, 12, 4
    z = rng.standard_normal((T, E)).astype(np.float32)
    idx = np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)
    dy = _bf16(rng, (T, D))
    Yg = rng.standard_normal((T, k, D))
    zS = np.take_along_axis(z.astype(np.float64), idx.astype(np.int64), axis=1)
    w = np.exp(zS - zS.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    d_w, dz = OL.router_grads(dy, Yg, w, z, idx)
    Z = torch.tensor(z.astype(np.float64), requires_grad=True)
    ii = torch.from_numpy(idx.astype(np.int64))
    W = torch.softmax(torch.gather(Z, 1, ii), dim=1)
    Wl = W.detach().clone().requires_grad_(True)
    dyt = torch.from_numpy(orc.bf16_to_f64(dy))
    Yt = torch.from_numpy(Yg)
    (torch.einsum("tk,tkd->td", Wl, Yt) * dyt).sum().backward()
    np.testing.assert_allclose(d_w, Wl.grad.numpy(), rtol=1e-12, atol=1e-12)
    (torch.einsum("tk,tkd->td", W, Yt) * dyt).sum().backward()
    np.testing.assert_allclose(dz, Z.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.all(dz[~_chosen(idx, E)] == 0)   # zero off the chosen set


def _chosen(idx, E):
    m = np.zeros((idx.shape[0], E), bool)
    np.put_along_axis(m, idx.astype(np.int64), True, axis=1)
    return m


def test_swiglu_bwd_matches_torch_autograd(orc):
    from oracle import layer as OL
    rng = np.random.default_rng(65)
    n, I = 64, 256
    g_b = _bf16(rng, (n, I), 3.0)
    u_b = _bf16(rng, (n, I), 1.0)
    dH = rng.standard_normal((n, I))
    dg, du = OL.swiglu_bwd(dH, g_b, u_b)
    G = torch.tensor(orc.bf16_to_f64(g_b), requires_grad=True)
    U = torch.tensor(orc.bf16_to_f64(u_b), requires_grad=True)
    (torch.nn.functional.silu(G) * U * torch.from_numpy(dH)).sum().backward()
    # both sides round an fp64 value to bf16: compare against the library
    # gradient within half a bf16 unit (plus fp64 noise)
    for got, ref in [(dg, G.grad.numpy()), (du, U.grad.numpy())]:
        gv = orc.bf16_to_f64(got)
        spacing = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64) * 2.0 ** 16
        assert np.all(np.abs(gv - ref) <= 0.5 * spacing * (1 + 1e-6) + 1e-300)
        assert np.array_equal(got, orc.bf16_round(ref)) or \
            np.mean(got != orc.bf16_round(ref)) < 1e-3


def test_unpermute_reduce_matches_numpy(orc):
    from oracle import layer as OL
    rng = np.random.default_rng(66)
    T, D, E, k = 120, 64, 7, 3
    idx = _zipf_idx(rng, T, E, k, 1.2, bad=2)
    counts, offsets, pos, src = orc.permute(idx, E, 128)
    R = int(offsets[E])
    dX = rng.standard_normal((R, D))
    got = OL.unpermute_reduce(dX, pos)
    acc = np.zeros((T, D))
    for j in range(k):
        ok = pos[:, j] >= 0
        np.add.at(acc, np.nonzero(ok)[0], dX[pos[ok, j]])
    assert np.array_equal(got, orc.bf16_round(acc))
    assert np.all(orc.bf16_to_f64(got[np.all(pos < 0, axis=1)]) == 0)
