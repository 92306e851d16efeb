"""Per-kernel parity of the CUDA path (through the C ABI) against the oracle,
on seeded inputs that span several tiles and a ragged tail.

Bit-exact: routing indices, counts, offsets, permutation indices, FP8 codes
and fp32 scales.  Floating-point outputs: the parity tolerance in _util.
"""
import numpy as np
import pytest
import torch

from _util import bf, close, dev, host, rand_bf16, same_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from moe_expert_layer_replay_b200 import abi, build
    build.build()
    abi.lib()
    return abi


def _special_bf16(rng, rows, cols):
    x = rand_bf16(rng, (rows, cols), 1.0)
    x[0, :] = 0                                   # all-zero blocks
    x[1, :] = rand_bf16(rng, (1, cols), 1e-38)    # subnormal scales
    x[2, ::3] = 0x8000                            # negative zeros
    x[3, :] = rand_bf16(rng, (1, cols), 1e4)
    return x


@pytest.mark.parametrize("rows,cols", [(256, 512), (200, 384), (1, 128), (333, 1152), (64, 48)])
def test_quant_1x128(A, orc, rows, cols):
    rng = np.random.default_rng(100 + rows)
    x = _special_bf16(rng, rows, cols) if rows >= 4 else rand_bf16(rng, (rows, cols))
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty((cols + 127) // 128, rows, dtype=torch.float32, device="cuda")
    A.quant_fp8_block(dev(x), rows, cols, cols, 1, 128, q, s)
    oq, os_ = orc.quant_block(x, 1, 128)
    same_bits(host(q), oq, "codes")
    same_bits(host(s).T, os_, "scales")


@pytest.mark.parametrize("rows,cols", [(256, 512), (208, 384), (128, 64), (96, 1040)])
def test_quant_rows128(A, orc, rows, cols):
    rng = np.random.default_rng(200 + rows)
    x = _special_bf16(rng, rows, cols)
    q = torch.empty(cols, rows, dtype=torch.uint8, device="cuda")
    s = torch.empty((rows + 127) // 128, cols, dtype=torch.float32, device="cuda")
    A.quant_fp8_block(dev(x), rows, cols, cols, 128, 1, q, s)
    oq, os_ = orc.quant_block(x, 128, 1)
    same_bits(host(q).T, oq, "codes")
    same_bits(host(s), os_, "scales")


@pytest.mark.parametrize("rows,cols,with_t", [(384, 256, True), (256, 640, False), (208, 336, True)])
def test_quant_128x128(A, orc, rows, cols, with_t):
    rng = np.random.default_rng(300 + rows)
    x = _special_bf16(rng, rows, cols)
    nbr, nbc = (rows + 127) // 128, (cols + 127) // 128
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(nbr, nbc, dtype=torch.float32, device="cuda")
    qT = torch.empty(cols, rows, dtype=torch.uint8, device="cuda") if with_t else None
    sT = torch.empty(nbc, nbr, dtype=torch.float32, device="cuda") if with_t else None
    A.quant_fp8_block(dev(x), rows, cols, cols, 128, 128, q, s, qT, sT)
    oq, os_ = orc.quant_block(x, 128, 128)
    same_bits(host(q), oq, "codes")
    same_bits(host(s), os_, "scales")
    if with_t:
        oqT, osT = orc.quant_block(np.ascontiguousarray(x.T), 128, 128)
        same_bits(host(qT), oqT, "transposed codes")
        same_bits(host(sT), osT, "transposed scales")


def test_quant_weights_layout(A, orc):
    from oracle.layer import quant_weights
    rng = np.random.default_rng(400)
    E, D, I = 3, 384, 256
    Wg, Wu, Wd = rand_bf16(rng, (E, I, D), .02), rand_bf16(rng, (E, I, D), .02), rand_bf16(rng, (E, D, I), .02)
    from moe_expert_layer_replay_b200 import layer
    d = A.dims(1, D, I, E, 1)
    W = layer.quantise_weights(d, dev(Wg), dev(Wu), dev(Wd), train=True)
    (gq, gs), (uq, us), (dq, ds) = quant_weights(Wg), quant_weights(Wu), quant_weights(Wd)
    wgu_q, wgu_s = host(W.wgu_q), host(W.wgu_s)
    for b in range(I // 128):
        same_bits(wgu_q[:, 256 * b:256 * b + 128], gq[:, 128 * b:128 * b + 128], "gate codes")
        same_bits(wgu_q[:, 256 * b + 128:256 * b + 256], uq[:, 128 * b:128 * b + 128], "up codes")
        same_bits(wgu_s[:, 2 * b], gs[:, b], "gate scales")
        same_bits(wgu_s[:, 2 * b + 1], us[:, b], "up scales")
    same_bits(host(W.wd_q), dq, "down codes")
    same_bits(host(W.wd_s), ds, "down scales")
    same_bits(host(W.wguT_q), wgu_q.transpose(0, 2, 1), "transposed gate/up codes")
    same_bits(host(W.wguT_s), wgu_s.transpose(0, 2, 1), "transposed gate/up scales")
    same_bits(host(W.wdT_q), dq.transpose(0, 2, 1), "transposed down codes")
    same_bits(host(W.wdT_s), ds.transpose(0, 2, 1), "transposed down scales")


@pytest.mark.parametrize("T,E,k,ties", [(300, 8, 2, False), (1000, 64, 6, False), (257, 32, 8, True),
                                        (40, 256, 16, False), (33, 5, 5, True)])
def test_route_topk(A, orc, T, E, k, ties):
    rng = np.random.default_rng(500 + T)
    z = (rng.integers(-3, 3, (T, E)) if ties else rng.standard_normal((T, E))).astype(np.float32)
    z[0, :E // 2] = -np.inf
    d = A.dims(T, 128, 128, E, k)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    A.route_topk(dev(z), d, idx, w)
    oi, ow = orc.route_topk(z, k)
    same_bits(host(idx), oi, "idx")
    np.testing.assert_allclose(host(w), ow, rtol=2e-6, atol=1e-7)


def test_route_replay(A, orc):
    rng = np.random.default_rng(600)
    T, E, k, L = 1000, 64, 6, 3
    P = np.stack([np.stack([rng.permutation(E)[:k] for _ in range(T)]).T for _ in range(L)]).astype(np.int32)
    w_in = rng.random((T, k)).astype(np.float32)
    z = rng.standard_normal((T, E)).astype(np.float32)
    d = A.dims(T, 128, 128, E, k)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    for layer in range(L):
        A.route_replay(dev(P), L, layer, d, dev(w_in), None, idx, w)
        oi, ow, st = orc.route_replay(P, layer, E, w_in=w_in)
        same_bits(host(idx), oi, "idx")
        same_bits(host(w), ow, "weights (copied)")
        A.route_replay(dev(P), L, layer, d, None, dev(z), idx, w)
        oi, ow, st = orc.route_replay(P, layer, E, z=z)
        same_bits(host(idx), oi, "idx")
        np.testing.assert_allclose(host(w), ow, rtol=2e-6, atol=1e-7)
    assert A.get_status() == A.OK


def test_route_replay_bad_payload(A, orc):
    T, E, k = 64, 8, 2
    rng = np.random.default_rng(601)
    P = np.stack([np.stack([rng.permutation(E)[:k] for _ in range(T)]).T]).astype(np.int32)
    P[0, 1, 5] = E + 3      # out of range
    P[0, 1, 9] = P[0, 0, 9]  # repeated
    w_in = np.full((T, k), 0.5, np.float32)
    d = A.dims(T, 128, 128, E, k)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    assert A.get_status() == A.OK
    A.route_replay(dev(P), 1, 0, d, dev(w_in), None, idx, w)
    assert A.get_status() == A.BAD_ROUTING
    assert A.get_status() == A.OK  # read clears
    oi, ow, st = orc.route_replay(P, 0, E, w_in=w_in)
    assert st == 4
    same_bits(host(idx), oi, "idx")
    same_bits(host(w), ow, "weights")


def _permute_case(A, orc, T, E, k, D, align, zipf, train, seed):
    rng = np.random.default_rng(seed)
    p = np.arange(1, E + 1, dtype=np.float64) ** -zipf
    if E > k + 2:
        p[-2:] = 0
    p /= p.sum()
    keys = np.log(p + 1e-300)[None, :] - np.log(-np.log(rng.random((T, E))))
    idx = np.argsort(-keys, axis=1, kind="stable")[:, :k].astype(np.int32)
    x = _special_bf16(rng, T, D) if T >= 4 else rand_bf16(rng, (T, D))
    d = A.dims(T, D, 128, E, k, align)
    R = A.rows_capacity(d)
    g = lambda *s, dt=torch.int32: torch.empty(*s, dtype=dt, device="cuda")
    counts, offsets, pos, src = g(E), g(E + 1), g(T, k), g(R)
    xq, xs = g(R, D, dt=torch.uint8), g(D // 128, R, dt=torch.float32)
    xqT = g(D, R, dt=torch.uint8) if train else None
    xsT = g(R // 128, D, dt=torch.float32) if train else None
    ws = g(A.permute_workspace_size(d), dt=torch.uint8)
    A.permute(dev(idx), d, counts, offsets, pos, src, dev(x), xq, xs, xqT, xsT, ws)
    oc, oo, op, osrc = orc.permute(idx, E, align, R)
    same_bits(host(counts), oc, "counts")
    same_bits(host(offsets), oo, "offsets")
    same_bits(host(pos), op, "pos")
    same_bits(host(src), osrc, "src_idx")
    Rp = int(oo[E])
    from oracle.layer import dispatch_rows
    Xp = dispatch_rows(x, osrc, np.arange(Rp), k)
    oq, os_ = orc.quant_block(Xp, 1, 128)
    same_bits(host(xq)[:Rp], oq, "dispatched codes")
    same_bits(host(xs)[:, :Rp].T, os_, "dispatched scales")
    if train:
        oqT, osT = orc.quant_block(Xp, 128, 1)
        same_bits(host(xqT)[:, :Rp].T, oqT, "128x1 codes")
        same_bits(host(xsT)[:Rp // 128], osT, "128x1 scales")


@pytest.mark.parametrize("T,E,k,D,align,zipf,train", [
    (256, 8, 2, 256, 128, 0.0, False), (4096, 64, 6, 512, 128, 1.1, True), (1000, 32, 8, 256, 1, 1.2, False),
    (5000, 32, 8, 384, 128, 1.2, True), (3, 4, 2, 128, 128, 0.0, True), (0, 4, 2, 128, 128, 0.0, False)])
def test_permute_and_dispatch(A, orc, T, E, k, D, align, zipf, train):
    _permute_case(A, orc, T, E, k, D, align, zipf, train, seed=700 + T)


def test_permute_drops_invalid(A, orc):
    T, E, k = 100, 8, 2
    idx = np.stack([np.random.default_rng(800).permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    idx[7, 1] = 9
    idx[50, 0] = -2
    d = A.dims(T, 128, 128, E, k, 128)
    R = A.rows_capacity(d)
    g = lambda *s: torch.empty(*s, dtype=torch.int32, device="cuda")
    counts, offsets, pos, src = g(E), g(E + 1), g(T, k), g(R)
    ws = torch.empty(A.permute_workspace_size(d), dtype=torch.uint8, device="cuda")
    A.permute(dev(idx), d, counts, offsets, pos, src, None, None, None, None, None, ws)
    assert A.get_status() == A.BAD_ROUTING
    oc, oo, op, osrc = orc.permute(idx, E, 128, R)
    same_bits(host(pos), op, "pos")
    same_bits(host(src), osrc, "src")


def test_combine_and_unpermute(A, orc):
    from oracle.layer import combine, unpermute_reduce
    rng = np.random.default_rng(900)
    T, E, k, D = 700, 16, 4, 640
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    oc, oo, op, osrc = orc.permute(idx, E, 128)
    R = len(osrc)
    Y = rand_bf16(rng, (R, D))
    w = rng.random((T, k)).astype(np.float32)
    d = A.dims(T, D, 128, E, k)
    y = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    A.combine(dev(Y), dev(w), dev(op), d, y)
    ref = combine(bf(Y)[op], w, op >= 0)
    close(bf(host(y)), bf(ref), bf16=True, what="combine")
    dx = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    A.unpermute_reduce(dev(Y), dev(op), d, dx)
    ref = unpermute_reduce(bf(Y), op)
    close(bf(host(dx)), bf(ref), bf16=True, what="unpermute")


def test_combine_bwd(A, orc):
    from oracle.layer import router_grads, scaled_rows
    rng = np.random.default_rng(1000)
    T, E, k, D = 600, 16, 4, 512
    z = rng.random((T, E)).astype(np.float32)
    idx, w = orc.route_topk(z, k)
    oc, oo, op, osrc = orc.permute(idx, E, 128)
    R = len(osrc)
    Rp = int(oo[E])
    Y = rand_bf16(rng, (R, D))
    dy = rand_bf16(rng, (T, D), 0.01)
    d = A.dims(T, D, 128, E, k)
    g = lambda *s, dt: torch.empty(*s, dtype=dt, device="cuda")
    dYq, dYs = g(R, D, dt=torch.uint8), g(D // 128, R, dt=torch.float32)
    dYb = g(R, D, dt=torch.bfloat16)
    d_w, dz = g(T, k, dt=torch.float32), g(T, E, dt=torch.float32)
    A.combine_bwd(dev(dy), dev(Y), dev(w), dev(op), dev(idx), dev(oc), dev(oo), d, dYq, dYs, dYb, d_w, dz)
    rows = scaled_rows(dy, w, op, Rp)
    same_bits(host(dYb)[:Rp], rows, "dY rows bf16")
    oq, os_ = orc.quant_block(rows, 1, 128)
    same_bits(host(dYq)[:Rp], oq, "dY codes")
    same_bits(host(dYs)[:, :Rp].T, os_, "dY scales")
    ref_dw, ref_dz = router_grads(dy, bf(Y)[op], w, z, idx)
    close(host(d_w), ref_dw, what="d_w")
    close(host(dz), ref_dz, what="d_logits")


@pytest.mark.parametrize("blk", [(1, 128), (128, 1), (128, 128)])
def test_quant_exhaustive_bf16(A, orc, blk):
    """Every finite bf16 value, in blocks whose amax (hence scale) varies from
    subnormal to large, quantises bit-exactly like the oracle's IEEE
    definition (scale = fp32(amax/448), code = e4m3(fp32(x/scale)))."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7F80) != 0x7F80
    vals = bits[finite]
    rng = np.random.default_rng(7)
    rng.shuffle(vals)
    n = (len(vals) + 16383) // 16384 * 16384
    x = np.zeros(n, np.uint16)
    x[:len(vals)] = vals
    x = x.reshape(-1, 128)  # 512 rows x 128
    # vary the block maxima: some blocks get a planted amax from subnormal to 1e30
    planted = orc.bf16_round(np.logspace(-40, 30, x.shape[0]) * rng.choice([-1, 1], x.shape[0]))
    x[np.arange(x.shape[0]), rng.integers(0, 128, x.shape[0])] = planted
    br, bc = blk
    rows, cols = x.shape
    if br == 1:
        q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
        s = torch.empty(cols // 128, rows, dtype=torch.float32, device="cuda")
        A.quant_fp8_block(dev(x), rows, cols, cols, 1, 128, q, s)
        oq, os_ = orc.quant_block(x, 1, 128)
        same_bits(host(q), oq, "codes")
        same_bits(host(s).T, os_, "scales")
    elif bc == 1:
        q = torch.empty(cols, rows, dtype=torch.uint8, device="cuda")
        s = torch.empty(rows // 128, cols, dtype=torch.float32, device="cuda")
        A.quant_fp8_block(dev(x), rows, cols, cols, 128, 1, q, s)
        oq, os_ = orc.quant_block(x, 128, 1)
        same_bits(host(q).T, oq, "codes")
        same_bits(host(s), os_, "scales")
    else:
        q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
        s = torch.empty(rows // 128, 1, dtype=torch.float32, device="cuda")
        A.quant_fp8_block(dev(x), rows, cols, cols, 128, 128, q, s)
        oq, os_ = orc.quant_block(x, 128, 128)
        same_bits(host(q), oq, "codes")
        same_bits(host(s), os_, "scales")


def test_quant_scale_sweep_bf16(A, orc):
    """Every bf16 mantissa against every block scale from the subnormal range
    up: block b holds its planted amax m_b * 2^e_b and the 128 bf16 mantissas
    spread over the 20 binades below it.  Amax mantissas include 1.75 and 1.5,
    for which many quotients fall exactly on e4m3 rounding midpoints (the ties
    the quantiser must decide exactly); the sweep crosses the scale range where
    the kernel switches from its reciprocal path to IEEE division."""
    rng = np.random.default_rng(11)
    mants = 1.0 + np.arange(128) / 128.0
    amax_m = np.array([1.0, 1.5, 1.75, 1.25, 1.9921875, 1.0078125, 1.375, 1.625])
    blocks = []
    for e in range(-126, 121):
        for am in amax_m:
            shift = rng.integers(0, 21, 128)
            sign = rng.choice([-1.0, 1.0], 128)
            v = sign * rng.permutation(mants) * np.ldexp(1.0, e - shift)
            v[rng.integers(0, 128)] = am * np.ldexp(1.0, e) * rng.choice([-1.0, 1.0])
            blocks.append(v)
    x = orc.bf16_round(np.stack(blocks))  # values below the bf16 range flush to signed zero
    rows, cols = x.shape
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, rows, dtype=torch.float32, device="cuda")
    A.quant_fp8_block(dev(x), rows, cols, cols, 1, 128, q, s)
    oq, os_ = orc.quant_block(x, 1, 128)
    same_bits(host(s).T, os_, "scales")
    same_bits(host(q), oq, "codes")
