"""Pins of the oracle's expert FFN, combine and backward.  No GPU.

The expert FFN form (SiLU-gated gate/up, down projection) and the rounding
points are readings stated in oracle/layer.py; these tests pin the fp64
composition against library routines (numpy matmul, torch autograd) and
closed forms, so that a dropped term, a wrong sign or a transposed operand
fails one of them.
"""
import numpy as np
import pytest
import torch

from moe_expert_layer_replay_b200.inputs import make_inputs, to_bf16_bits


def _small(T=48, D=256, I=128, E=4, k=2, seed=30):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, D))
    Wg = rng.standard_normal((E, I, D)) * 0.05
    Wu = rng.standard_normal((E, I, D)) * 0.05
    Wd = rng.standard_normal((E, D, I)) * 0.05
    z = rng.standard_normal((T, E))
    idx = np.argsort(-z, axis=1, kind="stable")[:, :k].astype(np.int32)
    zS = np.take_along_axis(z, idx.astype(np.int64), axis=1)
    w = np.exp(zS - zS.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    dy = rng.standard_normal((T, D))
    return x, Wg, Wu, Wd, z, idx, w, dy


def test_rowdot_matches_numpy_matmul(orc):
    rng = np.random.default_rng(31)
    E, N, K, n = 3, 256, 384, 50
    Wb = to_bf16_bits(rng.standard_normal((E, N, K)).astype(np.float32) * 0.02)
    from oracle.layer import quant_weights
    Wq, Ws = quant_weights(Wb)
    A = rng.standard_normal((n, K))
    ex = rng.integers(-1, E, n).astype(np.int32)
    out = orc.rowdot(A, ex, (Wq, Ws))
    Wf = np.stack([orc.dequant_block(Wq[e], Ws[e], 128, 128) for e in range(E)])
    for i in range(n):
        ref = Wf[ex[i]] @ A[i] if ex[i] >= 0 else np.zeros(N)
        assert np.allclose(out[i], ref, rtol=1e-12, atol=1e-12)
    B = rng.standard_normal((n, N))
    outT = orc.rowdot(B, ex, (Wq, Ws), trans=True)
    for i in range(n):
        ref = Wf[ex[i]].T @ B[i] if ex[i] >= 0 else np.zeros(K)
        assert np.allclose(outT[i], ref, rtol=1e-12, atol=1e-12)


def test_wgrad_matches_numpy(orc):
    rng = np.random.default_rng(32)
    A, B = rng.standard_normal((300, 40)), rng.standard_normal((300, 24))
    assert np.allclose(orc.wgrad(A, B), A.T @ B, rtol=1e-12, atol=1e-12)
    assert np.allclose(orc.wgrad(A, B, 5, 10, 3, 7), (A.T @ B)[5:15, 3:10], rtol=1e-12)


def test_single_expert_reduces_to_dense_gated_ffn(orc):
    from oracle.layer import forward_exact
    x, Wg, Wu, Wd, z, idx, w, dy = _small(E=1, k=1)
    y = forward_exact(x, idx, w, Wg, Wu, Wd)
    X = torch.from_numpy(x)
    ref = (torch.nn.functional.silu(X @ torch.from_numpy(Wg[0]).T) * (X @ torch.from_numpy(Wu[0]).T)) \
        @ torch.from_numpy(Wd[0]).T
    assert np.allclose(y, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_exact_backward_matches_torch_autograd(orc):
    from oracle.layer import backward_exact
    x, Wg, Wu, Wd, z, idx, w, dy = _small()
    got = backward_exact(x, idx, w, Wg, Wu, Wd, dy, z=z)
    X = torch.tensor(x, requires_grad=True)
    G = torch.tensor(Wg, requires_grad=True)
    U = torch.tensor(Wu, requires_grad=True)
    Dn = torch.tensor(Wd, requires_grad=True)
    Z = torch.tensor(z, requires_grad=True)
    ii = torch.from_numpy(idx.astype(np.int64))
    W = torch.softmax(torch.gather(Z, 1, ii), dim=1)
    y = torch.zeros_like(X)
    for j in range(idx.shape[1]):
        e = ii[:, j]
        g = torch.einsum("tid,td->ti", G[e], X)
        u = torch.einsum("tid,td->ti", U[e], X)
        Y = torch.einsum("tdi,ti->td", Dn[e], torch.nn.functional.silu(g) * u)
        y = y + W[:, j:j + 1] * Y
    (y * torch.from_numpy(dy)).sum().backward()
    for name, ref in [("dx", X.grad), ("dWg", G.grad), ("dWu", U.grad), ("dWd", Dn.grad), ("dz", Z.grad)]:
        assert np.allclose(got[name], ref.numpy(), rtol=1e-9, atol=1e-11), name


def test_exact_backward_central_differences(orc):
    """Finite differences of forward_exact on a few parameters (independent of
    autograd)."""
    from oracle.layer import backward_exact, forward_exact
    x, Wg, Wu, Wd, z, idx, w, dy = _small(T=8, D=128, I=128, E=2, k=2, seed=33)
    got = backward_exact(x, idx, w, Wg, Wu, Wd, dy)
    f = lambda xx, g, u, d, ww: float((forward_exact(xx, idx, ww, g, u, d) * dy).sum())
    h = 1e-6
    rng = np.random.default_rng(34)
    for name, arr in [("dx", x), ("dWg", Wg), ("dWu", Wu), ("dWd", Wd), ("d_w", w)]:
        for _ in range(3):
            pos = tuple(rng.integers(0, s) for s in arr.shape)
            if name in ("dWg", "dWu", "dWd") and not np.any(idx == pos[0]):
                continue
            arrs = {"dx": x, "dWg": Wg, "dWu": Wu, "dWd": Wd, "d_w": w}
            plus = {kk: v.copy() for kk, v in arrs.items()}
            minus = {kk: v.copy() for kk, v in arrs.items()}
            plus[name][pos] += h
            minus[name][pos] -= h
            num = (f(plus["dx"], plus["dWg"], plus["dWu"], plus["dWd"], plus["d_w"])
                   - f(minus["dx"], minus["dWg"], minus["dWu"], minus["dWd"], minus["d_w"])) / (2 * h)
            assert abs(num - got[name][pos]) <= 1e-6 * max(1.0, abs(num)), (name, pos)


def _bf16_inputs(T=256, seed=35):
    inp = make_inputs("tiny", seed=seed, T=T)
    return inp


def test_quantised_forward_close_to_exact(orc):
    """The quantised pipeline stays within FP8 error of the unquantised one
    (a wiring mistake — wrong scale layout, wrong expert, swapped operands —
    gives O(1) error)."""
    from oracle.layer import forward, forward_exact
    inp = _bf16_inputs()
    idx, w = orc.route_topk(inp["logits"], 2)
    fw = forward(inp["x"], idx, w, inp["W_gate"], inp["W_up"], inp["W_down"])
    f = orc.bf16_to_f64
    y_ref = forward_exact(f(inp["x"]), idx, w.astype(np.float64), f(inp["W_gate"]),
                          f(inp["W_up"]), f(inp["W_down"]))
    y = f(fw["y"])
    rel = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert rel < 0.08, rel


def test_quantised_backward_close_to_exact(orc):
    from oracle.layer import backward, backward_exact, forward
    rng = np.random.default_rng(37)
    E, D, I, k = 4, 256, 128, 2
    f = orc.bf16_to_f64
    Wg = to_bf16_bits(rng.standard_normal((E, I, D)).astype(np.float32) * 0.02)
    Wu = to_bf16_bits(rng.standard_normal((E, I, D)).astype(np.float32) * 0.02)
    Wd = to_bf16_bits(rng.standard_normal((E, D, I)).astype(np.float32) * 0.02)
    x = to_bf16_bits(rng.standard_normal((256, D)).astype(np.float32))
    dy = to_bf16_bits(rng.standard_normal((256, D)).astype(np.float32) * 0.01)
    z = rng.random((256, E)).astype(np.float32)
    idx, w = orc.route_topk(z, k)
    fw = forward(x, idx, w, Wg, Wu, Wd)
    bw = backward(fw, x, dy, idx, w, z=z)
    ex = backward_exact(f(x), idx, w.astype(np.float64), f(Wg), f(Wu), f(Wd), f(dy), z=z.astype(np.float64))
    for name, got in [("dx", f(bw["dx"])), ("dWg", bw["dWg"]), ("dWu", bw["dWu"]),
                      ("dWd", bw["dWd"]), ("d_w", bw["d_w"]), ("dz", bw["dz"])]:
        rel = np.linalg.norm(got - ex[name]) / np.linalg.norm(ex[name])
        assert rel < 0.1, (name, rel)


def test_zero_input_gives_zero_output(orc):
    """silu(0) = 0 and the s = 0 rule: x = 0 flows through as exact zeros."""
    from oracle.layer import forward
    inp = _bf16_inputs()
    idx, w = orc.route_topk(inp["logits"], 2)
    fw = forward(np.zeros_like(inp["x"]), idx, w, inp["W_gate"], inp["W_up"], inp["W_down"])
    assert np.all(fw["xs"] == 0) and np.all(fw["hq"] == 0) and np.all(fw["y"] == 0)


def test_identity_experts_combine_returns_input(orc):
    """With Y_r = x[src token] the weighted combine returns x (weights sum to
    1) within one bf16 ulp."""
    from oracle.layer import combine
    inp = _bf16_inputs()
    idx, w = orc.route_topk(inp["logits"], 2)
    counts, offsets, pos, src = orc.permute(idx, 8, 128)
    x = orc.bf16_to_f64(inp["x"])
    ok = pos >= 0
    Yg = x[:, None, :].repeat(2, axis=1)  # Y[pos[t, j]] = x[t]
    y = orc.bf16_to_f64(combine(Yg, w, ok))
    ulp = np.spacing(np.abs(x).astype(np.float32)).astype(np.float64) * 2 ** 16
    assert np.all(np.abs(y - x) <= ulp)
