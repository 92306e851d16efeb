"""Pins of the oracle's router logits, routing-payload capture and router
gradients ("RL at 1T scale: prime-rl performance deep dive", §Router Replay:
the experts chosen at inference are recorded as a [num_layers, top_k,
seq_len] integer tensor and replayed by the trainer).  No GPU."""
import json
import os

import numpy as np
import torch

from moe_expert_layer_replay_b200.inputs import to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(rng, shape, std):
    return to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def _t(b):
    """bf16 bits -> torch float64 through torch's own bf16 type."""
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).double()


def test_router_logits_match_torch_matmul(orc):
    from oracle.router import router_logits
    rng = np.random.default_rng(80)
    for T, D, E in [(70, 256, 8), (33, 1024, 64), (5, 128, 256)]:
        x, Wr = _bf16(rng, (T, D), 1.0), _bf16(rng, (E, D), 0.02)
        z = router_logits(x, Wr)
        ref = (_t(x) @ _t(Wr).T).numpy()
        np.testing.assert_allclose(z, ref, rtol=1e-12, atol=1e-12)


def test_capture_matches_golden_layout(orc):
    from oracle.router import capture_payload
    g = json.load(open(os.path.join(GOLDEN, "replay_payload_layout.json")))
    payload = capture_payload([np.array(i, np.int32) for i in g["idx_per_layer"]])
    assert payload.tolist() == g["payload"]


def test_replay_of_captured_router_topk(orc):
    """The capture is what replay consumes: for every layer, replaying the
    captured payload gives back the router's own top-k, and it is the flat
    layout element (l*k + j)*T + t."""
    from oracle.router import capture_payload, router_logits
    rng = np.random.default_rng(81)
    T, D, E, k, L = 300, 256, 16, 4, 3
    x = _bf16(rng, (T, D), 1.0)
    routed = []
    for _ in range(L):
        z = router_logits(x, _bf16(rng, (E, D), 0.05)).astype(np.float32)
        routed.append((z,) + orc.route_topk(z, k))
    payload = capture_payload([r[1] for r in routed])
    flat = payload.ravel()
    for l, (z, idx, w) in enumerate(routed):
        for j in range(k):
            assert np.array_equal(flat[(l * k + j) * T:(l * k + j + 1) * T], idx[:, j])
        idx_r, w_r, st = orc.route_replay(payload, l, E, z=z)
        assert st == 0 and np.array_equal(idx_r, idx) and np.array_equal(w_r, w)


def test_router_backward_matches_torch_autograd(orc):
    from oracle.router import router_backward
    rng = np.random.default_rng(82)
    T, D, E = 40, 384, 24
    x, Wr = _bf16(rng, (T, D), 1.0), _bf16(rng, (E, D), 0.02)
    dz = rng.standard_normal((T, E))
    dz[rng.random((T, E)) < 0.6] = 0.0   # zero off the chosen sets
    dx, dW = router_backward(x, Wr, dz)
    X = _t(x).requires_grad_(True)
    W = _t(Wr).requires_grad_(True)
    ((X @ W.T) * torch.from_numpy(dz)).sum().backward()
    np.testing.assert_allclose(dx, X.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dW, W.grad.numpy(), rtol=1e-12, atol=1e-12)
