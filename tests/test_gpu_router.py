"""Parity of the router (logits on the tensor cores, then the top-k), of the
capture of its decisions into the replay payload, and of the router backward,
through the C ABI, against the oracle ("RL at 1T scale: prime-rl performance
deep dive", §Router Replay: the experts chosen at inference are recorded as a
[num_layers, top_k, seq_len] tensor and replayed by the trainer).

The logits are float outputs (contract tolerance against the fp64 oracle);
the top-k decision is compared bit for bit with the oracle's top-k taken on
the kernel's own fp32 logits (both sides decide in the kernel's precision).
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


# T, D, E, k: several 128-token tiles with a ragged tail, E below / at / above
# one 16-column MMA step, the widest N (256), and d_model of the workloads
CASES = [(300, 256, 8, 2), (1000, 2048, 64, 6), (4096, 7168, 32, 8), (129, 128, 256, 16), (77, 6144, 20, 4)]


@pytest.mark.parametrize("T,D,E,k", CASES)
def test_router_fwd_and_capture(A, orc, T, D, E, k):
    from oracle.router import capture_payload, router_logits
    rng = np.random.default_rng(900 + T + E)
    x = rand_bf16(rng, (T, D))
    Wr = rand_bf16(rng, (E, D), 0.02)
    d = A.dims(T, D, 128, E, k)
    z = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    A.router_fwd(dev(x), dev(Wr), d, z, idx, w)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    zg = host(z)
    close(zg, router_logits(x, Wr), what="router logits")
    oi, ow = orc.route_topk(zg, k)
    same_bits(host(idx), oi, "top-k of the kernel's logits")
    np.testing.assert_allclose(host(w), ow, rtol=2e-6, atol=1e-7)
    # capture into layer 1 of a 3-layer payload; the other layers are untouched
    L = 3
    P = torch.full((L, k, T), -5, dtype=torch.int32, device="cuda")
    A.capture_payload(idx, d, L, 1, P)
    Pg = host(P)
    same_bits(Pg[1], capture_payload([oi])[0], "captured layer")
    assert np.all(Pg[0] == -5) and np.all(Pg[2] == -5)
    # and replay of the captured payload gives the router's choice back
    ri = torch.empty(T, k, dtype=torch.int32, device="cuda")
    rw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    A.route_replay(P, L, 1, d, None, z, ri, rw)
    same_bits(host(ri), oi, "replay(capture(top-k))")
    # the same softmax over the same set, summed in another order (1-ulp differences)
    np.testing.assert_allclose(host(rw), host(w), rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T,D,E", [(300, 256, 8), (1000, 2048, 64), (513, 7168, 32), (64, 384, 256)])
def test_router_bwd(A, orc, T, D, E):
    from oracle.router import router_backward
    rng = np.random.default_rng(950 + T)
    x = rand_bf16(rng, (T, D))
    Wr = rand_bf16(rng, (E, D), 0.02)
    dz = (rng.standard_normal((T, E)) * 1e-2).astype(np.float32)
    dz[rng.random((T, E)) < 0.7] = 0.0   # the logit gradient is zero off the chosen set
    dx_in = rand_bf16(rng, (T, D), 1e-2)
    dW0 = (rng.standard_normal((E, D)) * 1e-3).astype(np.float32)
    d = A.dims(T, D, 128, E, 1)
    ws = torch.empty(A.router_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    dx = dev(dx_in).clone()                # in place: dx_in == dx
    dW = dev(dW0)
    A.router_bwd(dev(dz), dev(x), dev(Wr), d, dx_in=dx, dx=dx, dw_r=dW, ws=ws)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    rdx, rdW = router_backward(x, Wr, dz)
    close(bf(host(dx)), bf(orc.bf16_round(bf(dx_in) + rdx)), bf16=True, what="dx (router share added in place)")
    close(host(dW), dW0.astype(np.float64) + rdW, what="dW_r (+=)")
    # dx alone, no input to add, no weight gradient
    dx2 = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    A.router_bwd(dev(dz), None, dev(Wr), d, dx=dx2)
    torch.cuda.synchronize()
    close(bf(host(dx2)), bf(orc.bf16_round(rdx)), bf16=True, what="dx (router share only)")
