"""Expert parallelism on one GPU ("RL at 1T scale: prime-rl performance deep
dive", §Parallelism strategy / EP).

* The segment-grouped GEMMs (moe_grouped_gemm_fp8_seg) on a received-rows
  layout: one 128-aligned segment per (source rank, local expert), empty
  segments included, segment v using local expert v % E_loc's weights —
  against the oracle's FFN steps on the same operands.
* ep.forward on a one-rank NCCL group (the exchange sends to itself) equals
  the plain layer forward bit for bit.
Several GPUs (the all-to-all between ranks) are covered on gloo ranks on the
host (test_ep_gloo.py); this run has one GPU.
"""
import os
import socket

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


@pytest.mark.parametrize("world,E_loc,D,I", [(2, 4, 512, 256), (8, 4, 256, 384), (4, 8, 2048, 1024)])
def test_segment_gemm_matches_oracle(A, orc, world, E_loc, D, I):
    from oracle import layer as OL
    rng = np.random.default_rng(70 + world)
    n_seg = world * E_loc
    cnt = rng.integers(0, 300, n_seg)
    cnt[rng.integers(0, n_seg, 2)] = 0                   # empty segments
    seg = (cnt + 127) // 128 * 128
    offs = np.concatenate([[0], np.cumsum(seg)]).astype(np.int32)
    R = int(offs[-1])
    rows_cap = R + 256                                     # capacity above the rows in use
    X = np.zeros((rows_cap, D), np.uint16)
    for v in range(n_seg):                                 # real rows, then zero padding rows
        X[offs[v]:offs[v] + cnt[v]] = rand_bf16(rng, (cnt[v], D))
    xq, xs = orc.quant_block(X, 1, 128)
    Wg, Wu, Wd = rand_bf16(rng, (E_loc, I, D), 0.02), rand_bf16(rng, (E_loc, I, D), 0.02), rand_bf16(rng, (E_loc, D, I), 0.02)
    from moe_expert_layer_replay_b200 import layer
    d = A.dims(16, D, I, E_loc, 2)
    W = layer.quantise_weights(d, dev(Wg), dev(Wu), dev(Wd), train=False)
    hq = torch.zeros(rows_cap, I, dtype=torch.uint8, device="cuda")
    hs = torch.zeros(I // 128, rows_cap, dtype=torch.float32, device="cuda")
    h = torch.zeros(rows_cap, I, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(rows_cap, D, dtype=torch.bfloat16, device="cuda")
    so = dev(offs)
    A.grouped_gemm_fp8_seg(A.GEMM_GATEUP_SILU, d, rows_cap, so, n_seg, dev(xq), dev(np.ascontiguousarray(xs.T)),
                           W.wgu_q, W.wgu_s, out_q=hq, out_s=hs, out_bf16=h)
    A.grouped_gemm_fp8_seg(A.GEMM_DOWN, d, rows_cap, so, n_seg, hq, hs, W.wd_q, W.wd_s, out_bf16=Y)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    Wq = (OL.quant_weights(Wg), OL.quant_weights(Wu), OL.quant_weights(Wd))
    expert = OL.expert_of_rows(offs, np.arange(R)) % E_loc
    g, u = OL.gateup_rows(xq[:R], xs[:R], expert, Wq[0], Wq[1])
    close(bf(host(h)[:R]), bf(OL.swiglu_h(g, u)), bf16=True, what="h over segments")
    hq_ref, hs_ref = orc.quant_block(host(h)[:R], 1, 128)
    same_bits(host(hq)[:R], hq_ref, "hq = quant(h)")
    Y_ref = OL.down_rows(host(hq)[:R], host(hs)[:, :R].T.copy(), expert, Wq[2])
    close(bf(host(Y)[:R]), bf(Y_ref), bf16=True, what="Y over segments")
    pad = np.concatenate([np.arange(offs[v] + cnt[v], offs[v + 1]) for v in range(n_seg)]).astype(np.int64)
    assert not np.any(host(Y)[pad]), "padding rows give zero outputs"


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_forward_one_rank_equals_layer_forward(A):
    import torch.distributed as dist
    from moe_expert_layer_replay_b200 import ep, layer
    from moe_expert_layer_replay_b200.inputs import make_inputs
    inp = make_inputs("replay", seed=3, T=1024)
    wl = inp["workload"]
    d = A.dims(wl.T, wl.D, wl.I, wl.E, wl.k)
    W = layer.quantise_weights(d, dev(inp["W_gate"]), dev(inp["W_up"]), dev(inp["W_down"]), train=False)
    B0 = layer.Buffers(d, "cuda", train=False)
    B1 = layer.Buffers(d, "cuda", train=False)
    P, w_in, x = dev(inp["payload"]), dev(inp["w_in"][0]), dev(inp["x"])
    for B in (B0, B1):
        layer.route(B, payload=P, layer=0, w_in=w_in)
    layer.forward(B0, x, W)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        ep.forward(B1, x, W)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert A.get_status() == A.OK
    Rp = int(host(B0.offsets)[wl.E])
    same_bits(host(B1.Y)[:Rp], host(B0.Y)[:Rp], "expert outputs")
    same_bits(host(B1.y), host(B0.y), "combined outputs")
