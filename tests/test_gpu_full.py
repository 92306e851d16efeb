"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times, on sampled tokens the oracle computes one by one.

Bit-exact over ALL tokens: routing indices, counts, offsets, permutation
indices, source rows.  On a seeded sample of tokens: their dispatched FP8 rows
(bit-exact), h (contract tolerance), the fused h-quantiser (bit-exact against
the oracle quantiser applied to the GPU's h), Y from the GPU's hq (contract
tolerance) and y end to end.
"""
import numpy as np
import pytest
import torch

from _util import MAX_ABS_RMS_E2E, bf, close, dev, host, same_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from moe_expert_layer_replay_b200 import abi, build
    build.build()
    abi.lib()
    return abi


@pytest.mark.parametrize("name,n_sample", [("replay", 192), ("shard", 48), ("prefill", 32)])
def test_full_size_forward_sampled(A, orc, name, n_sample):
    from oracle import layer as OL
    from moe_expert_layer_replay_b200 import layer
    from moe_expert_layer_replay_b200.inputs import make_inputs
    inp = make_inputs(name, seed=0)
    wl = inp["workload"]
    d = A.dims(wl.T, wl.D, wl.I, wl.E, wl.k)
    W = layer.quantise_weights(d, dev(inp["W_gate"]), dev(inp["W_up"]), dev(inp["W_down"]), train=False)
    B = layer.Buffers(d, "cuda", train=False)
    h = torch.empty(B.R_cap, wl.I, dtype=torch.bfloat16, device="cuda")
    lay = wl.L - 1
    if "payload" in inp:
        layer.route(B, payload=dev(inp["payload"]), layer=lay, w_in=dev(inp["w_in"][lay]))
        idx, w, st = orc.route_replay(inp["payload"], lay, wl.E, w_in=inp["w_in"][lay])
        assert st == 0
    else:
        layer.route(B, logits=dev(inp["logits"]))
        idx, w = orc.route_topk(inp["logits"], wl.k)
    layer.forward(B, dev(inp["x"]), W, h_out=h)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    same_bits(host(B.idx), idx, "idx (all tokens)")
    if "payload" in inp:
        same_bits(host(B.w), w, "w (all tokens)")
    else:
        np.testing.assert_allclose(host(B.w), w, rtol=2e-6, atol=1e-7)
    oc, oo, op, osrc = orc.permute(idx, wl.E, 128, B.R_cap)
    same_bits(host(B.counts), oc, "counts")
    same_bits(host(B.offsets), oo, "offsets")
    same_bits(host(B.pos), op, "pos")
    same_bits(host(B.src), osrc, "src_idx")
    if name == "prefill":
        assert np.sum(oc == 0) == 4 and oc.max() > 3 * oc.mean()   # skewed, with empty experts

    rng = np.random.default_rng(1)
    sample = np.sort(rng.choice(wl.T, n_sample, replace=False))
    wq = (OL.quant_weights(inp["W_gate"]), OL.quant_weights(inp["W_up"]), OL.quant_weights(inp["W_down"]))
    ref = OL.forward_tokens(inp["x"], idx, w, wq, sample)
    rows = ref["rows"].reshape(-1)
    xq, xs = host(B.xq[rows]), host(B.xs[:, rows]).T
    xr = np.repeat(inp["x"][sample], wl.k, axis=0)
    oq, os_ = orc.quant_block(xr, 1, 128)
    same_bits(xq, oq, "dispatched codes (sample)")
    same_bits(xs, os_, "dispatched scales (sample)")
    hg = host(h[rows])
    close(bf(hg), bf(ref["h"]), bf16=True, what="h (sample)")
    hq_ref, hs_ref = orc.quant_block(hg, 1, 128)
    same_bits(host(B.hq[rows]), hq_ref, "hq = quant(h) (sample)")
    same_bits(host(B.hs[:, rows]).T, hs_ref, "hs = quant(h) (sample)")
    expert = OL.expert_of_rows(oo, rows)
    Y_ref = OL.down_rows(host(B.hq[rows]), host(B.hs[:, rows]).T.copy(), expert, wq[2])
    close(bf(host(B.Y[rows])), bf(Y_ref), bf16=True, what="Y from the GPU's hq (sample)")
    close(bf(host(B.y[sample])), bf(ref["y"]), bf16=True, max_abs_rms=MAX_ABS_RMS_E2E, what="y end to end (sample)")


def test_full_size_train_sampled(A, orc):
    """The training workload (fwd + bwd, replayed routing, trainer logits) at
    full size: routing/permutation bit-exact over all tokens; per-step float
    outputs on sampled rows, tokens and dW blocks, from the GPU's own upstream
    operands (bit-exact where the contract says so)."""
    from oracle import layer as OL
    from moe_expert_layer_replay_b200 import layer
    from moe_expert_layer_replay_b200.inputs import make_inputs
    inp = make_inputs("train", seed=0)
    wl = inp["workload"]
    T, D, I, E, k = wl.T, wl.D, wl.I, wl.E, wl.k
    d = A.dims(T, D, I, E, k)
    W = layer.quantise_weights(d, dev(inp["W_gate"]), dev(inp["W_up"]), dev(inp["W_down"]), train=True)
    B = layer.Buffers(d, "cuda", train=True)
    z = inp["logits"]
    layer.route(B, payload=dev(inp["payload"]), layer=0, logits=dev(z))
    layer.forward(B, dev(inp["x"]), W)
    layer.backward(B, dev(inp["dy"]), W, router_logits=True)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    idx, w, st = orc.route_replay(inp["payload"], 0, E, z=z)
    assert st == 0
    same_bits(host(B.idx), idx, "idx")
    assert not np.array_equal(idx, np.argsort(-z, axis=1, kind="stable")[:, :k])  # replay overrides
    np.testing.assert_allclose(host(B.w), w, rtol=2e-6, atol=1e-7)
    oc, oo, op, osrc = orc.permute(idx, E, 128, B.R_cap)
    same_bits(host(B.offsets), oo, "offsets")
    same_bits(host(B.pos), op, "pos")
    rng = np.random.default_rng(3)
    gw = host(B.w)
    # ---- forward rows and combine on a sample of tokens
    sample = np.sort(rng.choice(T, 24, replace=False))
    rows = op[sample].reshape(-1)
    expert = OL.expert_of_rows(oo, rows)
    wq = (OL.quant_weights(inp["W_gate"]), OL.quant_weights(inp["W_up"]), OL.quant_weights(inp["W_down"]))
    g, u = OL.gateup_rows(host(B.xq[rows]), host(B.xs[:, rows]).T.copy(), expert, wq[0], wq[1])
    gu = host(B.gu[rows])
    blk = lambda a, o: np.concatenate([a[:, 256 * b + o:256 * b + o + 128] for b in range(I // 128)], axis=1)
    close(bf(blk(gu, 0)), bf(orc.bf16_round(g)), bf16=True, what="g (sample)")
    close(bf(blk(gu, 128)), bf(orc.bf16_round(u)), bf16=True, what="u (sample)")
    # ---- b1 over all tokens: dY rows bit-exact, d_w and d_logits
    dYr = OL.scaled_rows(inp["dy"][sample], gw[sample], np.arange(len(rows)).reshape(-1, k), len(rows))
    same_bits(host(B.dYb[rows]), dYr, "dY rows (sample)")
    q_ref, s_ref = orc.quant_block(dYr, 1, 128)
    same_bits(host(B.dYq[rows]), q_ref, "dYq (sample)")
    Yg = bf(host(B.Y[rows])).reshape(len(sample), k, D)
    dw_ref, dz_ref = OL.router_grads(inp["dy"][sample], Yg, gw[sample], z[sample], idx[sample])
    close(host(B.d_w[sample]), dw_ref, what="d_w (sample)")
    close(host(B.d_logits[sample]), dz_ref, what="d_logits (sample)")
    # ---- b2 on the GPU's dY codes
    dH = OL.dgrad_down(host(B.dYq[rows]), host(B.dYs[:, rows]).T.copy(), expert, wq[2])
    dG_ref, dU_ref = OL.swiglu_bwd(dH, blk(gu, 0), blk(gu, 128))
    dGU = host(B.dGU[rows])
    close(bf(blk(dGU, 0)), bf(dG_ref), bf16=True, what="dG (sample)")
    close(bf(blk(dGU, 128)), bf(dU_ref), bf16=True, what="dU (sample)")
    q_ref, s_ref = orc.quant_block(dGU, 1, 128)
    same_bits(host(B.dGUq[rows]), q_ref, "dGUq = quant(dGU) (sample)")
    # ---- b3 on the GPU's dGU codes, then the reduce of the sampled tokens
    dGUq, dGUs = host(B.dGUq[rows]), host(B.dGUs[:, rows]).T
    dX_ref = OL.dgrad_gateup(blk(dGUq, 0), dGUs[:, 0::2].copy(), blk(dGUq, 128), dGUs[:, 1::2].copy(),
                             expert, wq[0], wq[1])
    close(bf(host(B.dX[rows])), bf(dX_ref), bf16=True, what="dX (sample)")
    dx_ref = OL.unpermute_reduce(bf(host(B.dX[rows])), np.arange(len(rows)).reshape(-1, k))
    close(bf(host(B.dx[sample])), bf(dx_ref), bf16=True, what="dx (sample)")
    # ---- b4: two 128x128 blocks of each weight gradient for two experts, full K
    for e in rng.choice(E, 2, replace=False):
        r0, r1 = int(oo[e]), int(oo[e + 1])
        for (m0, n0) in [(0, 0), (128 * int(rng.integers(1, D // 128)), 128 * int(rng.integers(1, I // 128)))]:
            A_q = host(B.dYqT[m0:m0 + 128, r0:r1]).T.copy()
            A_s = host(B.dYsT[r0 // 128:r1 // 128, m0:m0 + 128])
            B_q = host(B.hqT[n0:n0 + 128, r0:r1]).T.copy()
            B_s = host(B.hsT[r0 // 128:r1 // 128, n0:n0 + 128])
            ref = OL.wgrad_expert(A_q, A_s, B_q, B_s, 0, r1 - r0)
            close(host(B.dWd[e, m0:m0 + 128, n0:n0 + 128]), ref, what=f"dW_down[{e}] block")
        n0 = 128 * int(rng.integers(0, D // 128))
        A_q = host(B.dGUqT[0:128, r0:r1]).T.copy()
        A_s = host(B.dGUsT[r0 // 128:r1 // 128, 0:128])
        B_q = host(B.xqT[n0:n0 + 128, r0:r1]).T.copy()
        B_s = host(B.xsT[r0 // 128:r1 // 128, n0:n0 + 128])
        close(host(B.dWgu[e, 0:128, n0:n0 + 128]), OL.wgrad_expert(A_q, A_s, B_q, B_s, 0, r1 - r0),
              what=f"dW_gate_up[{e}] block")
