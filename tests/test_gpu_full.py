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
