"""Parity of the grouped FP8 GEMMs and of the whole layer (forward and
backward) against the oracle, through the C ABI.

Each GEMM is checked against the oracle's step run on the same inputs (the
GPU's own upstream FP8 operands, which are bit-exact where the contract says
so); the whole layer is also checked end to end against the oracle run from
the raw inputs alone.
"""
import numpy as np
import pytest
import torch

from _util import MAX_ABS_RMS_E2E, bf, close, dev, host, rand_bf16, same_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from moe_expert_layer_replay_b200 import abi, build
    build.build()
    abi.lib()
    return abi


CASES = {
    # name: T, D, I, E, k, zipf, train
    "tiny": (256, 256, 128, 8, 2, 0.0, True),
    "multi_tile": (1024, 512, 256, 8, 4, 1.0, True),
    "ragged_n": (600, 384, 384, 6, 3, 1.5, True),
    "skew_empty": (512, 256, 256, 16, 4, 2.0, False),
    # training with three empty experts among skewed ones: wgrad skips their
    # tiles (no K blocks) and must leave their dW blocks untouched
    "skew_empty_train": (512, 256, 384, 16, 4, 2.0, True),
}
# one fixed seed per case (a new case takes the next number; the others keep theirs)
SEEDS = {"multi_tile": 11, "ragged_n": 12, "skew_empty": 13, "tiny": 14, "skew_empty_train": 15}


def _inputs(T, D, I, E, k, zipf, seed):
    rng = np.random.default_rng(seed)
    p = np.arange(1, E + 1, dtype=np.float64) ** -zipf
    if zipf >= 2.0:
        p[-3:] = 0  # empty experts
    z = (np.log(p / p.sum() + 1e-300)[None, :] - np.log(-np.log(rng.random((T, E))))).astype(np.float32)
    x = rand_bf16(rng, (T, D))
    Wg = rand_bf16(rng, (E, I, D), 0.02)
    Wu = rand_bf16(rng, (E, I, D), 0.02)
    Wd = rand_bf16(rng, (E, D, I), 0.02)
    dy = rand_bf16(rng, (T, D), 0.01)
    return z, x, Wg, Wu, Wd, dy


def _run_gpu(A, T, D, I, E, k, z, x, Wg, Wu, Wd, dy, train):
    from moe_expert_layer_replay_b200 import layer
    d = A.dims(T, D, I, E, k)
    W = layer.quantise_weights(d, dev(Wg), dev(Wu), dev(Wd), train=train)
    B = layer.Buffers(d, "cuda", train=train)
    h_out = None if train else torch.empty(B.R_cap, I, dtype=torch.bfloat16, device="cuda")
    layer.route(B, logits=dev(z))
    layer.forward(B, dev(x), W, h_out=h_out)
    if train:
        layer.backward(B, dev(dy), W, router_logits=True)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    return d, W, B, (B.h if train else h_out)


@pytest.mark.parametrize("case", list(CASES))
def test_layer_parity(A, orc, case):
    from oracle import layer as OL
    T, D, I, E, k, zipf, train = CASES[case]
    z, x, Wg, Wu, Wd, dy = _inputs(T, D, I, E, k, zipf, seed=SEEDS[case])
    d, W, B, h_gpu = _run_gpu(A, T, D, I, E, k, z, x, Wg, Wu, Wd, dy, train)

    # ---- oracle, end to end from the raw inputs
    idx, w = orc.route_topk(z, k)
    same_bits(host(B.idx), idx, "idx")
    fw = OL.forward(x, idx, w, Wg, Wu, Wd)
    Rp = int(fw["offsets"][E])
    same_bits(host(B.offsets), fw["offsets"], "offsets")
    same_bits(host(B.pos), fw["pos"], "pos")
    same_bits(host(B.xq)[:Rp], fw["xq"], "xq")
    same_bits(host(B.xs)[:, :Rp].T, fw["xs"], "xs")
    close(bf(host(B.y)), bf(fw["y"]), bf16=True, max_abs_rms=MAX_ABS_RMS_E2E, what="y end to end")

    # ---- GEMM1 step on the same (bit-exact) operands
    hg = host(h_gpu)[:Rp]
    close(bf(hg), bf(fw["h"]), bf16=True, what="h")
    hq_ref, hs_ref = orc.quant_block(hg, 1, 128)          # the fused h-quantiser
    same_bits(host(B.hq)[:Rp], hq_ref, "hq = quant(h)")
    same_bits(host(B.hs)[:, :Rp].T, hs_ref, "hs = quant(h)")
    if train:
        gu = host(B.gu)[:Rp]
        gi = np.concatenate([gu[:, 256 * b:256 * b + 128] for b in range(I // 128)], axis=1)
        ui = np.concatenate([gu[:, 256 * b + 128:256 * b + 256] for b in range(I // 128)], axis=1)
        close(bf(gi), bf(fw["g_b"]), bf16=True, what="g")
        close(bf(ui), bf(fw["u_b"]), bf16=True, what="u")

    # ---- GEMM2 step on the GPU's hq
    Wq = fw["Wq"]
    Y_ref = OL.down_rows(host(B.hq)[:Rp], host(B.hs)[:, :Rp].T.copy(), fw["expert"], Wq[2])
    close(bf(host(B.Y)[:Rp]), bf(Y_ref), bf16=True, what="Y")

    if not train:
        return
    bw = OL.backward(fw, x, dy, idx, w, z=z)
    dWd = host(B.dWd)
    dWgu = host(B.dWgu)

    # ---- backward steps on the GPU's own upstream operands
    expert = fw["expert"]
    # dY rows from the GPU's own routing weights (the same inputs): bit-exact
    dYr = OL.scaled_rows(dy, host(B.w), fw["pos"], Rp)
    same_bits(host(B.dYb)[:Rp], dYr, "dY rows")
    dYq_ref, dYs_ref = orc.quant_block(dYr, 1, 128)
    same_bits(host(B.dYq)[:Rp], dYq_ref, "dYq")
    same_bits(host(B.dYs)[:, :Rp].T, dYs_ref, "dYs")
    dH = OL.dgrad_down(host(B.dYq)[:Rp], host(B.dYs)[:, :Rp].T.copy(), expert, Wq[2])
    gu = host(B.gu)[:Rp]
    g_b = np.concatenate([gu[:, 256 * b:256 * b + 128] for b in range(I // 128)], axis=1)
    u_b = np.concatenate([gu[:, 256 * b + 128:256 * b + 256] for b in range(I // 128)], axis=1)
    dG_ref, dU_ref = OL.swiglu_bwd(dH, g_b, u_b)
    dGU = host(B.dGU)[:Rp]
    dG = np.concatenate([dGU[:, 256 * b:256 * b + 128] for b in range(I // 128)], axis=1)
    dU = np.concatenate([dGU[:, 256 * b + 128:256 * b + 256] for b in range(I // 128)], axis=1)
    close(bf(dG), bf(dG_ref), bf16=True, what="dG")
    close(bf(dU), bf(dU_ref), bf16=True, what="dU")
    q_ref, s_ref = orc.quant_block(dGU, 1, 128)     # the fused d[g|u] quantiser
    same_bits(host(B.dGUq)[:Rp], q_ref, "dGUq = quant(dGU)")
    same_bits(host(B.dGUs)[:, :Rp].T, s_ref, "dGUs = quant(dGU)")
    qT_ref, sT_ref = orc.quant_block(dGU, 128, 1)
    same_bits(host(B.dGUqT)[:, :Rp].T, qT_ref, "dGU 128x1 codes")
    same_bits(host(B.dGUsT)[:Rp // 128], sT_ref, "dGU 128x1 scales")
    # b3 on the GPU's dGU codes
    dGq = np.concatenate([host(B.dGUq)[:Rp, 256 * b:256 * b + 128] for b in range(I // 128)], axis=1)
    dUq = np.concatenate([host(B.dGUq)[:Rp, 256 * b + 128:256 * b + 256] for b in range(I // 128)], axis=1)
    dGUs = host(B.dGUs)[:, :Rp].T
    dGs = dGUs[:, 0::2].copy()
    dUs = dGUs[:, 1::2].copy()
    dX_ref = OL.dgrad_gateup(dGq, dGs, dUq, dUs, expert, Wq[0], Wq[1])
    close(bf(host(B.dX)[:Rp]), bf(dX_ref), bf16=True, what="dX")
    # b4 on the GPU's 128x1 operands
    hqT, hsT = host(B.hqT)[:, :Rp].T.copy(), host(B.hsT)[:Rp // 128]
    same_bits((hqT, hsT)[0], orc.quant_block(host(B.h)[:Rp], 128, 1)[0], "h 128x1 codes")
    dYqT, dYsT = host(B.dYqT)[:, :Rp].T.copy(), host(B.dYsT)[:Rp // 128]
    dYqT_ref, dYsT_ref = orc.quant_block(dYr, 128, 1)
    same_bits(dYqT, dYqT_ref, "dY 128x1 codes")
    same_bits(dYsT, dYsT_ref, "dY 128x1 scales")
    xqT, xsT = host(B.xqT)[:, :Rp].T.copy(), host(B.xsT)[:Rp // 128]
    offs = fw["offsets"]
    for e in range(E):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        if r0 == r1:   # an empty expert: its dW blocks stay as they were (zeros here)
            assert np.all(dWd[e] == 0) and np.all(dWgu[e] == 0), f"empty expert {e}"
            continue
        close(dWd[e], OL.wgrad_expert(dYqT, dYsT, hqT, hsT, r0, r1), what=f"dW_down[{e}]")
        close(dWgu[e], OL.wgrad_expert(host(B.dGUqT)[:, :Rp].T.copy(), host(B.dGUsT)[:Rp // 128],
                                       xqT, xsT, r0, r1), what=f"dW_gate_up[{e}]")

    # ---- backward, end to end from the raw inputs
    close(host(B.d_w), bw["d_w"], what="d_w")          # upstream of any re-quantisation
    close(host(B.d_logits), bw["dz"], what="d_logits")
    e2e = dict(max_abs_rms=MAX_ABS_RMS_E2E)
    close(bf(host(B.dx)), bf(bw["dx"]), bf16=True, what="dx end to end", **e2e)
    dWg = np.concatenate([dWgu[:, 256 * b:256 * b + 128] for b in range(I // 128)], axis=1)
    dWu = np.concatenate([dWgu[:, 256 * b + 128:256 * b + 256] for b in range(I // 128)], axis=1)
    close(dWd, bw["dWd"], what="dW_down end to end", **e2e)
    close(dWg, bw["dWg"], what="dW_gate end to end", **e2e)
    close(dWu, bw["dWu"], what="dW_up end to end", **e2e)


def test_layer_deterministic(A):
    T, D, I, E, k, zipf, train = CASES["multi_tile"]
    z, x, Wg, Wu, Wd, dy = _inputs(T, D, I, E, k, zipf, seed=5)
    outs = []
    for _ in range(2):
        d, W, B, h = _run_gpu(A, T, D, I, E, k, z, x, Wg, Wu, Wd, dy, train)
        Rp = int(host(B.offsets)[E])  # rows past the last segment are never written
        outs.append([host(t) for t in (B.y, B.dx, B.d_w, B.d_logits, B.dWd, B.dWgu)]
                    + [host(B.hq)[:Rp], host(B.dGUq)[:Rp], host(B.Y)[:Rp], host(B.dX)[:Rp]])
    for a, b in zip(*outs):
        same_bits(a, b, "repeat run")


def test_wgrad_accumulates(A):
    """dW += : a second backward adds the same gradient again."""
    T, D, I, E, k, zipf, train = CASES["tiny"]
    z, x, Wg, Wu, Wd, dy = _inputs(T, D, I, E, k, zipf, seed=6)
    from moe_expert_layer_replay_b200 import layer
    d, W, B, h = _run_gpu(A, T, D, I, E, k, z, x, Wg, Wu, Wd, dy, train)
    once = host(B.dWd).copy()
    layer.backward(B, dev(dy), W, router_logits=True)
    torch.cuda.synchronize()
    np.testing.assert_allclose(host(B.dWd), 2 * once, rtol=1e-6, atol=1e-12)


def test_wait_budget_timeout_is_reported_and_recoverable(A):
    """A wait budget too small for any real wait makes the GEMM's bounded
    waits run out: the kernel latches MOE_ERR_TIMEOUT, drains its own copies
    and MMAs, frees its tensor memory and returns; the context stays usable
    and the next run with the default budget is correct."""
    from moe_expert_layer_replay_b200 import layer
    T, D, I, E, k, zipf, train = CASES["multi_tile"]
    z, x, Wg, Wu, Wd, dy = _inputs(T, D, I, E, k, zipf, seed=8)
    d, W, B, h = _run_gpu(A, T, D, I, E, k, z, x, Wg, Wu, Wd, dy, False)
    ref_hq = host(B.hq).copy()
    Rp = int(host(B.offsets)[E])
    try:
        A.set_wait_budget(1)
        A.grouped_gemm_fp8(A.GEMM_GATEUP_SILU, d, B.offsets, B.xq, B.xs, W.wgu_q, W.wgu_s,
                           out_q=B.hq, out_s=B.hs)
        st = A.get_status()
    finally:
        A.set_wait_budget(0)
    assert st == A.TIMEOUT, A.strerror(st)
    A.grouped_gemm_fp8(A.GEMM_GATEUP_SILU, d, B.offsets, B.xq, B.xs, W.wgu_q, W.wgu_s, out_q=B.hq, out_s=B.hs)
    assert A.get_status() == A.OK
    same_bits(host(B.hq)[:Rp], ref_hq[:Rp], "after a timed-out run")


def test_empty_batch_forward_backward(A):
    """T = 0 through the whole layer, top-k and replay routing alike: every
    entry point returns OK, the outputs are empty, all segments are empty and
    the weight gradients are untouched."""
    from moe_expert_layer_replay_b200 import layer
    T, D, I, E, k = 0, 256, 128, 8, 2
    d = A.dims(T, D, I, E, k)
    rng = np.random.default_rng(5)
    W = layer.quantise_weights(d, dev(rand_bf16(rng, (E, I, D), 0.02)), dev(rand_bf16(rng, (E, I, D), 0.02)),
                               dev(rand_bf16(rng, (E, D, I), 0.02)), train=True)
    B = layer.Buffers(d, "cuda", train=True)
    layer.route(B, logits=torch.empty(0, E, device="cuda"))
    layer.route(B, payload=torch.empty(1, k, 0, dtype=torch.int32, device="cuda"), layer=0,
                w_in=torch.empty(0, k, device="cuda"))
    y = layer.forward(B, torch.empty(0, D, dtype=torch.bfloat16, device="cuda"), W)
    dx, d_w, dz = layer.backward(B, torch.empty(0, D, dtype=torch.bfloat16, device="cuda"), W, router_logits=True)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    assert y.shape == (0, D) and dx.shape == (0, D) and d_w.shape == (0, k) and dz.shape == (0, E)
    assert int(B.counts.abs().sum()) == 0 and int(B.offsets.abs().sum()) == 0
    assert int(torch.count_nonzero(B.dWd)) == 0 and int(torch.count_nonzero(B.dWgu)) == 0
