"""GATEUP_SILU with its A operand gathered from the token rows
(moe_gateup_gather_fp8: TMA tile::gather4 and cp.async) against the dispatched path
(moe_permute's FP8 dispatch, then moe_grouped_gemm_fp8): the A tile holds the
same bytes either way (1x128 quantisation is row-local, so a dispatched row
is its token's row), so h, its codes and scales must be bit-identical; and
both against the oracle.  The gather drops the R x D permuted FP8 copy that
every layer's dispatch otherwise writes ("prime-rl 0.6.0 løfter
trillion-parameter RL ...", §Drift og omkostninger i realiteten: the
dispatch/combine cost of every layer)."""
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


CASES = {  # T, D, I, E, k, zipf (>= 2: three empty experts)
    "tiny": (256, 256, 128, 8, 2, 0.0),
    "ragged_multi_tile": (1000, 512, 384, 8, 4, 1.0),
    "skew_empty": (700, 256, 256, 16, 4, 2.0),
    "replay_shape": (4096, 2048, 1024, 64, 6, 1.1),
}


@pytest.mark.parametrize("case", list(CASES))
def test_gateup_gather_equals_dispatched(A, orc, case):
    from oracle import layer as OL
    from moe_expert_layer_replay_b200 import layer
    T, D, I, E, k, zipf = CASES[case]
    rng = np.random.default_rng(300 + T)
    p = np.arange(1, E + 1, dtype=np.float64) ** -zipf
    if zipf >= 2.0:
        p[-3:] = 0.0
    with np.errstate(divide="ignore"):
        z = (np.log(p / p.sum())[None, :] - np.log(-np.log(rng.random((T, E))))).astype(np.float32)
    x = rand_bf16(rng, (T, D))
    Wg, Wu, Wd = rand_bf16(rng, (E, I, D), 0.02), rand_bf16(rng, (E, I, D), 0.02), rand_bf16(rng, (E, D, I), 0.02)
    d = A.dims(T, D, I, E, k)
    W = layer.quantise_weights(d, dev(Wg), dev(Wu), dev(Wd), train=False)
    B = layer.Buffers(d, "cuda", train=False)
    xd = dev(x)
    layer.route(B, logits=dev(z))
    R = B.R_cap
    # dispatched path
    A.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, xd, B.xq, B.xs, None, None, B.ws)
    h1 = torch.zeros(R, I, dtype=torch.bfloat16, device="cuda")
    A.grouped_gemm_fp8(A.GEMM_GATEUP_SILU, d, B.offsets, B.xq, B.xs, W.wgu_q, W.wgu_s, out_q=B.hq, out_s=B.hs,
                       out_bf16=h1)
    torch.cuda.synchronize()
    hq1, hs1 = host(B.hq), host(B.hs)
    # gathered path: token-row quantisation + index-only permute + gathered GEMM
    xq_tok = torch.empty(T, D, dtype=torch.uint8, device="cuda")
    xs_tok = torch.empty(D // 128, T, dtype=torch.float32, device="cuda")
    A.quant_fp8_block(xd, T, D, D, 1, 128, xq_tok, xs_tok)
    A.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, None, None, None, None, None, B.ws)
    hq2 = torch.full((R, I), 0x7F, dtype=torch.uint8, device="cuda")
    hs2 = torch.full((I // 128, R), -1.0, dtype=torch.float32, device="cuda")
    h2 = torch.zeros(R, I, dtype=torch.bfloat16, device="cuda")
    A.gateup_gather_fp8(d, B.offsets, B.src, xq_tok, xs_tok, W.wgu_q, W.wgu_s, out_q=hq2, out_s=hs2, out_bf16=h2)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    Rp = int(host(B.offsets)[E])
    same_bits(host(h2)[:Rp], host(h1)[:Rp], "h (gathered vs dispatched)")
    same_bits(host(hq2)[:Rp], hq1[:Rp], "hq (gathered vs dispatched)")
    same_bits(host(hs2)[:, :Rp], hs1[:, :Rp], "hs (gathered vs dispatched)")
    # the token-row codes are the oracle's, and the gathered h is the oracle's
    q_ref, s_ref = orc.quant_block(x, 1, 128)
    same_bits(host(xq_tok), q_ref, "token-row codes")
    same_bits(host(xs_tok).T, s_ref, "token-row scales")
    idx, w = orc.route_topk(z, k)
    fw = OL.forward(x, idx, w, Wg, Wu, Wd)
    close(bf(host(h2)[:Rp]), bf(fw["h"]), bf16=True, what="h (gathered) vs oracle")


def test_layer_forward_backward_gathered_equals_copy(A):
    """The whole layer, forward and backward, with Buffers(gather=True): the
    same outputs and gradients, bit for bit, as the permuted-copy path."""
    from moe_expert_layer_replay_b200 import layer
    rng = np.random.default_rng(320)
    T, D, I, E, k = 700, 512, 256, 8, 3
    z = rng.standard_normal((T, E)).astype(np.float32)
    x = rand_bf16(rng, (T, D))
    Wg, Wu, Wd = rand_bf16(rng, (E, I, D), 0.02), rand_bf16(rng, (E, I, D), 0.02), rand_bf16(rng, (E, D, I), 0.02)
    dy = rand_bf16(rng, (T, D), 0.01)
    d = A.dims(T, D, I, E, k)
    outs = []
    for gather in (False, True):
        W = layer.quantise_weights(d, dev(Wg), dev(Wu), dev(Wd), train=True)
        B = layer.Buffers(d, "cuda", train=True, gather=gather)
        layer.route(B, logits=dev(z))
        layer.forward(B, dev(x), W)
        layer.backward(B, dev(dy), W, router_logits=True)
        torch.cuda.synchronize()
        assert A.get_status() == A.OK
        Rp = int(host(B.offsets)[E])   # rows past the last segment are never written
        o = {n: host(getattr(B, n)) for n in ("y", "dx", "d_w", "d_logits", "dWd", "dWgu")}
        o.update(hq=host(B.hq)[:Rp], h=host(B.h)[:Rp], hs=host(B.hs)[:, :Rp])
        outs.append(o)
    for n in outs[0]:
        same_bits(outs[1][n], outs[0][n], f"{n} (gathered vs copy)")
