"""The 2-SM MMA variant of the rows-mode grouped GEMMs (tcgen05.mma
cta_group::2: a pair of SMs per 256-row x 256-column tile, each CTA loading
its own 128 rows of A and half of the weight tile, each K block issued as two
128-column halves) against the one-SM kernel:
bit-identical h codes, scales, Y, d[g|u] and dX on the same operands (the two
compute the same K-block partial products and promote them in the same
order), including segments with an odd number of 128-row tiles (the idle half
of their last pair writes nothing), empty segments and the segment-grouped
(expert-parallel) form."""
import numpy as np
import pytest
import torch

from _util import dev, host, rand_bf16, same_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from moe_expert_layer_replay_b200 import abi, build
    build.build()
    abi.lib()
    yield abi
    abi.set_gemm_variant(0)


CASES = {  # T, D, I, E, k, zipf (>= 2: three empty experts), train
    "tiny": (256, 256, 128, 8, 2, 0.0, True),
    "odd_tiles_ragged": (1000, 512, 384, 8, 4, 1.0, True),
    "skew_empty": (700, 256, 256, 16, 4, 2.0, False),
    "shard_shape": (2048, 7168, 2048, 32, 8, 0.0, False),
    "ragged_model_dim": (600, 384, 256, 8, 2, 0.5, True),   # a 128-column last tile in DOWN / DGRAD_GATEUP
}
VARIANTS = [1]


def _run(A, variant, T, D, I, E, k, z, x, Wg, Wu, Wd, dy, train):
    from moe_expert_layer_replay_b200 import layer
    A.set_gemm_variant(variant)
    d = A.dims(T, D, I, E, k)
    W = layer.quantise_weights(d, dev(Wg), dev(Wu), dev(Wd), train=train)
    B = layer.Buffers(d, "cuda", train=train)
    h = None if train else torch.zeros(B.R_cap, I, dtype=torch.bfloat16, device="cuda")
    layer.route(B, logits=dev(z))
    layer.forward(B, dev(x), W, h_out=h)
    if train:
        layer.backward(B, dev(dy), W, router_logits=True)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    Rp = int(host(B.offsets)[E])
    out = {"hq": host(B.hq)[:Rp], "hs": host(B.hs)[:, :Rp], "Y": host(B.Y)[:Rp], "y": host(B.y)}
    if train:
        out.update(gu=host(B.gu)[:Rp], dGU=host(B.dGU)[:Rp], dGUq=host(B.dGUq)[:Rp], dX=host(B.dX)[:Rp],
                   dx=host(B.dx))
    else:
        out["h"] = host(h)[:Rp]
    return out


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("case", list(CASES))
def test_pair_variant_equals_one_sm(A, case, variant):
    T, D, I, E, k, zipf, train = CASES[case]
    rng = np.random.default_rng(400 + T)
    p = np.arange(1, E + 1, dtype=np.float64) ** -zipf
    if zipf >= 2.0:
        p[-3:] = 0.0
    with np.errstate(divide="ignore"):
        z = (np.log(p / p.sum())[None, :] - np.log(-np.log(rng.random((T, E))))).astype(np.float32)
    x = rand_bf16(rng, (T, D))
    Wg, Wu, Wd = rand_bf16(rng, (E, I, D), 0.02), rand_bf16(rng, (E, I, D), 0.02), rand_bf16(rng, (E, D, I), 0.02)
    dy = rand_bf16(rng, (T, D), 0.01)
    one = _run(A, 0, T, D, I, E, k, z, x, Wg, Wu, Wd, dy, train)
    two = _run(A, variant, T, D, I, E, k, z, x, Wg, Wu, Wd, dy, train)
    for name in one:
        same_bits(two[name], one[name], f"{name} (variant {variant} vs 1-SM)")


@pytest.mark.parametrize("variant", VARIANTS)
def test_pair_variant_segment_gemm(A, variant):
    """Segments of an expert-parallel receiver, odd tile counts included."""
    rng = np.random.default_rng(410)
    E_loc, n_seg, D, I = 4, 8, 512, 256
    cnt = np.array([300, 0, 129, 128, 5, 256, 0, 390])
    seg = (cnt + 127) // 128 * 128
    offs = np.concatenate([[0], np.cumsum(seg)]).astype(np.int32)
    rows_cap = int(offs[-1]) + 128
    from moe_expert_layer_replay_b200 import layer
    d = A.dims(16, D, I, E_loc, 2)
    Wg, Wu, Wd = rand_bf16(rng, (E_loc, I, D), 0.02), rand_bf16(rng, (E_loc, I, D), 0.02), rand_bf16(rng, (E_loc, D, I), 0.02)
    W = layer.quantise_weights(d, dev(Wg), dev(Wu), dev(Wd), train=False)
    xq = torch.from_numpy(rng.integers(0, 0x7F, (rows_cap, D), dtype=np.uint8)).cuda()
    xs = torch.from_numpy((rng.random((D // 128, rows_cap)) * 1e-2).astype(np.float32)).cuda()
    outs = []
    for v in (0, variant):
        A.set_gemm_variant(v)
        hq = torch.zeros(rows_cap, I, dtype=torch.uint8, device="cuda")
        hs = torch.zeros(I // 128, rows_cap, dtype=torch.float32, device="cuda")
        Y = torch.zeros(rows_cap, D, dtype=torch.bfloat16, device="cuda")
        A.grouped_gemm_fp8_seg(A.GEMM_GATEUP_SILU, d, rows_cap, dev(offs), n_seg, xq, xs, W.wgu_q, W.wgu_s,
                               out_q=hq, out_s=hs)
        A.grouped_gemm_fp8_seg(A.GEMM_DOWN, d, rows_cap, dev(offs), n_seg, hq, hs, W.wd_q, W.wd_s, out_bf16=Y)
        torch.cuda.synchronize()
        assert A.get_status() == A.OK
        outs.append((host(hq), host(hs), host(Y)))
    for a, b, name in zip(outs[0], outs[1], ["hq", "hs", "Y"]):
        same_bits(b, a, f"{name} (variant {variant} vs 1-SM, segments)")
