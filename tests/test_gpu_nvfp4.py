"""NVFP4 block quantisation on the GPU (moe_quant_nvfp4) against the oracle's
rule, bit for bit: packed e2m1 codes, e4m3 block scales, tensor amax and
scale ("RL at 1T scale: prime-rl performance deep dive", §Future work: NVFP4
on Blackwell)."""
import numpy as np
import pytest
import torch

from _util import close, dev, host, same_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from moe_expert_layer_replay_b200 import abi, build
    build.build()
    abi.lib()
    return abi


def _case(name, rng):
    from moe_expert_layer_replay_b200.inputs import to_bf16_bits
    if name == "normal_rows":
        x = rng.standard_normal((300, 2048)) * np.exp(rng.uniform(-8, 8, (300, 1)))
    elif name == "zero_blocks_and_tiny":
        x = rng.standard_normal((64, 512))
        x[5, 32:48] = 0
        x[7] *= 1e-30            # block scales below e4m3's range: zero codes
        x[9, :16] = [6, -3, 1.5, 0.75, 0.25, 0, 2, 4, -6, 1, 0.5, 3, -1.5, 0.125, 5, -0.5]
    elif name == "all_zero":
        x = np.zeros((16, 128))
    else:   # every bf16 bit pattern's magnitude class, scaled across blocks
        x = rng.standard_normal((128, 4096)) * 10.0 ** rng.integers(-20, 20, (128, 256)).repeat(16, axis=1)
    return to_bf16_bits(x.astype(np.float32))


@pytest.mark.parametrize("name", ["normal_rows", "zero_blocks_and_tiny", "all_zero", "wide_range"])
def test_quant_nvfp4_matches_oracle(A, orc, name):
    from oracle import nvfp4
    rng = np.random.default_rng(95)
    x = _case(name, rng)
    rows, cols = x.shape
    q = torch.full((rows, cols // 2), 0xAA, dtype=torch.uint8, device="cuda")
    sf = torch.full((rows, cols // 16), 0xAA, dtype=torch.uint8, device="cuda")
    amax = torch.full((1,), 123.0, device="cuda")
    s_g = torch.empty(1, device="cuda")
    A.quant_nvfp4(dev(x), rows, cols, cols, q, sf, amax, s_g)
    torch.cuda.synchronize()
    codes, S8, sg = nvfp4.quant(x)
    same_bits(host(amax), np.array([np.abs(orc.bf16_to_f64(x)).max()], np.float32), "tensor amax")
    same_bits(host(s_g), np.array([sg], np.float32), "tensor scale")
    same_bits(host(sf), S8, "e4m3 block scales")
    same_bits(host(q), nvfp4.pack(codes), "packed e2m1 codes")


def sf_mma_layout(S8, side):
    """[rows][cols/16] e4m3 scale codes -> the NVFP4 GEMM's A- or B-side layout
    as moe.h states it: 4096-byte blocks, each scale stored once per TMEM lane
    quarter; inside a block, lane l, half h, byte 4 r1 + j (row 32 r1 + l % 32
    of a 128-row block, group j of a 64-column step) at (l >> 3) * 256 + h * 128
    + (l & 7) * 16 + 4 r1 + j.  A: block (row block, step pair), h = step
    parity.  B: block (row-block pair, step), h = row-block parity."""
    rows, nb = S8.shape
    cols = nb * 16
    out = np.zeros(4 * rows * nb, np.uint8)
    r = np.arange(rows)[:, None]
    b = np.arange(nb)[None, :]
    rb, rr, ks, j = r >> 7, r & 127, b >> 2, b & 3
    if side == "A":
        blk, h = rb * (cols // 128) + (ks >> 1), ks & 1
    else:
        blk, h = (rb >> 1) * (cols // 64) + ks, rb & 1
    for q in range(4):
        lane = 32 * q + (rr & 31)
        off = blk * 4096 + (lane >> 3) * 256 + h * 128 + (lane & 7) * 16 + (rr >> 5) * 4 + j
        out[np.broadcast_to(off, S8.shape).ravel()] = S8.ravel()
    return out


@pytest.mark.parametrize("side", ["A", "B"])
def test_quant_nvfp4_mma_layout(A, orc, side):
    from oracle import nvfp4
    from moe_expert_layer_replay_b200.inputs import to_bf16_bits
    rng = np.random.default_rng(96)
    rows, cols = 512, 1024
    x = to_bf16_bits((rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-4, 4, (rows, 1)))).astype(np.float32))
    q = torch.empty(rows, cols // 2, dtype=torch.uint8, device="cuda")
    sf = torch.full((4 * rows * cols // 16,), 0xAA, dtype=torch.uint8, device="cuda")
    amax = torch.empty(1, device="cuda")
    s_g = torch.empty(1, device="cuda")
    layout = A.NVFP4_SF_MMA_A if side == "A" else A.NVFP4_SF_MMA_B
    A.quant_nvfp4(dev(x), rows, cols, cols, q, sf, amax, s_g, sf_layout=layout)
    torch.cuda.synchronize()
    codes, S8, sg = nvfp4.quant(x)
    same_bits(host(sf), sf_mma_layout(S8, side), f"e4m3 block scales, {side}-side MMA layout")
    same_bits(host(q), nvfp4.pack(codes), "packed e2m1 codes")
    same_bits(host(s_g), np.array([sg], np.float32), "tensor scale")
    with pytest.raises(A.MoeError):   # the MMA layouts need whole 128-row (A) / 256-row (B) blocks
        A.quant_nvfp4(dev(x[:200]), 200, cols, cols, q, sf, amax, s_g, sf_layout=layout)


# segment row counts (multiples of 128, 0 = an empty segment), N, K
GEMM_CASES = {
    "one_tile": ([128], 256, 256),
    "grouped_empty_segment": ([128, 0, 384], 512, 768),
    "ffn_shape": ([256, 512, 128, 384], 2048, 2048),
    "deep_k": ([256], 256, 7168),
    "many_tiles_per_sm": ([2048, 1024, 0, 2048], 2048, 512),   # 320 tiles: 2-3 per persistent CTA
}


@pytest.mark.parametrize("case", list(GEMM_CASES))
def test_gemm_nvfp4_matches_oracle(A, orc, case):
    """The NVFP4 grouped GEMM against the oracle's fp64 product of the
    dequantised operands (oracle.nvfp4.gemm), per segment.  Both sides use the
    same codes and scales (the GPU quantiser's, equal to the oracle's bit for
    bit by the tests above); each product of two NVFP4 values is exact in fp32
    (at most 12 significant bits), so the kernel differs from the oracle only
    by its fp32 accumulation order and the final scaling: a relative error of
    order 1e-7, checked at 1e-5 (Frobenius) and 1e-4 * rms (max-abs)."""
    from oracle import nvfp4
    counts, N, K = GEMM_CASES[case]
    E = len(counts)
    rng = np.random.default_rng(97 + N + K)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offs[-1]) + 128   # one spare row block past the last segment
    from moe_expert_layer_replay_b200.inputs import to_bf16_bits
    x = to_bf16_bits(rng.standard_normal((R, K)).astype(np.float32))
    x[offs[-1]:] = 0
    W = to_bf16_bits((rng.standard_normal((E, N, K)) * 0.02).astype(np.float32))
    aq = torch.empty(R, K // 2, dtype=torch.uint8, device="cuda")
    asf = torch.empty(4 * R * K // 16, dtype=torch.uint8, device="cuda")
    amax = torch.empty(1, device="cuda")
    a_sg = torch.empty(1, device="cuda")
    A.quant_nvfp4(dev(x), R, K, K, aq, asf, amax, a_sg, sf_layout=A.NVFP4_SF_MMA_A)
    bq = torch.empty(E, N, K // 2, dtype=torch.uint8, device="cuda")
    bsf = torch.empty(E, 4 * N * K // 16, dtype=torch.uint8, device="cuda")
    bamax = torch.empty(E, device="cuda")
    b_sg = torch.empty(E, device="cuda")
    Wd = dev(W)
    for e in range(E):
        A.quant_nvfp4(Wd[e], N, K, K, bq[e], bsf[e], bamax[e:e + 1], b_sg[e:e + 1], sf_layout=A.NVFP4_SF_MMA_B)
    out = torch.full((R, N), -7.0, dtype=torch.float32, device="cuda")
    A.gemm_nvfp4(R, N, K, E, dev(offs), aq, asf, a_sg, bq, bsf, b_sg, out)
    torch.cuda.synchronize()
    assert A.get_status() == A.OK
    got = host(out)
    ca, Sa, sga = nvfp4.quant(x)
    for e in range(E):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        if r1 == r0:
            continue
        cb, Sb, sgb = nvfp4.quant(W[e])
        ref = nvfp4.gemm(ca[r0:r1], Sa[r0:r1], sga, cb, Sb, sgb)
        close(got[r0:r1], ref, rel_fro=1e-5, max_abs_rms=1e-4, what=f"{case}: segment {e}")
    assert np.all(got[offs[-1]:] == -7.0), "rows past the last segment are untouched"
