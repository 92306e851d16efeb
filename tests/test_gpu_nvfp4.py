"""NVFP4 block quantisation on the GPU (moe_quant_nvfp4) against the oracle's
rule, bit for bit: packed e2m1 codes, e4m3 block scales, tensor amax and
scale ("RL at 1T scale: prime-rl performance deep dive", §Future work: NVFP4
on Blackwell)."""
import numpy as np
import pytest
import torch

from _util import dev, host, same_bits

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
