"""NVFP4 block quantisation and the NVFP4 expert GEMM in fp64 — TEST
INFRASTRUCTURE ONLY.

Source: "RL at 1T scale: prime-rl performance deep dive", §Future work: NVFP4
training and inference on Blackwell.  The pages name the format only; its
definition is NVIDIA's NVFP4: 4-bit e2m1 elements (magnitudes 0, 0.5, 1,
1.5, 2, 3, 4, 6) in blocks of 16 consecutive elements along a row, each block
with an e4m3 scale, and one fp32 scale per tensor.

Readings (every rounding point written out; the pages give none):

* tensor scale: amax_t = max |x| over the tensor (exact from bf16);
  s_g = fp32(2688 / amax_t) by IEEE fp32 division (2688 = 6 * 448, the
  largest e2m1 magnitude times the largest e4m3 value), s_g = 1 if amax_t = 0;
* block scale: amax_b = max |x| over the block; s_b = fp32(amax_b / 6);
  stored as S8 = e4m3(round to nearest even, saturate to 448)(fp32(s_b * s_g));
  S_b = the value of S8;
* codes: 0x0 if S_b = 0 (an all-zero block, or s_b * s_g below e4m3's
  smallest value), else e2m1(round to nearest even, saturate to +-6)(
  fp32(x * fp32(s_g / S_b))), the division and the product IEEE fp32; the
  sign of zero is kept (-0 -> code 8);
* value: x ~ e2m1(q) * S_b / s_g;
* NVFP4 GEMM: C[m, n] = sum over K of value(A)[m, k] * value(B)[n, k],
  accumulated here in fp64 (exact products; the tensor cores accumulate in
  fp32).
"""
from __future__ import annotations

import numpy as np

from . import e4m3_decode, e4m3_encode

E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
TENSOR_SCALE_NUM = np.float32(6.0 * 448.0)


def e2m1_encode(v) -> np.ndarray:
    """fp32 -> e2m1 codes (0..15, bit 3 = sign): the nearest magnitude, ties
    to the even code, values past 6 saturate to 6."""
    v = np.asarray(v, np.float32)
    a = np.abs(v).astype(np.float64)
    mags = np.array(E2M1_MAGNITUDES)
    d = np.abs(a[..., None] - mags)                     # distance to each magnitude
    best = d.min(axis=-1, keepdims=True)
    cand = d == best                                     # one or two nearest codes
    codes = np.arange(8)
    even = cand & (codes % 2 == 0)
    idx = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    idx = np.where(a > 6.0, 7, idx)
    sign = np.signbit(v).astype(np.int64) << 3
    return (idx | sign).astype(np.uint8)


def e2m1_decode(c) -> np.ndarray:
    c = np.asarray(c, np.uint8)
    mag = np.array(E2M1_MAGNITUDES)[c & 7]
    return np.where(c & 8, -mag, mag)


def tensor_scale(x_bf16) -> np.float32:
    """s_g = fp32(2688 / amax_t), 1 for an all-zero tensor."""
    from . import bf16_to_f64
    amax = np.float32(np.abs(bf16_to_f64(x_bf16)).max()) if np.size(x_bf16) else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(TENSOR_SCALE_NUM / amax)


def quant(x_bf16, s_g=None):
    """NVFP4 of a bf16 matrix [rows, cols] (cols % 16 == 0).

    Returns (codes uint8 [rows, cols] one code per element, S8 uint8
    [rows, cols/16] e4m3 block-scale codes, s_g float32)."""
    from . import bf16_to_f64
    x = bf16_to_f64(x_bf16).astype(np.float32)
    rows, cols = x.shape
    assert cols % 16 == 0
    s_g = tensor_scale(x_bf16) if s_g is None else np.float32(s_g)
    blocks = x.reshape(rows, cols // 16, 16)
    amax_b = np.abs(blocks).max(axis=-1)                                   # exact
    s_b = (amax_b / np.float32(6.0)).astype(np.float32)                    # IEEE fp32 division
    S8 = e4m3_encode((s_b * s_g).astype(np.float32))                       # fp32 product, RNE, saturate
    S_b = e4m3_decode(S8).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = np.where(S_b > 0, (s_g / S_b).astype(np.float32), np.float32(0.0)).astype(np.float32)
    q = (blocks * inv[..., None]).astype(np.float32)                       # IEEE fp32 product
    codes = e2m1_encode(q)
    codes = np.where((S_b > 0)[..., None], codes, np.uint8(0))   # a zero block scale: zero codes
    return codes.reshape(rows, cols).astype(np.uint8), S8, s_g


def dequant(codes, S8, s_g) -> np.ndarray:
    """fp64 values e2m1(q) * S_b / s_g (exact: a few significant bits each)."""
    rows, cols = codes.shape
    S_b = e4m3_decode(S8).astype(np.float64)
    return (e2m1_decode(codes).reshape(rows, cols // 16, 16) * S_b[..., None]).reshape(rows, cols) / np.float64(s_g)


def pack(codes) -> np.ndarray:
    """Two codes per byte along a row, element 2i in the low nibble."""
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack(packed) -> np.ndarray:
    p = np.asarray(packed, np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), np.uint8)
    out[:, 0::2] = p & 15
    out[:, 1::2] = p >> 4
    return out


def gemm(a_codes, a_S8, a_sg, b_codes, b_S8, b_sg) -> np.ndarray:
    """C [M, N] = value(A) value(B)^T in fp64 (A [M, K], B [N, K])."""
    from . import wgrad
    A = dequant(a_codes, a_S8, a_sg)
    B = dequant(b_codes, b_S8, b_sg)
    return wgrad(np.ascontiguousarray(A.T), np.ascontiguousarray(B.T))
