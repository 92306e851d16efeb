"""CPU oracle of the MoE expert layer — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
(``moe_expert_layer_replay_b200``) and never imports it.

The heavy loops live in ``moe_oracle.c`` (plain C, fp64, OpenMP over
independent outputs); the layer is composed step by step in ``layer.py`` with
numpy fp64.  Readings of the pages that fix each rounding point are stated in
``moe_oracle.c`` and ``layer.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
          "-shared", "-fPIC", "-Wall"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.orc_bf16_from_double.restype = ctypes.c_uint16
        L.orc_bf16_from_double.argtypes = [ctypes.c_double]
        L.orc_e4m3_from_float.restype = ctypes.c_uint8
        L.orc_e4m3_from_float.argtypes = [ctypes.c_float]
        L.orc_e4m3_to_double.restype = ctypes.c_double
        L.orc_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.orc_bf16_round_array.argtypes = [P, I64, P]
        L.orc_e4m3_encode_array.argtypes = [P, I64, P]
        L.orc_e4m3_decode_array.argtypes = [P, I64, P]
        L.orc_quant_block.argtypes = [P, I64, I64, I64, I, I, P, P]
        L.orc_route_topk.argtypes = [P, I64, I, I, P, P]
        L.orc_route_replay.restype = I
        L.orc_route_replay.argtypes = [P, I, I, I64, I, I, P, P, P, P]
        L.orc_permute.argtypes = [P, I64, I, I, I, P, P, P, P, I64]
        L.orc_rowdot.argtypes = [P, I64, P, I, P, P, P, I64, I64, I, P]
        L.orc_wgrad.argtypes = [P, I64, I64, I64, P, I64, I64, I64, I64, P]
        L.orc_num_threads.restype = I
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# scalar codecs
# --------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """fp64 -> bf16 bits (uint16), round to nearest even, directly from fp64."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_bf16_round_array(_p(x), x.size, _p(out))
    return out


def bf16_to_f64(b) -> np.ndarray:
    b = np.asarray(b, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_encode(v) -> np.ndarray:
    """fp32 -> e4m3fn codes, round to nearest even, saturate to +-448."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode_array(_p(c), c.size, _p(out))
    return out


# --------------------------------------------------------------------------
# block quantisation (natural layouts)
# --------------------------------------------------------------------------

def quant_block(x_bf16, br: int, bc: int):
    """Block-scaled FP8 of a bf16 matrix [rows, cols].

    Returns (q uint8 [rows, cols], s float32 [ceil(rows/br), ceil(cols/bc)]).
    """
    x = _c(x_bf16, np.uint16)
    rows, cols = x.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty(((rows + br - 1) // br, (cols + bc - 1) // bc), np.float32)
    lib().orc_quant_block(_p(x), rows, cols, cols, br, bc, _p(q), _p(s))
    return q, s


def dequant_block(q, s, br: int, bc: int) -> np.ndarray:
    """q * s in fp64 (exact: 4 significant bits times 24)."""
    rows, cols = q.shape
    sf = np.repeat(np.repeat(s.astype(np.float64), br, axis=0)[:rows], bc, axis=1)[:, :cols]
    return e4m3_decode(q) * sf


# --------------------------------------------------------------------------
# routing and permute
# --------------------------------------------------------------------------

def route_topk(z, k: int):
    z = _c(z, np.float32)
    T, E = z.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    lib().orc_route_topk(_p(z), T, E, k, _p(idx), _p(w))
    return idx, w


def route_replay(payload, layer: int, E: int, w_in=None, z=None):
    P = _c(payload, np.int32)
    L, k, T = P.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    wi = None if w_in is None else _c(w_in, np.float32)
    zz = None if z is None else _c(z, np.float32)
    st = lib().orc_route_replay(_p(P), L, layer, T, E, k, _p(wi), _p(zz), _p(idx), _p(w))
    return idx, w, int(st)


def rows_capacity(T: int, k: int, E: int, align: int) -> int:
    """Upper bound of the padded row count, rounded up to 128."""
    r = T * k + E * (align - 1)
    return (r + 127) // 128 * 128


def permute(idx, E: int, align: int, rows_cap: int | None = None):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    if rows_cap is None:
        rows_cap = rows_capacity(T, k, E, align)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    pos = np.empty((T, k), np.int32)
    src = np.empty(rows_cap, np.int32)
    lib().orc_permute(_p(idx), T, k, E, align, _p(counts), _p(offsets), _p(pos), _p(src), rows_cap)
    return counts, offsets, pos, src


# --------------------------------------------------------------------------
# fp64 contractions
# --------------------------------------------------------------------------

def rowdot(A, expert, W, trans: bool = False):
    """out[i] = W[expert[i]] @ A[i]  (trans=False, W[e] is [N, K])
       out[i] = W[expert[i]].T @ A[i] (trans=True,  W[e] is [K, N]).

    W is either a float64 array [E, nr, nc] or a tuple (codes uint8
    [E, nr, nc], scales float32 [E, nr/128, nc/128]) of 128x128 blocks.
    """
    A = _c(A, np.float64)
    expert = _c(expert, np.int32)
    if isinstance(W, tuple):
        Wq, Ws = _c(W[0], np.uint8), _c(W[1], np.float32)
        Wf = None
        E, nr, nc = Wq.shape
    else:
        Wf = _c(W, np.float64)
        Wq = Ws = None
        E, nr, nc = Wf.shape
    n = A.shape[0]
    N = nc if trans else nr
    out = np.empty((n, N), np.float64)
    lib().orc_rowdot(_p(A), n, _p(expert), E, _p(Wq), _p(Ws), _p(Wf), nr, nc, int(trans), _p(out))
    return out


def wgrad(A, B, m0=0, M=None, n0=0, N=None):
    """out[m, n] = sum_r A[r, m0+m] * B[r, n0+n], fp64, rows in order."""
    A = _c(A, np.float64)
    B = _c(B, np.float64)
    R = A.shape[0]
    M = A.shape[1] - m0 if M is None else M
    N = B.shape[1] - n0 if N is None else N
    out = np.empty((M, N), np.float64)
    lib().orc_wgrad(_p(A), A.shape[1], m0, M, _p(B), B.shape[1], n0, N, R, _p(out))
    return out


def num_threads() -> int:
    return int(lib().orc_num_threads())
