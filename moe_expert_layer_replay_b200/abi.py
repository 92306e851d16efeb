"""ctypes binding of libmoe.so: one Python function per C entry point, same
names without the ``moe_`` prefix.  Argument marshalling only — every step of
the layer runs in the library's CUDA kernels; torch tensors supply device
memory and the current stream.  Contracts and layouts: include/moe.h.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

OK, INVALID_ARG, UNSUPPORTED, CUDA_ERR, BAD_ROUTING, TIMEOUT = range(6)
GEMM_GATEUP_SILU, GEMM_DOWN, GEMM_DGRAD_DOWN_SILU, GEMM_DGRAD_GATEUP, GEMM_WGRAD_DOWN, GEMM_WGRAD_GATEUP = range(6)

EXPORTS = [
    "moe_rows_capacity", "moe_permute_workspace_size", "moe_strerror", "moe_get_status",
    "moe_set_wait_budget", "moe_route_topk", "moe_route_replay", "moe_permute",
    "moe_quant_fp8_block", "moe_quant_weights", "moe_grouped_gemm_fp8", "moe_combine",
    "moe_combine_bwd", "moe_unpermute_reduce", "moe_permute_noalloc", "moe_kernel_launches",
    "moe_router_fwd", "moe_capture_payload", "moe_router_bwd_workspace_size", "moe_router_bwd",
    "moe_grouped_gemm_fp8_seg", "moe_gateup_gather_fp8", "moe_set_gemm_variant", "moe_quant_nvfp4",
    "moe_gemm_pair_clusters", "moe_gemm_nvfp4",
]


class MoeError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call}: {strerror(status)} (status {status})")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("D", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("align", ctypes.c_int32)]

    def __repr__(self):
        return f"Dims(T={self.T}, D={self.D}, I={self.I}, E={self.E}, k={self.k}, align={self.align})"


class GemmArgs(ctypes.Structure):
    _fields_ = [("a", ctypes.c_void_p), ("sa", ctypes.c_void_p), ("b", ctypes.c_void_p),
                ("sb", ctypes.c_void_p), ("aux", ctypes.c_void_p), ("out_q", ctypes.c_void_p),
                ("out_s", ctypes.c_void_p), ("out_bf16", ctypes.c_void_p), ("out_f32", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so.  Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m moe_expert_layer_replay_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64
        D = ctypes.POINTER(Dims)
        sig = {
            "moe_rows_capacity": (I64, [D]),
            "moe_permute_workspace_size": (SZ, [D]),
            "moe_strerror": (ctypes.c_char_p, [ctypes.c_int]),
            "moe_get_status": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_int)]),
            "moe_set_wait_budget": (None, [U64]),
            "moe_kernel_launches": (U64, []),
            "moe_set_gemm_variant": (ctypes.c_int, [ctypes.c_int]),
            "moe_gemm_pair_clusters": (ctypes.c_int, []),
            "moe_route_topk": (ctypes.c_int, [P, D, P, P, P]),
            "moe_route_replay": (ctypes.c_int, [P, I32, I32, D, P, P, P, P, P]),
            "moe_router_fwd": (ctypes.c_int, [P, P, D, P, P, P, P]),
            "moe_capture_payload": (ctypes.c_int, [P, D, I32, I32, P, P]),
            "moe_router_bwd_workspace_size": (SZ, [D]),
            "moe_router_bwd": (ctypes.c_int, [P, P, P, D, P, P, P, P, SZ, P]),
            "moe_permute": (ctypes.c_int, [P, D, P, P, P, P, P, P, P, P, P, P, SZ, P]),
            "moe_permute_noalloc": (ctypes.c_int, [P, D, P, P, P, P, P, P, P, P]),
            "moe_quant_fp8_block": (ctypes.c_int, [P, I64, I64, I64, I32, I32, P, P, P, P, P]),
            "moe_quant_weights": (ctypes.c_int, [P, P, P, D, P, P, P, P, P, P, P, P, P]),
            "moe_quant_nvfp4": (ctypes.c_int, [P, I64, I64, I64, P, P, I32, P, P, P]),
            "moe_gemm_nvfp4": (ctypes.c_int, [I64, I32, I32, I32, P, P, P, P, P, P, P, P, P]),
            "moe_grouped_gemm_fp8": (ctypes.c_int, [I32, D, P, ctypes.POINTER(GemmArgs), P]),
            "moe_grouped_gemm_fp8_seg": (ctypes.c_int, [I32, D, I64, P, I32, ctypes.POINTER(GemmArgs), P]),
            "moe_gateup_gather_fp8": (ctypes.c_int, [D, P, P, ctypes.POINTER(GemmArgs), P]),
            "moe_combine": (ctypes.c_int, [P, P, P, D, P, P]),
            "moe_combine_bwd": (ctypes.c_int, [P, P, P, P, P, P, P, D, P, P, P, P, P, P]),
            "moe_unpermute_reduce": (ctypes.c_int, [P, P, D, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(name, st):
    if st != OK:
        raise MoeError(name, st)


def dims(T, D, I, E, k, align=128) -> Dims:
    return Dims(int(T), int(D), int(I), int(E), int(k), int(align))


# ---------------------------------------------------------------- queries --
def rows_capacity(d: Dims) -> int:
    return int(lib().moe_rows_capacity(ctypes.byref(d)))


def permute_workspace_size(d: Dims) -> int:
    return int(lib().moe_permute_workspace_size(ctypes.byref(d)))


def strerror(st: int) -> str:
    return lib().moe_strerror(int(st)).decode()


def get_status(stream=None) -> int:
    out = ctypes.c_int(0)
    _check("moe_get_status", lib().moe_get_status(_s(stream), ctypes.byref(out)))
    return out.value


def set_wait_budget(cycles: int) -> None:
    lib().moe_set_wait_budget(int(cycles))


def set_gemm_variant(variant: int) -> None:
    """0: one-SM tiles (default), 1: the 2-SM MMA, -1: chosen per call."""
    _check("moe_set_gemm_variant", lib().moe_set_gemm_variant(int(variant)))


def gemm_pair_clusters() -> int:
    """CTA pairs of the last 2-SM GEMM launch (0 before any)."""
    return int(lib().moe_gemm_pair_clusters())


def kernel_launches() -> int:
    """Kernels launched (or recorded into a capture) by the library so far."""
    return int(lib().moe_kernel_launches())


# ------------------------------------------------------------ entry points --
def route_topk(logits, d: Dims, idx, w, stream=None):
    _check("moe_route_topk", lib().moe_route_topk(_p(logits), ctypes.byref(d), _p(idx), _p(w), _s(stream)))


def route_replay(payload, L, layer, d: Dims, w_in, logits, idx, w, stream=None):
    _check("moe_route_replay", lib().moe_route_replay(_p(payload), int(L), int(layer), ctypes.byref(d),
                                                      _p(w_in), _p(logits), _p(idx), _p(w), _s(stream)))


def router_fwd(x, w_r, d: Dims, z, idx=None, w=None, stream=None):
    _check("moe_router_fwd", lib().moe_router_fwd(_p(x), _p(w_r), ctypes.byref(d), _p(z), _p(idx), _p(w), _s(stream)))


def capture_payload(idx, d: Dims, L, layer, payload, stream=None):
    _check("moe_capture_payload", lib().moe_capture_payload(_p(idx), ctypes.byref(d), int(L), int(layer),
                                                            _p(payload), _s(stream)))


def router_bwd_workspace_size(d: Dims) -> int:
    return int(lib().moe_router_bwd_workspace_size(ctypes.byref(d)))


def router_bwd(dz, x, w_r, d: Dims, dx_in=None, dx=None, dw_r=None, ws=None, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("moe_router_bwd", lib().moe_router_bwd(_p(dz), _p(x), _p(w_r), ctypes.byref(d), _p(dx_in), _p(dx),
                                                  _p(dw_r), _p(ws), nbytes, _s(stream)))


def permute(idx, d: Dims, counts, offsets, pos, src_idx, x, xq, xs, xqT, xsT, ws, stream=None):
    _check("moe_permute", lib().moe_permute(_p(idx), ctypes.byref(d), _p(counts), _p(offsets), _p(pos),
                                            _p(src_idx), _p(x), _p(xq), _p(xs), _p(xqT), _p(xsT), _p(ws),
                                            ws.numel() * ws.element_size(), _s(stream)))


def permute_noalloc(idx, d: Dims, counts, offsets, pos, src_idx, x, xq, xs, stream=None):
    """moe_permute with the library's own fixed scratch (no workspace argument)."""
    _check("moe_permute_noalloc", lib().moe_permute_noalloc(_p(idx), ctypes.byref(d), _p(counts), _p(offsets),
                                                            _p(pos), _p(src_idx), _p(x), _p(xq), _p(xs), _s(stream)))


def quant_fp8_block(inp, rows, cols, ld, blk_r, blk_c, q, s, qT=None, sT=None, stream=None):
    _check("moe_quant_fp8_block", lib().moe_quant_fp8_block(_p(inp), int(rows), int(cols), int(ld), int(blk_r),
                                                            int(blk_c), _p(q), _p(s), _p(qT), _p(sT), _s(stream)))


NVFP4_SF_ROWS, NVFP4_SF_MMA_A, NVFP4_SF_MMA_B = 0, 1, 2


def quant_nvfp4(inp, rows, cols, ld, q, sf, amax, s_g, sf_layout=NVFP4_SF_ROWS, stream=None):
    """NVFP4: packed e2m1 codes q [rows, cols/2], e4m3 block scales sf ([rows, cols/16], or the
    NVFP4 GEMM's A- or B-side layout: NVFP4_SF_MMA_A / _B, 4 * rows * cols/16 bytes), tensor amax
    and scale s_g (one float each, device)."""
    _check("moe_quant_nvfp4", lib().moe_quant_nvfp4(_p(inp), int(rows), int(cols), int(ld), _p(q), _p(sf),
                                                    int(sf_layout), _p(amax), _p(s_g), _s(stream)))


def gemm_nvfp4(rows_cap, N, K, n_seg, offsets, a, sfa, a_sg, b, sfb, b_sg, out, stream=None):
    """NVFP4 grouped GEMM: out [rows_cap, N] fp32 = value(A) value(B_e)^T per segment."""
    _check("moe_gemm_nvfp4", lib().moe_gemm_nvfp4(int(rows_cap), int(N), int(K), int(n_seg), _p(offsets), _p(a),
                                                  _p(sfa), _p(a_sg), _p(b), _p(sfb), _p(b_sg), _p(out),
                                                  _s(stream)))


def quant_weights(w_gate, w_up, w_down, d: Dims, wgu_q, wgu_s, wd_q, wd_s,
                  wguT_q=None, wguT_s=None, wdT_q=None, wdT_s=None, stream=None):
    _check("moe_quant_weights", lib().moe_quant_weights(_p(w_gate), _p(w_up), _p(w_down), ctypes.byref(d),
                                                        _p(wgu_q), _p(wgu_s), _p(wd_q), _p(wd_s), _p(wguT_q),
                                                        _p(wguT_s), _p(wdT_q), _p(wdT_s), _s(stream)))


def grouped_gemm_fp8(op, d: Dims, offsets, a, sa, b, sb, aux=None, out_q=None, out_s=None,
                     out_bf16=None, out_f32=None, stream=None):
    g = GemmArgs(*[None if t is None else t.data_ptr() for t in (a, sa, b, sb, aux, out_q, out_s, out_bf16, out_f32)])
    _check("moe_grouped_gemm_fp8", lib().moe_grouped_gemm_fp8(int(op), ctypes.byref(d), _p(offsets),
                                                              ctypes.byref(g), _s(stream)))


def grouped_gemm_fp8_seg(op, d: Dims, rows_cap, offsets, n_seg, a, sa, b, sb, aux=None, out_q=None, out_s=None,
                         out_bf16=None, stream=None):
    """Grouped GEMM over n_seg row segments; segment v uses expert v % d.E's weights."""
    g = GemmArgs(*[None if t is None else t.data_ptr() for t in (a, sa, b, sb, aux, out_q, out_s, out_bf16, None)])
    _check("moe_grouped_gemm_fp8_seg", lib().moe_grouped_gemm_fp8_seg(int(op), ctypes.byref(d), int(rows_cap),
                                                                      _p(offsets), int(n_seg), ctypes.byref(g),
                                                                      _s(stream)))


def gateup_gather_fp8(d: Dims, offsets, src_idx, a_tok, sa_tok, b, sb, aux=None, out_q=None, out_s=None,
                      out_bf16=None, stream=None):
    """GATEUP_SILU with A gathered from the token-row codes (no permuted copy)."""
    g = GemmArgs(*[None if t is None else t.data_ptr() for t in (a_tok, sa_tok, b, sb, aux, out_q, out_s, out_bf16,
                                                                None)])
    _check("moe_gateup_gather_fp8", lib().moe_gateup_gather_fp8(ctypes.byref(d), _p(offsets), _p(src_idx),
                                                                ctypes.byref(g), _s(stream)))


def combine(Y, w, pos, d: Dims, y, stream=None):
    _check("moe_combine", lib().moe_combine(_p(Y), _p(w), _p(pos), ctypes.byref(d), _p(y), _s(stream)))


def combine_bwd(dy, Y, w, pos, idx, counts, offsets, d: Dims, dYq, dYs, dY_bf16, d_w, d_logits, stream=None):
    _check("moe_combine_bwd", lib().moe_combine_bwd(_p(dy), _p(Y), _p(w), _p(pos), _p(idx), _p(counts),
                                                    _p(offsets), ctypes.byref(d), _p(dYq), _p(dYs), _p(dY_bf16),
                                                    _p(d_w), _p(d_logits), _s(stream)))


def unpermute_reduce(dX, pos, d: Dims, dx, stream=None):
    _check("moe_unpermute_reduce", lib().moe_unpermute_reduce(_p(dX), _p(pos), ctypes.byref(d), _p(dx), _s(stream)))
