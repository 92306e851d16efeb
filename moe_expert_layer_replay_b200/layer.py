"""The MoE expert layer, forward and backward, as a sequence of C-ABI calls.

This module only allocates device buffers (torch) and calls the entry points
of libmoe.so in order on the current stream; it computes nothing itself.

Forward:  route (top-k, or replay of a [num_layers, top_k, seq_len] payload)
          -> permute + fused 1x128 FP8 dispatch -> GEMM gate/up + SiLU + h-quant
          -> GEMM down -> weighted combine.
Backward: combine backward (dY rows in FP8, d_w, d_logits) -> 128x1 FP8 of dY
          and h -> dgrad down + SiLU backward -> 128x1 FP8 of d[g|u] -> dgrad
          gate/up -> unpermute-reduce -> wgrad down and gate/up (fp32 +=).
"""
from __future__ import annotations

import torch

from . import abi

U8, F32, I32, BF16 = torch.uint8, torch.float32, torch.int32, torch.bfloat16


class Weights:
    """128x128 block-FP8 expert weights (plus their transposes for training)."""

    def __init__(self, d: abi.Dims, device, train: bool):
        E, D, I = d.E, d.D, d.I
        z = dict(device=device)
        self.wgu_q = torch.empty(E, 2 * I, D, dtype=U8, **z)
        self.wgu_s = torch.empty(E, 2 * I // 128, D // 128, dtype=F32, **z)
        self.wd_q = torch.empty(E, D, I, dtype=U8, **z)
        self.wd_s = torch.empty(E, D // 128, I // 128, dtype=F32, **z)
        self.train = train
        if train:
            self.wguT_q = torch.empty(E, D, 2 * I, dtype=U8, **z)
            self.wguT_s = torch.empty(E, D // 128, 2 * I // 128, dtype=F32, **z)
            self.wdT_q = torch.empty(E, I, D, dtype=U8, **z)
            self.wdT_s = torch.empty(E, I // 128, D // 128, dtype=F32, **z)
        else:
            self.wguT_q = self.wguT_s = self.wdT_q = self.wdT_s = None


def quantise_weights(d: abi.Dims, w_gate, w_up, w_down, train: bool, out: Weights | None = None,
                     stream=None) -> Weights:
    """a5: W_gate, W_up [E, I, D] and W_down [E, D, I] (bf16) -> Weights."""
    W = out if out is not None else Weights(d, w_gate.device, train)
    abi.quant_weights(w_gate, w_up, w_down, d, W.wgu_q, W.wgu_s, W.wd_q, W.wd_s,
                      W.wguT_q, W.wguT_s, W.wdT_q, W.wdT_s, stream=stream)
    return W


class Buffers:
    """Every device buffer one layer pass needs, sized from the dims alone
    (R_cap rows bound the permuted rows, so nothing is read back)."""

    def __init__(self, d: abi.Dims, device, train: bool, gather: bool = False):
        self.d = d
        self.train = train
        self.gather = gather
        T, D, I, E, k = d.T, d.D, d.I, d.E, d.k
        R = abi.rows_capacity(d)
        self.R_cap = R
        z = dict(device=device)
        self.idx = torch.empty(T, k, dtype=I32, **z)
        self.w = torch.empty(T, k, dtype=F32, **z)
        self.counts = torch.empty(E, dtype=I32, **z)
        self.offsets = torch.empty(E + 1, dtype=I32, **z)
        self.pos = torch.empty(T, k, dtype=I32, **z)
        self.src = torch.empty(R, dtype=I32, **z)
        self.ws = torch.empty(max(16, abi.permute_workspace_size(d)), dtype=U8, **z)
        self.xq = torch.empty(R, D, dtype=U8, **z)
        self.xs = torch.empty(D // 128, R, dtype=F32, **z)
        self.hq = torch.empty(R, I, dtype=U8, **z)
        self.hs = torch.empty(I // 128, R, dtype=F32, **z)
        self.Y = torch.empty(R, D, dtype=BF16, **z)
        self.y = torch.empty(T, D, dtype=BF16, **z)
        if gather:   # 1x128 FP8 of the token rows, read by the gathering gate/up GEMM
            self.xq_tok = torch.empty(T, D, dtype=U8, **z)
            self.xs_tok = torch.empty(D // 128, T, dtype=F32, **z)
        if train:
            self.gu = torch.empty(R, 2 * I, dtype=BF16, **z)
            self.h = torch.empty(R, I, dtype=BF16, **z)
            self.xqT = torch.empty(D, R, dtype=U8, **z)
            self.xsT = torch.empty(R // 128, D, dtype=F32, **z)
            self.hqT = torch.empty(I, R, dtype=U8, **z)
            self.hsT = torch.empty(R // 128, I, dtype=F32, **z)
            self.dYq = torch.empty(R, D, dtype=U8, **z)
            self.dYs = torch.empty(D // 128, R, dtype=F32, **z)
            self.dYb = torch.empty(R, D, dtype=BF16, **z)
            self.dYqT = torch.empty(D, R, dtype=U8, **z)
            self.dYsT = torch.empty(R // 128, D, dtype=F32, **z)
            self.dGU = torch.empty(R, 2 * I, dtype=BF16, **z)
            self.dGUq = torch.empty(R, 2 * I, dtype=U8, **z)
            self.dGUs = torch.empty(2 * I // 128, R, dtype=F32, **z)
            self.dGUqT = torch.empty(2 * I, R, dtype=U8, **z)
            self.dGUsT = torch.empty(R // 128, 2 * I, dtype=F32, **z)
            self.dX = torch.empty(R, D, dtype=BF16, **z)
            self.dx = torch.empty(T, D, dtype=BF16, **z)
            self.d_w = torch.empty(T, k, dtype=F32, **z)
            self.d_logits = torch.empty(T, E, dtype=F32, **z)
            self.dWd = torch.zeros(E, D, I, dtype=F32, **z)
            self.dWgu = torch.zeros(E, 2 * I, D, dtype=F32, **z)


def route(B: Buffers, logits=None, payload=None, layer: int = 0, w_in=None, stream=None):
    """a1 (logits only) or a2 (payload [L, k, T], with w_in or trainer logits)."""
    if payload is None:
        abi.route_topk(logits, B.d, B.idx, B.w, stream=stream)
    else:
        abi.route_replay(payload, payload.shape[0], layer, B.d, w_in, logits, B.idx, B.w, stream=stream)


def forward(B: Buffers, x, W: Weights, stream=None, h_out=None):
    """a3-a8 after routing.  Returns B.y.  ``h_out`` (optional, [R_cap, I]
    bf16) receives h; training runs keep h in B.h.  Buffers made with
    gather=True quantise the token rows once and let the gate/up GEMM gather
    its rows (no permuted FP8 copy; the forward's results are the same)."""
    d = B.d
    t = B.train
    if B.gather:
        abi.quant_fp8_block(x, d.T, d.D, d.D, 1, 128, B.xq_tok, B.xs_tok, stream=stream)
        abi.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, x if t else None, None, None,
                    B.xqT if t else None, B.xsT if t else None, B.ws, stream=stream)
        abi.gateup_gather_fp8(d, B.offsets, B.src, B.xq_tok, B.xs_tok, W.wgu_q, W.wgu_s,
                              aux=B.gu if t else None, out_q=B.hq, out_s=B.hs,
                              out_bf16=B.h if t else h_out, stream=stream)
    else:
        abi.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, x, B.xq, B.xs,
                    B.xqT if t else None, B.xsT if t else None, B.ws, stream=stream)
        abi.grouped_gemm_fp8(abi.GEMM_GATEUP_SILU, d, B.offsets, B.xq, B.xs, W.wgu_q, W.wgu_s,
                             aux=B.gu if t else None, out_q=B.hq, out_s=B.hs,
                             out_bf16=B.h if t else h_out, stream=stream)
    abi.grouped_gemm_fp8(abi.GEMM_DOWN, d, B.offsets, B.hq, B.hs, W.wd_q, W.wd_s, out_bf16=B.Y, stream=stream)
    abi.combine(B.Y, B.w, B.pos, d, B.y, stream=stream)
    return B.y


def backward(B: Buffers, dy, W: Weights, router_logits: bool, stream=None):
    """b1-b4.  Returns (dx, d_w, d_logits or None); dW accumulate into B.dWd, B.dWgu."""
    d = B.d
    R, D, I = B.R_cap, d.D, d.I
    abi.combine_bwd(dy, B.Y, B.w, B.pos, B.idx, B.counts, B.offsets, d, B.dYq, B.dYs, B.dYb, B.d_w,
                    B.d_logits if router_logits else None, stream=stream)
    abi.quant_fp8_block(B.dYb, R, D, D, 128, 1, B.dYqT, B.dYsT, stream=stream)
    abi.quant_fp8_block(B.h, R, I, I, 128, 1, B.hqT, B.hsT, stream=stream)
    abi.grouped_gemm_fp8(abi.GEMM_DGRAD_DOWN_SILU, d, B.offsets, B.dYq, B.dYs, W.wdT_q, W.wdT_s, aux=B.gu,
                         out_q=B.dGUq, out_s=B.dGUs, out_bf16=B.dGU, stream=stream)
    abi.quant_fp8_block(B.dGU, R, 2 * I, 2 * I, 128, 1, B.dGUqT, B.dGUsT, stream=stream)
    abi.grouped_gemm_fp8(abi.GEMM_DGRAD_GATEUP, d, B.offsets, B.dGUq, B.dGUs, W.wguT_q, W.wguT_s,
                         out_bf16=B.dX, stream=stream)
    abi.unpermute_reduce(B.dX, B.pos, d, B.dx, stream=stream)
    abi.grouped_gemm_fp8(abi.GEMM_WGRAD_DOWN, d, B.offsets, B.dYqT, B.dYsT, B.hqT, B.hsT, out_f32=B.dWd,
                         stream=stream)
    abi.grouped_gemm_fp8(abi.GEMM_WGRAD_GATEUP, d, B.offsets, B.dGUqT, B.dGUsT, B.xqT, B.xsT, out_f32=B.dWgu,
                         stream=stream)
    return B.dx, B.d_w, (B.d_logits if router_logits else None)
