"""The MoE expert layer, step by step, in fp64 — TEST INFRASTRUCTURE ONLY.

Each function is one step of the layer, written in the order of the method:
route (or replay) -> permute -> block-FP8 quantise and dispatch -> gated
expert FFN -> weighted combine, and the backward of all of it.  Sources:

* top-k routing per token: "prime-rl 0.6.0 løfter trillion-parameter RL ...",
  §Drift og omkostninger i realiteten;
* router replay of a [num_layers, top_k, seq_len] payload: "RL at 1T scale:
  prime-rl performance deep dive", §Router Replay;
* dispatch/combine per layer: "RL at 1T scale ...", §Wide Expert Parallelism
  and §Parallelism / EP;
* block-scaled FP8 as in DeepSeek-V3 for training: "RL at 1T scale ...",
  §FP8 Training.

The pages do not give the FFN form, block shapes, scale rule or rounding
points.  The readings used (all listed in the design notes):

* expert FFN: g = W_gate x, u = W_up x, h = silu(g) * u, Y = W_down h,
  silu(g) = g * sigmoid(g); Y is unweighted and the combine applies w;
* activations are quantised in 1x128 blocks along the contraction axis,
  weights in 128x128 blocks, wgrad operands in 128x1 blocks along rows;
* h, Y, dY rows, d[g|u], dX and dx are rounded to bf16 at the points below;
  g and u are saved as bf16 for the backward;
* the gradient passes straight through each quantiser;
* dY row = bf16(fp32(w * dy)): the product is taken in fp32, the precision the
  kernel computes in, so that the FP8 codes derived from it are bit-exact.
"""
from __future__ import annotations

import numpy as np

from . import (bf16_round, bf16_to_f64, dequant_block, permute, quant_block,
               rowdot, wgrad)


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------

def expert_of_rows(offsets, rows) -> np.ndarray:
    """Expert owning each permuted row (-1 for rows past the last segment)."""
    rows = np.asarray(rows, np.int64)
    e = np.searchsorted(np.asarray(offsets, np.int64), rows, side="right") - 1
    E = len(offsets) - 1
    e[(rows >= offsets[E]) | (e < 0)] = -1
    return e.astype(np.int32)


def quant_weights(W_bf16):
    """128x128 block-FP8 of a stack of expert matrices [E, nr, nc]."""
    E, nr, nc = W_bf16.shape
    q = np.empty((E, nr, nc), np.uint8)
    s = np.empty((E, (nr + 127) // 128, (nc + 127) // 128), np.float32)
    for e in range(E):
        q[e], s[e] = quant_block(W_bf16[e], 128, 128)
    return q, s


def silu(g):
    return g / (1.0 + np.exp(-g))


def dispatch_rows(x_bf16, src, rows, k: int):
    """bf16 rows of the permuted activation matrix; padding rows are zero."""
    src_r = np.asarray(src)[rows]
    out = np.zeros((len(rows), x_bf16.shape[1]), np.uint16)
    ok = src_r >= 0
    out[ok] = x_bf16[src_r[ok] // k]
    return out


# --------------------------------------------------------------------------
# forward steps
# --------------------------------------------------------------------------

def gateup_rows(xq, xs_grid, expert, Wg, Wu):
    """g, u (fp64) of permuted rows from their 1x128 FP8 codes and scales.

    xq [n, D] codes, xs_grid [n, D/128] scales; Wg, Wu as accepted by rowdot.
    """
    A = dequant_block(xq, xs_grid, 1, 128)
    return rowdot(A, expert, Wg), rowdot(A, expert, Wu)


def swiglu_h(g, u):
    """h = bf16(silu(g) * u) from fp64 g, u."""
    return bf16_round(silu(g) * u)


def down_rows(hq, hs_grid, expert, Wd):
    """Y rows (bf16 bits) = bf16(W_down[e] @ dequant(h))."""
    return bf16_round(rowdot(dequant_block(hq, hs_grid, 1, 128), expert, Wd))


def combine(Y_rows_f64, w, pos_ok):
    """y_t = bf16(sum_j w[t,j] * Y[pos[t,j]]) in fp64, j ascending.

    Y_rows_f64 [T, k, D] = the gathered Y rows per token; pos_ok [T, k] masks
    invalid entries."""
    acc = np.zeros((Y_rows_f64.shape[0], Y_rows_f64.shape[2]), np.float64)
    for j in range(Y_rows_f64.shape[1]):
        acc += np.where(pos_ok[:, j:j + 1], w[:, j:j + 1].astype(np.float64) * Y_rows_f64[:, j], 0.0)
    return bf16_round(acc)


def forward(x_bf16, idx, w, Wg_bf16, Wu_bf16, Wd_bf16, align: int = 128, quantised_w=None):
    """Full forward of one layer for all tokens (small problems only).

    Returns a dict with every intermediate the GPU path also produces.
    """
    T, k = idx.shape
    E = Wg_bf16.shape[0] if Wg_bf16 is not None else quantised_w[0][0].shape[0]
    counts, offsets, pos, src = permute(idx, E, align)
    R_pad = int(offsets[E])
    rows = np.arange(R_pad)
    Xp = dispatch_rows(x_bf16, src, rows, k)
    xq, xs = quant_block(Xp, 1, 128)
    if quantised_w is None:
        quantised_w = (quant_weights(Wg_bf16), quant_weights(Wu_bf16), quant_weights(Wd_bf16))
    Wg, Wu, Wd = quantised_w
    expert = expert_of_rows(offsets, rows)
    g, u = gateup_rows(xq, xs, expert, Wg, Wu)
    h = swiglu_h(g, u)
    hq, hs = quant_block(h, 1, 128)
    Y = down_rows(hq, hs, expert, Wd)
    ok = pos >= 0
    Yg = bf16_to_f64(Y)[np.where(ok, pos, 0)]
    y = combine(Yg, w, ok)
    return dict(counts=counts, offsets=offsets, pos=pos, src=src, Xp=Xp, xq=xq, xs=xs,
                g=g, u=u, g_b=bf16_round(g), u_b=bf16_round(u), h=h, hq=hq, hs=hs,
                Y=Y, y=y, expert=expert, Wq=quantised_w)


def forward_tokens(x_bf16, idx, w, quantised_w, tokens, align: int = 128):
    """Forward outputs of a sample of tokens, one token at a time.

    Runs the permutation over all T tokens (it decides each routed row's
    expert), then the expert FFN only for the rows the sampled tokens occupy:
    for token t and slot j, row pos[t, j] holds x[t] quantised in 1x128
    blocks (quantisation is row-local, so this equals that row of the full
    dispatch).  Returns a dict with, per sampled token, its rows' h, hq, hs,
    Y and the combined y.
    """
    T, k = idx.shape
    Wg, Wu, Wd = quantised_w
    E = Wg[0].shape[0]
    counts, offsets, pos, src = permute(idx, E, align)
    tokens = np.asarray(tokens, np.int64)
    rows = pos[tokens].reshape(-1)                       # [n*k]
    ok = rows >= 0
    xr = np.repeat(x_bf16[tokens], k, axis=0)            # row (t, j) holds x[t]
    xq, xs = quant_block(xr, 1, 128)
    expert = np.where(ok, expert_of_rows(offsets, np.where(ok, rows, 0)), -1).astype(np.int32)
    g, u = gateup_rows(xq, xs, expert, Wg, Wu)
    h = swiglu_h(g, u)
    hq, hs = quant_block(h, 1, 128)
    Y = down_rows(hq, hs, expert, Wd)
    n = len(tokens)
    Yg = bf16_to_f64(Y).reshape(n, k, -1)
    y = combine(Yg, w[tokens], ok.reshape(n, k))
    return dict(rows=rows.reshape(n, k), h=h, hq=hq, hs=hs, Y=Y, y=y, offsets=offsets, pos=pos)


# --------------------------------------------------------------------------
# backward steps
# --------------------------------------------------------------------------

def scaled_rows(dy_bf16, w, pos, rows_total: int):
    """dY rows (bf16 bits) in permuted order: bf16(fp32(w[t,j] * dy[t]))."""
    T, k = pos.shape
    D = dy_bf16.shape[1]
    out = np.zeros((rows_total, D), np.uint16)
    dyf = bf16_to_f64(dy_bf16).astype(np.float32)
    for j in range(k):
        ok = pos[:, j] >= 0
        prod32 = (w[:, j:j + 1].astype(np.float32) * dyf)  # IEEE fp32 product
        out[pos[ok, j]] = bf16_round(prod32[ok].astype(np.float64))
    return out


def router_grads(dy_bf16, Y_gathered_f64, w, z=None, idx=None):
    """d_w[t,j] = <dy_t, Y[pos[t,j]]>; dz over the chosen set (0 elsewhere).

    w is the softmax over the chosen set S; for i in S:
    dz_i = p_i * (d_w_i - sum_j p_j d_w_j), recomputed in fp64 from z."""
    dyf = bf16_to_f64(dy_bf16)
    d_w = np.einsum("td,tkd->tk", dyf, Y_gathered_f64)
    dz = None
    if z is not None:
        T, k = idx.shape
        zS = np.take_along_axis(z.astype(np.float64), idx.astype(np.int64), axis=1)
        m = zS.max(axis=1, keepdims=True)
        p = np.exp(zS - m)
        p /= p.sum(axis=1, keepdims=True)
        inner = (p * d_w).sum(axis=1, keepdims=True)
        dzS = p * (d_w - inner)
        dz = np.zeros(z.shape, np.float64)
        np.put_along_axis(dz, idx.astype(np.int64), dzS, axis=1)
    return d_w, dz


def swiglu_bwd(dH, g_b, u_b):
    """dg = dH * u * s * (1 + g (1 - s)), du = dH * silu(g), s = sigmoid(g),
    with g, u the bf16 values saved by the forward.  Returns bf16 bits."""
    g = bf16_to_f64(g_b)
    u = bf16_to_f64(u_b)
    s = 1.0 / (1.0 + np.exp(-g))
    dg = dH * u * s * (1.0 + g * (1.0 - s))
    du = dH * g * s
    return bf16_round(dg), bf16_round(du)


def dgrad_down(dYq, dYs_grid, expert, Wd):
    """dH = W_down[e]^T dY over the 1x128 FP8 dY rows (fp64)."""
    return rowdot(dequant_block(dYq, dYs_grid, 1, 128), expert, Wd, trans=True)


def dgrad_gateup(dGq, dGs, dUq, dUs, expert, Wg, Wu):
    """dX rows = bf16(W_gate^T dG + W_up^T dU) (fp64 sums)."""
    a = rowdot(dequant_block(dGq, dGs, 1, 128), expert, Wg, trans=True)
    b = rowdot(dequant_block(dUq, dUs, 1, 128), expert, Wu, trans=True)
    return bf16_round(a + b)


def unpermute_reduce(dX_rows_f64, pos):
    """dx_t = bf16(sum_j dX[pos[t,j]]), fp64, j ascending."""
    T, k = pos.shape
    acc = np.zeros((T, dX_rows_f64.shape[1]), np.float64)
    for j in range(k):
        ok = pos[:, j] >= 0
        acc[ok] += dX_rows_f64[pos[ok, j]]
    return bf16_round(acc)


def quant_rows128(M_bf16):
    """128x1 blocks along rows: (codes [rows, cols], scales [rows/128, cols])."""
    return quant_block(M_bf16, 128, 1)


def wgrad_expert(Aq, As, Bq, Bs, r0: int, r1: int, m0=0, M=None, n0=0, N=None):
    """dW[m, n] = sum_{r in [r0, r1)} deq(A)[r, m] * deq(B)[r, n].

    A, B: 128x1 FP8 (codes [rows, cols], scales [rows/128, cols]); r0 and r1
    are multiples of 128 (segments are 128-aligned)."""
    A = dequant_block(Aq[r0:r1], As[r0 // 128:(r1 + 127) // 128], 128, 1)
    B = dequant_block(Bq[r0:r1], Bs[r0 // 128:(r1 + 127) // 128], 128, 1)
    return wgrad(A, B, m0, M, n0, N)


def backward(fw, x_bf16, dy_bf16, idx, w, z=None):
    """Full backward of one layer (small problems only), from forward dict fw."""
    T, k = idx.shape
    offsets, pos, expert = fw["offsets"], fw["pos"], fw["expert"]
    E = len(offsets) - 1
    R_pad = int(offsets[E])
    Wg, Wu, Wd = fw["Wq"]
    ok = pos >= 0
    Yg = bf16_to_f64(fw["Y"])[np.where(ok, pos, 0)]
    d_w, dz = router_grads(dy_bf16, Yg, w, z, idx)
    dYr = scaled_rows(dy_bf16, w, pos, R_pad)
    dYq, dYs = quant_block(dYr, 1, 128)
    dYqT, dYsT = quant_rows128(dYr)
    dH = dgrad_down(dYq, dYs, expert, Wd)
    dG, dU = swiglu_bwd(dH, fw["g_b"], fw["u_b"])
    dGq, dGs = quant_block(dG, 1, 128)
    dUq, dUs = quant_block(dU, 1, 128)
    dX = dgrad_gateup(dGq, dGs, dUq, dUs, expert, Wg, Wu)
    dx = unpermute_reduce(bf16_to_f64(dX), pos)
    hqT, hsT = quant_rows128(fw["h"])
    xqT, xsT = quant_rows128(fw["Xp"])
    dGqT, dGsT = quant_rows128(dG)
    dUqT, dUsT = quant_rows128(dU)
    D = x_bf16.shape[1]
    I = fw["h"].shape[1]
    dWd = np.zeros((E, D, I))
    dWg = np.zeros((E, I, D))
    dWu = np.zeros((E, I, D))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        dWd[e] = wgrad_expert(dYqT, dYsT, hqT, hsT, r0, r1)
        dWg[e] = wgrad_expert(dGqT, dGsT, xqT, xsT, r0, r1)
        dWu[e] = wgrad_expert(dUqT, dUsT, xqT, xsT, r0, r1)
    return dict(d_w=d_w, dz=dz, dYr=dYr, dYq=dYq, dYs=dYs, dYqT=dYqT, dYsT=dYsT, dH=dH,
                dG=dG, dU=dU, dGq=dGq, dGs=dGs, dUq=dUq, dUs=dUs, dGqT=dGqT, dGsT=dGsT,
                dUqT=dUqT, dUsT=dUsT, hqT=hqT, hsT=hsT, xqT=xqT, xsT=xsT,
                dX=dX, dx=dx, dWd=dWd, dWg=dWg, dWu=dWu)


# --------------------------------------------------------------------------
# unquantised, unrounded layer (for the autograd and finite-difference pins)
# --------------------------------------------------------------------------

def forward_exact(x, idx, w, Wg, Wu, Wd):
    """Same composition with every operand fp64 and no rounding point."""
    T, k = idx.shape
    E = Wg.shape[0]
    y = np.zeros((T, x.shape[1]))
    for j in range(k):
        e = idx[:, j].astype(np.int32)
        g = rowdot(x, e, Wg)
        u = rowdot(x, e, Wu)
        Y = rowdot(silu(g) * u, e, Wd)
        y += w[:, j:j + 1] * Y
    return y


def backward_exact(x, idx, w, Wg, Wu, Wd, dy, z=None):
    """Exact gradients of sum(dy * forward_exact) w.r.t. x, W*, w and z."""
    T, k = idx.shape
    E = Wg.shape[0]
    dx = np.zeros_like(x)
    dWg = np.zeros_like(Wg)
    dWu = np.zeros_like(Wu)
    dWd = np.zeros_like(Wd)
    d_w = np.zeros((T, k))
    for j in range(k):
        e = idx[:, j].astype(np.int32)
        g = rowdot(x, e, Wg)
        u = rowdot(x, e, Wu)
        h = silu(g) * u
        Y = rowdot(h, e, Wd)
        d_w[:, j] = (dy * Y).sum(axis=1)
        dYr = w[:, j:j + 1] * dy
        dH = rowdot(dYr, e, Wd, trans=True)
        s = 1.0 / (1.0 + np.exp(-g))
        dg = dH * u * s * (1.0 + g * (1.0 - s))
        du = dH * g * s
        dx += rowdot(dg, e, Wg, trans=True) + rowdot(du, e, Wu, trans=True)
        for ee in range(E):
            r = np.nonzero(e == ee)[0]
            if len(r) == 0:
                continue
            dWd[ee] += wgrad(dYr[r], h[r])
            dWg[ee] += wgrad(dg[r], x[r])
            dWu[ee] += wgrad(du[r], x[r])
    dz = None
    if z is not None:
        zS = np.take_along_axis(z, idx.astype(np.int64), axis=1)
        p = np.exp(zS - zS.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        inner = (p * d_w).sum(axis=1, keepdims=True)
        dz = np.zeros_like(z)
        np.put_along_axis(dz, idx.astype(np.int64), p * (d_w - inner), axis=1)
    return dict(dx=dx, dWg=dWg, dWu=dWu, dWd=dWd, d_w=d_w, dz=dz)
