"""Router logits, capture of the routing payload, and the router gradients, in
fp64 — TEST INFRASTRUCTURE ONLY.

Source: "RL at 1T scale: prime-rl performance deep dive", §Router Replay: the
inference engine records, per layer, which experts the router chose for each
token; the trainer receives that record as an integer tensor of shape
[num_layers, top_k, seq_len] and replays it instead of routing again.  The
router itself is the plain linear gate of an MoE layer: logits z = W_r x over
the E experts, then the top-k of a1.

Readings (the pages give no formula for the router):

* z[t, e] = sum_d x[t, d] * W_r[e, d] over bf16 x and W_r, accumulated in
  fp64 here (the kernel accumulates in fp32; z is compared within the float
  tolerance, and the top-k decision is compared on the kernel's own z);
* the payload stores slot j of token t of layer l at (l * k + j) * T + t
  (row-major [L][k][T], seq_len fastest), the layout replay reads;
* the router backward: dx_r[t, d] = sum_e dz[t, e] * W_r[e, d] and
  dW_r[e, d] = sum_t dz[t, e] * x[t, d], with dz the gradient of the logits
  (zero off the chosen set).
"""
from __future__ import annotations

import numpy as np

from . import bf16_to_f64, rowdot, wgrad


def router_logits(x_bf16, Wr_bf16) -> np.ndarray:
    """z [T, E] (fp64) = x W_r^T over the bf16 operands."""
    x = bf16_to_f64(x_bf16)
    W = bf16_to_f64(Wr_bf16)
    return rowdot(x, np.zeros(x.shape[0], np.int32), W[None])


def capture_payload(idx_per_layer) -> np.ndarray:
    """The [num_layers, top_k, seq_len] record of the chosen experts: one
    [T, k] index array per layer in, payload[l, j, t] = idx_l[t, j] out."""
    L = len(idx_per_layer)
    T, k = np.asarray(idx_per_layer[0]).shape
    payload = np.empty((L, k, T), np.int32)
    for l in range(L):
        idx = np.asarray(idx_per_layer[l], np.int32)
        for j in range(k):
            payload[l, j, :] = idx[:, j]
    return payload


def router_backward(x_bf16, Wr_bf16, dz):
    """(dx_r [T, D], dW_r [E, D]) in fp64 from the logit gradient dz [T, E]."""
    x = bf16_to_f64(x_bf16)
    W = bf16_to_f64(Wr_bf16)
    dz = np.asarray(dz, np.float64)
    dx = rowdot(dz, np.zeros(dz.shape[0], np.int32), W[None], trans=True)
    dW = wgrad(dz, x)
    return dx, dW
