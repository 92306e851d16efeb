"""Seeded synthetic inputs for the MoE expert layer workloads.

This module only draws random inputs; it holds none of the layer's arithmetic.
Both the CUDA path's tests/benchmark and the CPU oracle's tests take their
inputs from here.

Recipe (numpy ``default_rng(seed)``, PCG64; draw order: routing -> x ->
W_gate -> W_up -> W_down -> dy):

* normals are drawn in fp32 and rounded to bf16 (round to nearest even);
* x ~ N(0, 1) (``x_std`` scales it), weights ~ N(0, 0.02), dy ~ 0.01 N(0, 1);
* routing, per workload:
  - ``topk_normal``: router logits N(0, 1) fp32 [T, E];
  - ``replay_zipf``: a replay payload int32 [L, k, T]; expert popularity
    p_e ~ (e+1)^-s; each token draws k distinct experts by Gumbel keys
    (log p + Gumbel, the k largest keys, i.e. sampling without replacement);
    weights Dirichlet(1) per token (normalised Exp(1));
  - ``topk_zipf_skew``: router logits log p_e + Gumbel with p_e ~ (e+1)^-s,
    and the ``empty`` least popular experts at p = 0 (logit -inf), so the
    router itself samples the skewed, partly empty load;
  - ``replay_uniform``: inference logits U(0, 1) fp32; the payload is their
    top-k order; the trainer's logits are the inference logits plus
    0.05 N(0, 1), so replay must override the trainer's own choice;
  - ``replay_skew``: the same with inference logits log p_e + Gumbel,
    p_e ~ (e+1)^-s (hot and cold experts).
  The replay payloads are drawn here, as inputs, so that the kernels and the
  oracle replay the same routing; the library's own router and capture
  (moe_router_fwd, moe_capture_payload) are checked on their own.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    D: int
    I: int
    E: int
    k: int
    routing: str
    L: int = 1
    x_std: float = 1.0
    zipf: float = 0.0
    empty: int = 0
    train: bool = False

    @property
    def R(self) -> int:
        return self.T * self.k

    def fwd_flop(self) -> float:
        """Algorithmic FLOP of the three expert GEMMs (routed rows only)."""
        return 6.0 * self.R * self.D * self.I


WORKLOADS = {
    "tiny": Workload("tiny", T=256, D=256, I=128, E=8, k=2, routing="topk_normal"),
    "replay": Workload("replay", T=4096, D=2048, I=1024, E=64, k=6, routing="replay_zipf",
                       L=4, zipf=1.1),
    "shard": Workload("shard", T=16384, D=7168, I=2048, E=32, k=8, routing="topk_normal",
                      x_std=0.5),
    "prefill": Workload("prefill", T=131072, D=6144, I=2048, E=32, k=8,
                        routing="topk_zipf_skew", zipf=1.2, empty=4),
    "train": Workload("train", T=32768, D=7168, I=2048, E=32, k=8, routing="replay_uniform",
                      train=True),
    "train_skew": Workload("train_skew", T=32768, D=7168, I=2048, E=32, k=8, routing="replay_skew",
                           zipf=1.2, train=True),
}


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _normal_bf16(rng, shape, std: float) -> np.ndarray:
    a = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return to_bf16_bits(a)


def _gumbel(rng, shape) -> np.ndarray:
    u = rng.random(shape, dtype=np.float64)
    u = np.clip(u, 1e-300, 1.0)
    return -np.log(-np.log(u))


def _draw_routing(rng, wl: Workload, T: int) -> dict:
    E, k = wl.E, wl.k
    if wl.routing == "topk_normal":
        return {"logits": rng.standard_normal((T, E), dtype=np.float32)}
    if wl.routing == "topk_zipf_skew":
        p = (np.arange(1, E + 1, dtype=np.float64)) ** (-wl.zipf)
        logp = np.log(p / p.sum())
        if wl.empty:
            logp[E - wl.empty:] = -np.inf
        z = logp[None, :] + _gumbel(rng, (T, E))
        return {"logits": z.astype(np.float32)}
    if wl.routing == "replay_zipf":
        p = (np.arange(1, E + 1, dtype=np.float64)) ** (-wl.zipf)
        logp = np.log(p / p.sum())
        payload = np.empty((wl.L, k, T), np.int32)
        w_in = np.empty((wl.L, T, k), np.float32)
        for layer in range(wl.L):
            keys = logp[None, :] + _gumbel(rng, (T, E))
            chosen = np.argsort(-keys, axis=1, kind="stable")[:, :k]
            payload[layer] = chosen.T.astype(np.int32)
            g = rng.standard_exponential((T, k))
            w_in[layer] = (g / g.sum(axis=1, keepdims=True)).astype(np.float32)
        return {"payload": payload, "w_in": w_in}
    if wl.routing in ("replay_uniform", "replay_skew"):
        if wl.routing == "replay_uniform":
            z_inf = rng.random((T, E), dtype=np.float32)
        else:
            p = (np.arange(1, E + 1, dtype=np.float64)) ** (-wl.zipf)
            z_inf = (np.log(p / p.sum())[None, :] + _gumbel(rng, (T, E))).astype(np.float32)
        chosen = np.argsort(-z_inf, axis=1, kind="stable")[:, :k]
        payload = chosen.T[None].astype(np.int32).copy()
        z_train = (z_inf + np.float32(0.05) * rng.standard_normal((T, E), dtype=np.float32))
        return {"payload": payload, "logits": z_train.astype(np.float32)}
    raise ValueError(wl.routing)


def make_inputs(wl: Workload | str, seed: int = 0, T: int | None = None,
                weights: bool = True, dy: bool | None = None, E: int | None = None) -> dict:
    """Draw one workload's inputs.  ``T`` and ``E`` override the token and
    expert counts (for small cases of the same recipe).  bf16 tensors come
    back as uint16 bit patterns; shapes: x [T, D], W_gate/W_up [E, I, D],
    W_down [E, D, I], dy [T, D]."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    if T is not None:
        wl = dataclasses.replace(wl, T=T)
    if E is not None:
        wl = dataclasses.replace(wl, E=E)
    rng = np.random.default_rng(seed)
    out = {"workload": wl}
    out.update(_draw_routing(rng, wl, wl.T))
    out["x"] = _normal_bf16(rng, (wl.T, wl.D), wl.x_std)
    if weights:
        out["W_gate"] = _normal_bf16(rng, (wl.E, wl.I, wl.D), 0.02)
        out["W_up"] = _normal_bf16(rng, (wl.E, wl.I, wl.D), 0.02)
        out["W_down"] = _normal_bf16(rng, (wl.E, wl.D, wl.I), 0.02)
    if dy is None:
        dy = wl.train
    if dy:
        out["dy"] = _normal_bf16(rng, (wl.T, wl.D), 0.01)
    return out


def replace(wl: Workload, **kw) -> Workload:
    return dataclasses.replace(wl, **kw)
