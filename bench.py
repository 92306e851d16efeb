"""Benchmark of the MoE expert layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|replay|shard|train]

Workload (default): the long-sequence prefill chunk forward — T=131072 tokens,
d_model=6144, expert FFN I=2048 (SiLU-gated), E=32 experts, top-8 routing from
router logits log p + Gumbel with Zipf(1.2) expert popularity and the 4 least
popular experts empty (logit -inf), bf16 N(0,1) activations, N(0,0.02)
weights quantised once to 128x128 FP8 blocks.  It is the largest
configuration of the layer that fits one GPU.  One step = one layer forward:
top-k routing -> permute + FP8 dispatch -> grouped GEMM gate/up + SiLU +
h-quant -> grouped GEMM down -> weighted combine.  value = tokens / step time.
``--workload replay`` times the router-replay forward instead (T=4096, L=4
replayed layers of a [4, 6, 4096] payload, one set of weights).

N > 1 (torchrun, one rank per GPU): replicas — every rank runs its own batch
(seed + rank) with the same weights; the layer has no cross-GPU exchange in
data parallelism.  Timing is on the device, max over ranks.

The roofline denominator of the grouped GEMMs is the dense FP8 peak measured
in the same process: torch._scaled_mm (cuBLAS) on e4m3 8192^3 with tensor-wise
scales and bf16 output, best of 10 single calls (burst) and a 4 s loop
(sustained).

--impl reference times the CPU oracle (test infrastructure, fp64) on the host
cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; grouped FP8 GEMM TFLOP/s as % of dense FP8 peak"
UNIT = "tokens/s"
FP8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s), used only when no FP8 peak was measured
FP4_OVER_FP8 = 2.0   # nominal dense ratio (9 / 4.5 PFLOP/s): the FP4 peak is this times the measured FP8 peak

# DRAM traffic (read + write bytes) of one gate/up GEMM launch per workload,
# from an ncu capture of dram__bytes_read.sum + dram__bytes_write.sum on that
# kernel.  Valid only for the kernel sources it was taken on: reported as null
# as soon as their hash differs.
GEMM1_TRAFFIC = {
    "prefill": {"sources_sha256_16": "262bd4a4ae5c7163", "bytes": 8.02e9 + 2.22e9},
}


def _gemm_sources_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm_sm100.cu", "sm100.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "moe_expert_layer_replay_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return pk["hbm_gbs"], pk["bf16_tflops"], pk.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def measure_fp8_peak(seconds: float = 4.0) -> dict:
    """Dense FP8 (e4m3) GEMM throughput of cuBLAS through torch._scaled_mm:
    8192^3, tensor-wise scales, bf16 output; the faster of the two
    accumulation modes.  burst = best of 10 single calls; sustained = a
    back-to-back loop of about ``seconds``."""
    import torch
    M = N = K = 8192
    g = torch.Generator(device="cuda").manual_seed(0)
    a = (torch.randn(M, K, device="cuda", generator=g) * 0.5).to(torch.float8_e4m3fn)
    b = (torch.randn(N, K, device="cuda", generator=g) * 0.5).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device="cuda")
    flop = 2.0 * M * N * K
    best = {}
    for fast in (False, True):
        f = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16,
                                     use_fast_accum=fast)
        for _ in range(5):
            f()
        torch.cuda.synchronize()
        t = []
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            e1.synchronize()
            t.append(e0.elapsed_time(e1))
        best[fast] = (flop / (min(t) * 1e-3) / 1e12, f)
    fast = max(best, key=lambda k: best[k][0])
    burst, f = best[fast]
    n, t0 = 0, time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    while time.time() - t0 < seconds:
        for _ in range(25):
            f()
        n += 25
        torch.cuda.synchronize()
    e1.record()
    e1.synchronize()
    sustained = n * flop / (e0.elapsed_time(e1) * 1e-3) / 1e12
    del a, b
    return {"burst_tflops": burst, "sustained_tflops": sustained, "use_fast_accum": fast,
            "method": "torch._scaled_mm e4m3 8192^3, tensor-wise scales, bf16 out; burst = best of 10, "
                      f"sustained = {n} back-to-back calls"}


def _workload_desc(wl):
    return (f"{wl.name}: T={wl.T} D={wl.D} I={wl.I} E={wl.E} k={wl.k} L={wl.L} routing={wl.routing}"
            + (f" zipf={wl.zipf}" if wl.zipf else "") + (f" empty={wl.empty}" if wl.empty else ""))


class Clocks:
    """nvidia-smi sampling (every 20 ms, with timestamps) of SM clocks and
    throttle reasons; stop() keeps the samples taken between mark() and the
    stop call (warm-up plus the timed steps: the same work)."""

    def __init__(self, index: int, path: str):
        self.path = path
        self.p = None
        self.t0 = None
        q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(path, "w")
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={q}",
                                       "--format=csv,noheader,nounits", "-lms", "20"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.5)  # let the sampler start before the region of interest
        except Exception:
            self.p = None

    def mark(self):
        import datetime
        self.t0 = datetime.datetime.now()

    def stop(self):
        import datetime
        if self.p is None:
            return None
        t1 = datetime.datetime.now()
        time.sleep(0.1)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                if self.t0 is not None and not (self.t0 <= ts <= t1):
                    continue
                sm.append(float(parts[2]))
                mx.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "window": "warm-up and timed steps"}


# --------------------------------------------------------------------------
# multi-rank plumbing (replicas: no data-path collective)
# --------------------------------------------------------------------------

def replica_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch of the workload."""
    return seed + rank


def reduce_max(value: float) -> float:
    """Max over ranks (the step time every rank must wait for); identity on
    one process.  Uses the process group's backend (NCCL: a CUDA tensor)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, units_per_rank: float, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return world * units_per_rank / max_seconds


# --------------------------------------------------------------------------
# reference arm / CPU baseline: the oracle on host cores
# --------------------------------------------------------------------------

def oracle_route(inp, layer: int = 0):
    """The workload's routing through the oracle: replay of the payload (with
    the given weights, or the trainer logits) or top-k of the router logits."""
    import oracle
    wl = inp["workload"]
    if "payload" in inp:
        if "w_in" in inp:
            idx, w, st = oracle.route_replay(inp["payload"], layer, wl.E, w_in=inp["w_in"][layer])
        else:
            idx, w, st = oracle.route_replay(inp["payload"], layer, wl.E, z=inp["logits"])
        assert st == 0
        return idx, w
    return oracle.route_topk(inp["logits"], wl.k)


def oracle_sample_step(inp, wq, tokens: int, layer: int = 0):
    """One bounded sample of the workload through the oracle: routing and
    permute of all T tokens of layer `layer`, then the expert FFN and combine
    of `tokens` evenly spaced tokens."""
    from oracle import layer as OL
    wl = inp["workload"]
    idx, w = oracle_route(inp, layer)
    sample = np.arange(tokens) * (wl.T // tokens)
    return OL.forward_tokens(inp["x"], idx, w, wq, sample)["y"]


def oracle_weights(inp):
    from oracle import layer as OL
    return (OL.quant_weights(inp["W_gate"]), OL.quant_weights(inp["W_up"]), OL.quant_weights(inp["W_down"]))


def default_sample_tokens(wl, budget_flop: float) -> int:
    """Tokens of a bounded oracle sample: about ``budget_flop`` fp64 FLOPs of
    expert FFN (6*k*D*I per token), a power of two between 16 and 1024.  At
    the oracle's rate on 16 host cores (about 40 fp64 GFLOP/s) the bench's
    sample (1.2e12) takes 10-30 s."""
    n = budget_flop / (6.0 * wl.k * wl.D * wl.I)
    p = 16
    while p * 2 <= min(n, 1024):
        p *= 2
    return p


def cpu_baseline(inp, tokens: int, reps: int = 1):
    import oracle
    wq = oracle_weights(inp)
    t0 = time.perf_counter()
    for r in range(reps):
        oracle_sample_step(inp, wq, tokens, layer=r % inp["workload"].L)
    dt = time.perf_counter() - t0
    return {"value": reps * tokens / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"routing + permute of all tokens, then expert FFN + combine of {tokens} evenly spaced "
                      f"tokens x {reps} layer pass(es) of the same workload through the fp64 oracle (weights "
                      f"quantised once, outside the timing); {dt:.1f} s"}


def run_reference(args, wl_name):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from moe_expert_layer_replay_b200.inputs import make_inputs
    inp = make_inputs(wl_name, seed=args.seed, T=args.tokens)
    wl = inp["workload"]
    tokens = args.ref_tokens or default_sample_tokens(wl, 4e10)
    wq = oracle_weights(inp)
    for _ in range(args.warmup):
        oracle_sample_step(inp, wq, tokens)
    times = []
    for s in range(args.steps):
        t0 = time.perf_counter()
        oracle_sample_step(inp, wq, tokens, layer=s % wl.L)
        times.append(time.perf_counter() - t0)
    import oracle
    tot = sum(times)
    val = args.steps * tokens / tot
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": _workload_desc(wl), "sample_tokens_per_step": tokens},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"routing + permute of all tokens, expert FFN + combine of {tokens} "
                                       "evenly spaced tokens per step"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def _to_dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


class RoutingInput:
    """The routing input of one step on the device (payload + weights or
    trainer logits for replay, router logits for top-k) and the call that
    routes layer l from it."""

    def __init__(self, inp, dev=True):
        import torch
        self.keys = [k for k in ("payload", "w_in", "logits") if k in inp]
        self.t = {k: (_to_dev(inp[k]) if dev else torch.from_numpy(np.ascontiguousarray(inp[k])).pin_memory())
                  for k in self.keys}

    def route(self, B, l):
        from moe_expert_layer_replay_b200 import layer
        t = self.t
        if "payload" in t:
            layer.route(B, payload=t["payload"], layer=l, w_in=t["w_in"][l] if "w_in" in t else None,
                        logits=t.get("logits"))
        else:
            layer.route(B, logits=t["logits"])

    def nbytes(self):
        return sum(v.numel() * v.element_size() for v in self.t.values())

    def copy_from(self, other, stream):
        for k in self.keys:
            self.t[k].copy_(other.t[k], non_blocking=True)


def forward_calls(B, x, W, d, gather: bool, gemm1_events=None, stream=None):
    """The layer's forward after routing, call by call (as layer.forward), with
    the gate/up GEMM bracketed by CUDA events when a list is given."""
    import torch

    from moe_expert_layer_replay_b200 import abi
    if gather:
        abi.quant_fp8_block(x, d.T, d.D, d.D, 1, 128, B.xq_tok, B.xs_tok)
        abi.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, None, None, None, None, None, B.ws)
    else:
        abi.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, x, B.xq, B.xs, None, None, B.ws)
    if gemm1_events is not None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
    if gather:
        abi.gateup_gather_fp8(d, B.offsets, B.src, B.xq_tok, B.xs_tok, W.wgu_q, W.wgu_s, out_q=B.hq, out_s=B.hs)
    else:
        abi.grouped_gemm_fp8(abi.GEMM_GATEUP_SILU, d, B.offsets, B.xq, B.xs, W.wgu_q, W.wgu_s,
                             out_q=B.hq, out_s=B.hs)
    if gemm1_events is not None:
        e1.record(stream)
        gemm1_events.append((e0, e1))
    abi.grouped_gemm_fp8(abi.GEMM_DOWN, d, B.offsets, B.hq, B.hs, W.wd_q, W.wd_s, out_bf16=B.Y)


def run_ours(args, wl_name):
    import torch
    import torch.distributed as dist

    from moe_expert_layer_replay_b200 import abi, layer
    from moe_expert_layer_replay_b200.inputs import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    abi.lib()

    inp = make_inputs(wl_name, seed=replica_seed(args.seed, rank), T=args.tokens)
    wl = inp["workload"]
    d = abi.dims(wl.T, wl.D, wl.I, wl.E, wl.k)
    W = layer.quantise_weights(d, _to_dev(inp["W_gate"]), _to_dev(inp["W_up"]), _to_dev(inp["W_down"]),
                               train=False)
    gather = args.dispatch == "gather"
    B = layer.Buffers(d, "cuda", train=False, gather=gather)
    x = _to_dev(inp["x"])
    rt = RoutingInput(inp)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    gemm1_events = []

    def step(timed_gemm: bool):
        for l in range(wl.L):
            rt.route(B, l)
            forward_calls(B, x, W, d, gather, gemm1_events if timed_gemm else None, stream)
            abi.combine(B.Y, B.w, B.pos, d, B.y)

    for _ in range(max(3, args.warmup)):
        step(False)
    torch.cuda.synchronize()
    st = abi.get_status()
    if st != abi.OK:
        raise RuntimeError(f"device status after warm-up: {abi.strerror(st)}")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # One step captured as a CUDA graph (all launches of the L layers); the
    # timed steps replay it.  The gate/up GEMM is timed live in separate eager
    # steps right after.
    graph = None
    n0 = abi.kernel_launches()
    if not args.no_graph:
        gs = torch.cuda.Stream()
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            step(False)  # every first-call set-up happens before capture
        torch.cuda.current_stream().wait_stream(gs)
        torch.cuda.synchronize()
        n0 = abi.kernel_launches()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(False)
        torch.cuda.synchronize()
    launches_per_step = abi.kernel_launches() - n0 if graph is not None else None

    import tempfile
    clocks_dir = os.environ.get("MOE_BENCH_CLOCKS_DIR", tempfile.gettempdir())  # raw nvidia-smi samples
    clocks = Clocks(local, os.path.join(clocks_dir, f"moe_clocks_rank{rank}.csv"))
    barrier()
    clocks.mark()
    n1 = abi.kernel_launches()
    step_ms = []
    for _ in range(args.steps):
        flush.fill_(1)  # L2 flush between timed steps, outside the events
        e0, e1 = ev(), ev()
        e0.record(stream)
        if graph is not None:
            graph.replay()
        else:
            step(True)
        e1.record(stream)
        step_ms.append((e0, e1))
    barrier()
    clk = clocks.stop()
    if graph is None:
        launches_per_step = (abi.kernel_launches() - n1) / args.steps
    step_ms = [a.elapsed_time(b) for a, b in step_ms]
    if graph is not None:  # the dominant kernel's launch duration, same workload, eager
        for _ in range(min(args.steps, 5)):
            flush.fill_(1)
            step(True)
        torch.cuda.synchronize()
    g1_ms = [a.elapsed_time(b) for a, b in gemm1_events]
    tot_ms = reduce_max(sum(step_ms))
    ms_per_step = tot_ms / args.steps
    value = aggregate_rate(world, wl.L * wl.T * args.steps, tot_ms / 1e3)
    del graph

    # ---------------- end to end through the public API with host buffers:
    # every step copies its inputs (x, routing input) from pinned host memory
    # and every layer's output y back.  The copies run on two copy streams
    # ordered by events (double-buffered inputs; one y buffer per layer), so
    # they overlap the layer's kernels.
    e2e_val, h2d, d2h = e2e_run(args, wl, d, W, inp, world, barrier, gather)

    st = abi.get_status()
    if st != abi.OK:
        raise RuntimeError(f"device status after timing: {abi.strerror(st)}")

    fp8 = measure_fp8_peak() if rank == 0 else None
    if rank == 0:
        hbm, bf16_tf, bf16_sus, src = _peaks()
        fp8_peak = fp8["burst_tflops"]
        R = wl.T * wl.k
        g1_flop = 2.0 * R * wl.D * (2 * wl.I)
        g1_avg = statistics.mean(g1_ms)
        achieved = g1_flop / (g1_avg / 1e3) / 1e12
        gemm_tflops = wl.fwd_flop() * wl.L / (ms_per_step / 1e3) / 1e12  # whole-step view (lower bound)
        tr = GEMM1_TRAFFIC.get(wl.name)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": _workload_desc(wl), "tokens_per_step_per_gpu": wl.L * wl.T,
                       "launch": "CUDA graph of one step" if not args.no_graph else "eager",
                       "l2": "flushed between timed steps (512 MiB write, outside the timed events)",
                       "dispatch": "gate/up GEMM gathers the token rows" if gather else "permuted FP8 copy",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "roofline": {"bound": "tensor", "kernel": "grouped_gemm gate/up + SiLU + h-quant",
                         "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s", "frac": achieved / fp8_peak,
                         "traffic": (tr["bytes"] if tr and _gemm_sources_hash() == tr["sources_sha256_16"]
                                     else None),
                         "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                         "peak_note": "measured dense FP8 burst (cuBLAS torch._scaled_mm, this process)",
                         "frac_of_sustained": achieved / fp8["sustained_tflops"],
                         "frac_of_fp8_spec_4500": achieved / 4500.0,
                         "algorithmic": f"2*R*D*2I = {g1_flop:.4g} FLOP per launch (R = T*k routed rows)",
                         "avg_launch_ms": g1_avg},
            "fp8_peak": fp8,
            "gemm_tflops_step": gemm_tflops,
            "gemm_frac_fp8_peak_step": gemm_tflops / fp8_peak,
            "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "note": "inputs copied from pinned host memory and y copied back every step, overlapped "
                            "with the kernels on two copy streams"},
            "gpu_launches": int(round(launches_per_step * args.steps)),
            "gpu_launches_note": f"{launches_per_step:g} library kernel launches per step (counted by the "
                                 "library during capture) x steps",
            "clocks": clk,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(inp, args.cpu_tokens or default_sample_tokens(wl, 1.2e12))
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def e2e_run(args, wl, d, W, inp, world, barrier, gather=False):
    """Same metric through the public API with host buffers.  Returns
    (tokens/s over all ranks, H2D bytes per step, D2H bytes per step)."""
    import torch

    from moe_expert_layer_replay_b200 import abi, layer

    B = layer.Buffers(d, "cuda", train=False, gather=gather)
    xh = torch.from_numpy(inp["x"].view(np.int16)).pin_memory()
    rth = RoutingInput(inp, dev=False)
    xd = [torch.empty(wl.T, wl.D, dtype=torch.int16, device="cuda") for _ in range(2)]
    rtd = [RoutingInput(inp) for _ in range(2)]
    yd = [[torch.empty(wl.T, wl.D, dtype=torch.bfloat16, device="cuda") for _ in range(wl.L)] for _ in range(2)]
    yh = torch.empty(wl.L, wl.T, wl.D, dtype=torch.int16).pin_memory()
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    Ev = torch.cuda.Event
    in_free = [None, None]     # the step two back has finished with input buffer s%2
    y_free = [None, None]      # the step two back has copied out output buffer s%2
    y_done = [None] * wl.L     # this step's layer-l output is on the host

    def one_step(s):
        b = s % 2
        with torch.cuda.stream(s_in):
            if in_free[b] is not None:
                s_in.wait_event(in_free[b])
            xd[b].copy_(xh, non_blocking=True)
            rtd[b].copy_from(rth, s_in)
            h2d_done = Ev()
            h2d_done.record(s_in)
        comp.wait_event(h2d_done)
        if y_free[b] is not None:
            comp.wait_event(y_free[b])
        x = xd[b].view(torch.bfloat16)
        for l in range(wl.L):
            rtd[b].route(B, l)
            forward_calls(B, x, W, d, gather)
            abi.combine(B.Y, B.w, B.pos, d, yd[b][l])
            y_ready = Ev()
            y_ready.record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(y_ready)
                yh[l].copy_(yd[b][l].view(torch.int16), non_blocking=True)
                y_done[l] = Ev()
                y_done[l].record(s_out)
        in_free[b] = Ev()
        in_free[b].record(comp)
        y_free[b] = y_done[wl.L - 1]   # the copy stream runs the layers' copies in order

    for s in range(2):
        one_step(s)
    barrier()
    e0, e1 = Ev(enable_timing=True), Ev(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    for s in range(args.steps):
        one_step(s)
    comp.wait_event(y_done[wl.L - 1])
    e1.record(comp)
    barrier()
    ms = reduce_max(e0.elapsed_time(e1))
    val = aggregate_rate(world, wl.L * wl.T * args.steps, ms / 1e3)
    h2d = xh.numel() * 2 + rth.nbytes()
    d2h = yh.numel() * 2
    del B
    return val, h2d, d2h


def nvfp4_stages(abi, d, B, x, wg, wu, R_pad):
    """The NVFP4 variant of the gate/up GEMM (f4) as extra report stages: the
    permuted rows of x and each expert's [W_gate; W_up] quantised to NVFP4
    (scales in the block-scaled MMA's layout), then the grouped NVFP4 GEMM
    with fp32 output.  The permuted bf16 rows are gathered by torch once,
    outside the timed stages (input preparation only)."""
    import torch
    D, I, E = d.D, d.I, d.E
    R_cap = B.R_cap
    src = B.src[:R_cap].long()
    rows = torch.zeros(R_cap, D, dtype=torch.bfloat16, device="cuda")
    ok = src >= 0
    rows[ok] = x[src[ok] // d.k]
    wgu = torch.cat([wg, wu], dim=1).contiguous()          # [E][2I][D]
    q = torch.empty(R_cap, D // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(4 * R_cap * D // 16, dtype=torch.uint8, device="cuda")
    amax = torch.empty(1, device="cuda")
    sg = torch.empty(1, device="cuda")
    wq = torch.empty(E, 2 * I, D // 2, dtype=torch.uint8, device="cuda")
    wsf = torch.empty(E, 4 * 2 * I * D // 16, dtype=torch.uint8, device="cuda")
    wamax = torch.empty(E, device="cuda")
    wsg = torch.empty(E, device="cuda")
    for e in range(E):
        abi.quant_nvfp4(wgu[e], 2 * I, D, D, wq[e], wsf[e], wamax[e:e + 1], wsg[e:e + 1],
                        sf_layout=abi.NVFP4_SF_MMA_B)
    out = torch.empty(R_cap, 2 * I, dtype=torch.float32, device="cuda")
    return [
        ("NVFP4 quant of the permuted rows", lambda: abi.quant_nvfp4(rows, R_cap, D, D, q, sf, amax, sg,
                                                                      sf_layout=abi.NVFP4_SF_MMA_A),
         "B", 2 * 2 * R_cap * D + R_cap * (D // 2 + 4 * D // 16)),
        ("gemm gate/up NVFP4 (fp32 out)", lambda: abi.gemm_nvfp4(R_cap, 2 * I, D, E, B.offsets, q, sf, sg, wq, wsf,
                                                                  wsg, out),
         "F4", 4.0 * d.T * d.k * D * I),
    ]


def run_kernels(args, names):
    """Per-stage device time of one layer pass for each named workload (the
    stages of the hot path, forward and, for the training workload, backward):
    each stage is captured N times in its own CUDA graph and replayed after an
    L2 flush; the median over replays / N is its time.  Each stage reports its
    algorithmic bytes or FLOPs (R = T*k routed rows) and the achieved fraction
    of the measured peak (HBM copy GB/s, or 2 x bf16 burst for FP8).  One JSON
    line per workload; not the bench line."""
    import torch

    from moe_expert_layer_replay_b200 import abi, layer
    from moe_expert_layer_replay_b200.inputs import make_inputs

    torch.cuda.set_device(0)
    abi.lib()
    hbm, bf16_tf, _, src = _peaks()
    fp8 = bf16_tf * FP8_OVER_BF16
    fp8_src = src + " (2 x bf16)"
    if not args.once:   # the FP8 GEMM peak measured in this process, as the bench line does
        fp8 = measure_fp8_peak(seconds=1.0)["burst_tflops"]
        fp8_src = "measured dense FP8 burst (cuBLAS torch._scaled_mm, this process)"
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    for name in names:
        inp = make_inputs(name, seed=args.seed, T=args.tokens, E=args.experts)
        wl = inp["workload"]
        T, D, I, E, k = wl.T, wl.D, wl.I, wl.E, wl.k
        R = T * k
        d = abi.dims(T, D, I, E, k)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else
                                         np.ascontiguousarray(a)).cuda()
        bfd = lambda a: dev(a).view(torch.bfloat16)
        train = wl.train
        wg, wu, wd = bfd(inp["W_gate"]), bfd(inp["W_up"]), bfd(inp["W_down"])
        W = layer.quantise_weights(d, wg, wu, wd, train=train)
        B = layer.Buffers(d, "cuda", train=train, gather=True)
        x = bfd(inp["x"])
        if "payload" in inp:
            P = dev(inp["payload"])
            w_in = dev(inp["w_in"][0]) if "w_in" in inp else None
            z = dev(inp["logits"]) if "logits" in inp else None
            route = lambda: layer.route(B, payload=P, layer=0, w_in=w_in, logits=z)
            route_bytes = 4 * R + (4 * R if w_in is not None else 4 * T * E) + 8 * R
        else:
            z = dev(inp["logits"])
            route = lambda: layer.route(B, logits=z)
            route_bytes = 4 * T * E + 8 * R
        route()
        abi.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, None, None, None, None, None, B.ws)
        torch.cuda.synchronize()
        R_pad = int(B.offsets[E].item())
        xT = (B.xqT, B.xsT) if train else (None, None)
        st = [
            ("route", route, "B", route_bytes),
            ("permute index", lambda: abi.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, None, None, None,
                                                  None, None, B.ws), "B", 8 * R + 4 * R_pad),
            ("permute index + dispatch quant", lambda: abi.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, x,
                                                                   B.xq, B.xs, xT[0], xT[1], B.ws), "B",
             8 * R + 4 * R_pad + 2 * T * D + R * (D + D // 32) + (R * (D + D // 32) if train else 0)),
            ("gemm gate/up + SiLU + h-quant", lambda: abi.grouped_gemm_fp8(
                abi.GEMM_GATEUP_SILU, d, B.offsets, B.xq, B.xs, W.wgu_q, W.wgu_s, aux=B.gu if train else None,
                out_q=B.hq, out_s=B.hs, out_bf16=B.h if train else None), "F", 4.0 * R * D * I),
            ("gemm down", lambda: abi.grouped_gemm_fp8(abi.GEMM_DOWN, d, B.offsets, B.hq, B.hs, W.wd_q, W.wd_s,
                                                       out_bf16=B.Y), "F", 2.0 * R * D * I),
            ("combine", lambda: abi.combine(B.Y, B.w, B.pos, d, B.y), "B", 2 * R * D + 8 * R + 2 * T * D),
            # the gathered dispatch: x quantised once per token row, rows gathered by the GEMM
            ("1x128 quant of the token rows", lambda: abi.quant_fp8_block(x, T, D, D, 1, 128, B.xq_tok, B.xs_tok),
             "B", 2 * T * D + T * (D + D // 32)),
            ("gemm gate/up gathering the token rows", lambda: abi.gateup_gather_fp8(
                d, B.offsets, B.src, B.xq_tok, B.xs_tok, W.wgu_q, W.wgu_s, out_q=B.hq, out_s=B.hs), "F",
             4.0 * R * D * I),
        ]
        if not args.once and D % 256 == 0:
            st += nvfp4_stages(abi, d, B, x, wg, wu, R_pad)
        if train:
            dy = bfd(inp["dy"])
            st += [
                ("weight quant (with transposes)", lambda: layer.quantise_weights(d, wg, wu, wd, train=True, out=W),
                 "B", 6 * E * D * I + 2 * 3 * E * D * I * (1 + 1 / 4096)),
                ("combine bwd", lambda: abi.combine_bwd(dy, B.Y, B.w, B.pos, B.idx, B.counts, B.offsets, d, B.dYq,
                                                        B.dYs, B.dYb, B.d_w, B.d_logits), "B",
                 2 * T * D + 2 * R * D + 8 * R + R * D * (1 + 1 / 32) + 2 * R * D),
                ("128x1 quant of dY", lambda: abi.quant_fp8_block(B.dYb, B.R_cap, D, D, 128, 1, B.dYqT, B.dYsT), "B",
                 2 * R * D + R * D * (1 + 1 / 32)),
                ("128x1 quant of h", lambda: abi.quant_fp8_block(B.h, B.R_cap, I, I, 128, 1, B.hqT, B.hsT), "B",
                 2 * R * I + R * I * (1 + 1 / 32)),
                ("gemm dgrad down + SiLU bwd", lambda: abi.grouped_gemm_fp8(
                    abi.GEMM_DGRAD_DOWN_SILU, d, B.offsets, B.dYq, B.dYs, W.wdT_q, W.wdT_s, aux=B.gu, out_q=B.dGUq,
                    out_s=B.dGUs, out_bf16=B.dGU), "F", 2.0 * R * D * I),
                ("128x1 quant of dGU", lambda: abi.quant_fp8_block(B.dGU, B.R_cap, 2 * I, 2 * I, 128, 1, B.dGUqT,
                                                                   B.dGUsT), "B",
                 4 * R * I + 2 * R * I * (1 + 1 / 32)),
                ("gemm dgrad gate/up", lambda: abi.grouped_gemm_fp8(
                    abi.GEMM_DGRAD_GATEUP, d, B.offsets, B.dGUq, B.dGUs, W.wguT_q, W.wguT_s, out_bf16=B.dX), "F",
                 4.0 * R * D * I),
                ("unpermute reduce", lambda: abi.unpermute_reduce(B.dX, B.pos, d, B.dx), "B", 2 * R * D + 2 * T * D),
                ("gemm wgrad down", lambda: abi.grouped_gemm_fp8(abi.GEMM_WGRAD_DOWN, d, B.offsets, B.dYqT, B.dYsT,
                                                                 B.hqT, B.hsT, out_f32=B.dWd), "F",
                 2.0 * R * D * I),
                ("gemm wgrad gate/up", lambda: abi.grouped_gemm_fp8(
                    abi.GEMM_WGRAD_GATEUP, d, B.offsets, B.dGUqT, B.dGUsT, B.xqT, B.xsT, out_f32=B.dWgu), "F",
                 4.0 * R * D * I),
            ]
        for _, f, _, _ in st:  # every stage once, in order (first-call set-up, valid operands)
            f()
        torch.cuda.synchronize()
        if abi.get_status() != abi.OK:
            raise RuntimeError("device status after the warm-up pass")
        if args.once:   # one eager launch of every stage (for a profiler), no timing
            print(json.dumps({"kernels_once": _workload_desc(wl), "stages": [n for n, _, _, _ in st]}), flush=True)
            del B, W, x
            torch.cuda.empty_cache()
            continue
        gs = torch.cuda.Stream()
        out = []
        for sname, f, kind, units in st:
            n = 10 if (kind == "B" or units < 1e12) else 2
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(gs):
                f()
                torch.cuda.synchronize()
                with torch.cuda.graph(g, stream=gs):
                    for _ in range(n):
                        f()
            torch.cuda.synchronize()
            ts = []
            for r in range(max(3, args.steps // 4)):
                flush.fill_(r & 0xFF)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) / n)
            del g
            ms = statistics.median(ts)
            if kind in ("F", "F4"):
                ach = units / (ms * 1e-3) / 1e12
                pk = fp8 * (FP4_OVER_FP8 if kind == "F4" else 1.0)
                out.append({"stage": sname, "us": round(ms * 1e3, 2), "flop": units, "tflops": round(ach, 1),
                            "frac": round(ach / pk, 4)})
                if kind == "F4":
                    out[-1]["peak_note"] = "dense FP4 = 2 x the measured FP8 peak (nominal 9 vs 4.5 PFLOP/s)"
            else:
                ach = units / (ms * 1e-3) / 1e9
                out.append({"stage": sname, "us": round(ms * 1e3, 2), "bytes": units, "gbs": round(ach, 1),
                            "frac": round(ach / hbm, 4)})
        torch.cuda.synchronize()
        if abi.get_status() != abi.OK:
            raise RuntimeError("device status after the timed replays")
        # (the gathered gate/up GEMM is an alternative to the copy path's, not an extra step)
        gf = [o for o in out if "flop" in o and "gathering" not in o["stage"] and "NVFP4" not in o["stage"]]
        line = {"kernels_report": _workload_desc(wl), "R": R, "R_pad": R_pad,
                "gemm_pair_clusters": abi.gemm_pair_clusters(),
                "peaks": {"hbm_gbs": hbm, "hbm_source": src, "fp8_tflops": fp8, "fp8_source": fp8_src},
                "gemm_tflops": round(sum(o["flop"] for o in gf) / (sum(o["us"] for o in gf) * 1e-6) / 1e12, 1),
                "stages": out}
        line["gemm_frac"] = round(line["gemm_tflops"] / fp8, 4)
        print(json.dumps(line), flush=True)
        del B, W, x
        torch.cuda.empty_cache()
    return 0


def build_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (a smaller case of the same workload, e.g. for profiling)")
    ap.add_argument("--experts", type=int, default=None,
                    help="with --kernels: override E (a smaller case of the same workload, e.g. for profiling)")
    ap.add_argument("--cpu-tokens", type=int, default=0, help="oracle sample size (0: sized to ~10 s)")
    ap.add_argument("--ref-tokens", type=int, default=0, help="oracle sample per reference step (0: ~1 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps eagerly")
    ap.add_argument("--dispatch", choices=["copy", "gather"], default="copy",
                    help="copy: the permute writes the permuted FP8 rows; gather: the gate/up GEMM gathers "
                         "them from the token rows")
    ap.add_argument("--gemm-variant", type=int, default=None,
                    help="grouped GEMM kernel: 0 one SM per tile, 1 the 2-SM MMA, -1 chosen per call "
                         "(default: the library's)")
    ap.add_argument("--once", action="store_true",
                    help="with --kernels: run every stage once, eagerly and untimed (for a profiler)")
    ap.add_argument("--kernels", default=None,
                    help="comma-separated workloads: per-stage device times and roofline fractions instead "
                         "of the bench line")
    return ap


def main():
    args = build_parser().parse_args()
    if args.gemm_variant is not None and args.impl == "ours":
        from moe_expert_layer_replay_b200 import abi
        abi.set_gemm_variant(args.gemm_variant)
    if args.kernels:
        return run_kernels(args, [w for w in args.kernels.split(",") if w])
    if args.impl == "reference":
        return run_reference(args, args.workload)
    return run_ours(args, args.workload)


if __name__ == "__main__":
    sys.exit(main())
