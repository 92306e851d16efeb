"""Expert parallelism (EP): the per-layer all-to-all dispatch of the routed
rows to the ranks that own their experts, and the all-to-all return of the
expert outputs before the combine ("RL at 1T scale: prime-rl performance deep
dive", §Parallelism strategy / EP: EP over the 8 GPUs of a node with an
all-to-all per layer; §Wide Expert Parallelism).

Rank r of N owns experts [r*E_loc, (r+1)*E_loc), E_loc = E / N, and its
weight arrays hold only those.  One layer forward on every rank:

1. route its own tokens over all E experts and permute them (moe_permute
   with the fused FP8 dispatch): rows grouped by expert in 128-row segments,
   so the rows bound for rank d are the contiguous permuted range
   [offsets[d*E_loc], offsets[(d+1)*E_loc]);
2. exchange the padded segment sizes (one all-to-all of N*E_loc integers):
   every rank then knows what it sends to and receives from every other;
3. dispatch: one all-to-all of the FP8 codes (rows of D bytes) and one of the
   1x128 scales (sent row-major [rows][D/128], stored back K-block major);
4. the grouped GEMMs over the received rows, which form one 128-aligned
   segment per (source rank, local expert): segment s*E_loc + e uses local
   expert e's weights (moe_grouped_gemm_fp8_seg);
5. return: one all-to-all of the bf16 expert outputs Y back to the ranks that
   own the tokens, into their own permuted layout;
6. the weighted combine (moe_combine) on every rank.

Padding rows travel with their segments (zero codes and scales, so their
outputs are zero).  The exchange uses torch.distributed's all_to_all_single
(NCCL over NVLink between GPUs; gloo for the host-side tests).  This module
moves bytes and computes sizes; every arithmetic step runs in the library's
kernels (or, in the CPU tests, in the oracle).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch
import torch.distributed as dist


@dataclasses.dataclass
class Plan:
    world: int
    rank: int
    E: int                    # experts over all ranks
    E_loc: int                # experts per rank
    send_start: list          # first permuted row sent to each rank
    send_rows: list           # rows (padded segments) sent to each rank
    recv_rows: list           # rows received from each rank
    seg: np.ndarray           # [world, E_loc] padded segment sizes received
    seg_offsets: np.ndarray   # [world*E_loc + 1] offsets of the received segments
    rows_recv: int            # rows received in all
    rows_cap: int             # rows_recv rounded up to 128 (at least 128)

    @property
    def rows_sent(self) -> int:
        return int(sum(self.send_rows))


def _words(t):
    """A row-major tensor viewed as 32-bit words along its last axis (the
    rows cross the link byte for byte; gloo has no 8- or 16-bit types)."""
    return t.view(torch.int32)


def make_plan(offsets, world: int, rank: int, group=None, device="cpu") -> Plan:
    """The exchange plan of one layer from this rank's permute offsets
    (host int array [E+1]); one all-to-all of the padded segment sizes."""
    off = np.asarray(offsets, np.int64)
    E = len(off) - 1
    if E % world:
        raise ValueError(f"{E} experts do not split over {world} ranks")
    E_loc = E // world
    sizes = np.diff(off).reshape(world, E_loc)           # [dest rank, local expert]
    send = torch.from_numpy(np.ascontiguousarray(sizes.reshape(-1))).to(device)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)       # equal splits: E_loc per rank
    seg = recv.cpu().numpy().reshape(world, E_loc)
    seg_offsets = np.concatenate([[0], np.cumsum(seg.reshape(-1))]).astype(np.int64)
    rows_recv = int(seg_offsets[-1])
    return Plan(world=world, rank=rank, E=E, E_loc=E_loc,
                send_start=[int(off[d * E_loc]) for d in range(world)],
                send_rows=[int(off[(d + 1) * E_loc] - off[d * E_loc]) for d in range(world)],
                recv_rows=[int(seg[s].sum()) for s in range(world)],
                seg=seg, seg_offsets=seg_offsets, rows_recv=rows_recv,
                rows_cap=max(128, (rows_recv + 127) // 128 * 128))


def dispatch(plan: Plan, xq, xs, group=None):
    """Send the permuted FP8 rows to their experts' ranks.

    xq: codes [R_cap, D] uint8; xs: scales [D/128, R_cap] fp32 (K-block major),
    this rank's permuted layout.  Returns (xq_r [rows_cap, D], xs_r
    [D/128, rows_cap]) in the received layout (rows past rows_recv zero)."""
    R = plan.rows_sent
    D = xq.shape[1]
    xq_r = torch.zeros(plan.rows_cap, D, dtype=xq.dtype, device=xq.device)
    dist.all_to_all_single(_words(xq_r[:plan.rows_recv]), _words(xq[:R].contiguous()),
                           output_split_sizes=plan.recv_rows, input_split_sizes=plan.send_rows, group=group)
    s_send = xs[:, :R].t().contiguous()                   # [R, D/128], row-major for the exchange
    s_recv = torch.empty(plan.rows_recv, xs.shape[0], dtype=xs.dtype, device=xs.device)
    dist.all_to_all_single(s_recv, s_send, output_split_sizes=plan.recv_rows, input_split_sizes=plan.send_rows,
                           group=group)
    xs_r = torch.zeros(xs.shape[0], plan.rows_cap, dtype=xs.dtype, device=xs.device)
    xs_r[:, :plan.rows_recv] = s_recv.t()
    return xq_r, xs_r


def combine_back(plan: Plan, Y_r, Y, group=None):
    """Return the expert outputs: Y_r [rows_cap, D] (received layout) ->
    rows [0, rows_sent) of Y (this rank's permuted layout)."""
    dist.all_to_all_single(_words(Y[:plan.rows_sent]), _words(Y_r[:plan.rows_recv].contiguous()),
                           output_split_sizes=plan.send_rows, input_split_sizes=plan.recv_rows, group=group)
    return Y


def local_segment_offsets(plan: Plan, device) -> torch.Tensor:
    """The received segments' offsets as the int32 device array the segment
    GEMM reads."""
    return torch.from_numpy(plan.seg_offsets.astype(np.int32)).to(device)


def forward(B, x, W_loc, group=None, stream=None):
    """One EP layer forward on this rank, after routing into B (layer.Buffers
    over all E experts).  W_loc: layer.Weights of this rank's E_loc experts.
    Returns B.y.  The permute offsets are read back to the host to size the
    exchange (one synchronisation per layer)."""
    from . import abi
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    d = B.d
    abi.permute(B.idx, d, B.counts, B.offsets, B.pos, B.src, x, B.xq, B.xs, None, None, B.ws, stream=stream)
    plan = make_plan(B.offsets.cpu().numpy(), world, rank, group, device=B.offsets.device)
    xq_r, xs_r = dispatch(plan, B.xq, B.xs, group)
    E_loc = plan.E_loc
    dl = abi.dims(d.T, d.D, d.I, E_loc, d.k)
    segs = local_segment_offsets(plan, x.device)
    n_seg = world * E_loc
    hq = torch.empty(plan.rows_cap, d.I, dtype=torch.uint8, device=x.device)
    hs = torch.empty(d.I // 128, plan.rows_cap, dtype=torch.float32, device=x.device)
    Y_r = torch.empty(plan.rows_cap, d.D, dtype=torch.bfloat16, device=x.device)
    abi.grouped_gemm_fp8_seg(abi.GEMM_GATEUP_SILU, dl, plan.rows_cap, segs, n_seg, xq_r, xs_r, W_loc.wgu_q,
                             W_loc.wgu_s, out_q=hq, out_s=hs, stream=stream)
    abi.grouped_gemm_fp8_seg(abi.GEMM_DOWN, dl, plan.rows_cap, segs, n_seg, hq, hs, W_loc.wd_q, W_loc.wd_s,
                             out_bf16=Y_r, stream=stream)
    combine_back(plan, Y_r, B.Y, group)
    abi.combine(B.Y, B.w, B.pos, d, B.y, stream=stream)
    return B.y
