"""Expert parallelism on gloo ranks (CPU, no GPU): the exchange plan, the
all-to-all dispatch of FP8 rows and scales, the segment layout the receiving
rank computes on, and the return of the expert outputs ("RL at 1T scale:
prime-rl performance deep dive", §Parallelism strategy / EP).

Every rank routes and permutes its own tokens over all experts, sends each
row to the rank that owns its expert, computes its local experts on what it
received (the oracle's FFN steps stand in for the kernels, one segment per
(source rank, local expert)), and gets its rows back for the combine.  The
result must equal, bit for bit, the single-rank forward of the same tokens
with all experts: EP moves rows, it changes no arithmetic."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from moe_expert_layer_replay_b200.inputs import to_bf16_bits

D, I, K = 256, 128, 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _weights(E):
    rng = np.random.default_rng(1234)   # the same on every rank
    b = lambda shape: to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(0.05))
    return b((E, I, D)), b((E, I, D)), b((E, D, I))


def _tokens(rank, E):
    rng = np.random.default_rng(77 + rank)
    T = 40 + 56 * rank                  # ranks hold different numbers of tokens
    p = np.arange(1, E + 1, dtype=np.float64) ** -1.3
    p[-1] = 0.0                         # one expert gets no token anywhere
    with np.errstate(divide="ignore"):
        z = (np.log(p / p.sum())[None, :] - np.log(-np.log(rng.random((T, E))))).astype(np.float32)
    x = to_bf16_bits(rng.standard_normal((T, D)).astype(np.float32))
    return z, x


def _rank_main(rank, world, port, E, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from oracle import layer as OL
        from moe_expert_layer_replay_b200 import ep
        z, x = _tokens(rank, E)
        idx, w = oracle.route_topk(z, K)
        counts, offsets, pos, src = oracle.permute(idx, E, 128)
        R_cap = len(src)
        xq, xs_rows = oracle.quant_block(OL.dispatch_rows(x, src, np.arange(R_cap), K), 1, 128)
        plan = ep.make_plan(offsets, world, rank)
        assert plan.rows_sent == int(offsets[E])
        xq_r, xs_r = ep.dispatch(plan, torch.from_numpy(xq), torch.from_numpy(np.ascontiguousarray(xs_rows.T)))
        # this rank's experts on the received segments (segment v -> local expert v % E_loc)
        Wg, Wu, Wd = _weights(E)
        lo, hi = rank * plan.E_loc, (rank + 1) * plan.E_loc
        Wq = [OL.quant_weights(W[lo:hi]) for W in (Wg, Wu, Wd)]
        n = plan.rows_recv
        seg_expert = OL.expert_of_rows(plan.seg_offsets, np.arange(n)) % plan.E_loc
        g, u = OL.gateup_rows(xq_r.numpy()[:n], np.ascontiguousarray(xs_r.numpy()[:, :n].T), seg_expert, Wq[0], Wq[1])
        h = OL.swiglu_h(g, u)
        hq, hs = oracle.quant_block(h, 1, 128)
        Y_r = torch.zeros(plan.rows_cap, D, dtype=torch.int16)
        Y_r[:n] = torch.from_numpy(OL.down_rows(hq, hs, seg_expert, Wq[2]).view(np.int16))
        Y = torch.zeros(R_cap, D, dtype=torch.int16)
        ep.combine_back(plan, Y_r, Y)
        Yb = Y.numpy().view(np.uint16)
        ok = pos >= 0
        y = OL.combine(oracle.bf16_to_f64(Yb)[np.where(ok, pos, 0)], w, ok)
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), y=y, Y=Yb[:int(offsets[E])], idx=idx, w=w,
                 seg=plan.seg, recv=np.array(plan.recv_rows), send=np.array(plan.send_rows))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E", [(2, 8), (4, 8), (4, 16)])
def test_ep_forward_matches_single_rank(orc, world, E):
    from oracle import layer as OL
    with tempfile.TemporaryDirectory() as outdir:
        mp.spawn(_rank_main, args=(world, _free_port(), E, outdir), nprocs=world, join=True)
        res = [dict(np.load(os.path.join(outdir, f"rank{r}.npz"))) for r in range(world)]
    Wg, Wu, Wd = _weights(E)
    Wq = (OL.quant_weights(Wg), OL.quant_weights(Wu), OL.quant_weights(Wd))
    E_loc = E // world
    for r in range(world):
        z, x = _tokens(r, E)
        fw = OL.forward(x, res[r]["idx"], res[r]["w"], None, None, None, quantised_w=Wq)
        assert np.array_equal(res[r]["Y"], fw["Y"]), f"rank {r}: expert outputs"
        assert np.array_equal(res[r]["y"], fw["y"]), f"rank {r}: combined outputs"
        # what rank r received from s is what s sent to r, segment by segment
        for s in range(world):
            assert res[r]["recv"][s] == res[s]["send"][r]
            off = np.diff(OL.forward(_tokens(s, E)[1], res[s]["idx"], res[s]["w"], None, None, None,
                                     quantised_w=Wq)["offsets"])
            assert np.array_equal(res[r]["seg"][s], off[r * E_loc:(r + 1) * E_loc])
