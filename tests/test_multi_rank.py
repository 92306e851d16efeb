"""Multi-rank host logic of the benchmark on CPU with the gloo backend
(world_size 2): replicas draw different batches, the step time is the max
over ranks, and the whole-job rate counts every rank's units."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    from datetime import timedelta

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    from moe_expert_layer_replay_b200.inputs import make_inputs
    t = bench.reduce_max(10.0 * (rank + 1))
    seed = bench.replica_seed(0, rank)
    x = make_inputs("tiny", seed=seed, weights=False)["x"]
    out.put((rank, t, seed, int(x[0, 0]), bench.aggregate_rate(world, 100.0, t)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, s0, x0, v0), (r1, t1, s1, x1, v1) = res
    assert t0 == t1 == 20.0                    # max over ranks
    assert s0 != s1 and x0 != x1               # replicas draw different batches
    assert v0 == v1 == 2 * 100.0 / 20.0        # all ranks' units over the slowest time


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
