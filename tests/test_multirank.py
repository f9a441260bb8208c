"""The multi-rank (N > 1) host path of the benchmark on CPU: two gloo ranks, each with
its own batch (weak scaling, no data-path collective), timing reduced as the max over
ranks and work as the sum.  The per-rank work here is the oracle's plan of that rank's
batch, so the ranks really do process different problems."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        import workload
        seed = bench.rank_seed(0, rank)
        r = workload.make_routing(workload.CONFIGS[0], seed=seed)
        p = oracle.plan(r.ids, r.cfg.E, r.expert_rank, r.cfg.R)
        fake_seconds = 0.5 + rank                     # rank 1 is the slow one
        agg = bench.aggregate(r.cfg.N, fake_seconds, world, "cpu")
        d_all = torch.zeros(world, dtype=torch.int64)
        d_all[rank] = p["D"]
        dist.all_reduce(d_all)
        out[rank] = (agg["tokens"], agg["seconds"], agg["tokens_per_s"], int(d_all[0]), int(d_all[1]))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_aggregate():
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    a, b = out[0], out[1]
    assert a == b                                     # every rank agrees on the aggregate
    tokens, seconds, tps, d0, d1 = a
    assert tokens == 2 * 4096 and seconds == 1.5 and abs(tps - 8192 / 1.5) < 1e-9
    assert d0 != d1                                   # the ranks planned different batches
