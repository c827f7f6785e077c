"""World-size-2 `gloo` test, on CPU, of the benchmark's multi-rank timing:
every rank's timed region is reduced with MAX and the whole-job figure is that
time over the layer-steps of all ranks.  The multi-GPU path is replicas (one
independent cache per GPU), so this reduction and the barriers are its only
cross-rank traffic."""
import os
import socket
from datetime import timedelta

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=30))
    import bench
    dist.barrier()
    t = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
    q.put((rank, t, bench.us_per_layer_step(t, 100, world)))
    dist.barrier()
    dist.destroy_process_group()


def test_timing_is_max_over_ranks_and_counts_all_ranks_steps():
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
    assert [r for r, _, _ in res] == [0, 1]
    for _, t, us in res:
        assert t == 15.0                      # the slower rank's 15 ms on both ranks
        assert us == 15.0 * 1e3 / (100 * 2)   # over both ranks' 200 layer-steps


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1, torch.device("cpu")) == 12.5
    assert bench.us_per_layer_step(12.5, 50, 1) == 250.0
