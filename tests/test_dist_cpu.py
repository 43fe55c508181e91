"""The multi-process (N > 1) plumbing of bench.py on CPU: two gloo ranks.

bench.py --gpus N runs one independent replica of the decode workload per
rank (the path shards with no data exchange). The only cross-rank steps are the
barrier around the timed region and the reduction of the step time to the
slowest rank's, from which the whole-job throughput is computed. These run
here on two CPU processes with the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        elapsed = [120.0, 150.0][rank]              # the rank's timed region, ms
        slowest = bench.max_over_ranks(elapsed, world)
        value = bench.aggregate_gbs(419_430_400, 50, world, slowest)
        q.put((rank, slowest, value))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_rank_and_count_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=90) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value in out:
        assert slowest == 150.0                      # both ranks see the slowest rank's time
        # every rank's bytes over the slowest time: 2 x 50 x 419,430,400 B / 0.15 s
        assert abs(value - 2 * 50 * 419_430_400 / 0.150 / 1e9) < 1e-9
