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


def _reference_rank(rank, world, port, q):
    """bench.py --impl reference under a 2-rank launch: rank 0 runs the oracle on a
    bounded sample and prints the line, the other ranks exit without work."""
    import io
    import contextlib
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    args = type("A", (), {"steps": 2, "warmup": 1})()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.run_reference(args, world, rank)
    q.put((rank, rc, buf.getvalue()))


@pytest.mark.timeout(300)
def test_reference_arm_prints_on_rank0_only():
    import json
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_reference_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict((r, (rc, txt)) for r, rc, txt in (q.get(timeout=240) for _ in range(2)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[1] == (0, "")
    rc, txt = out[0]
    assert rc == 0
    line = json.loads(txt.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 2
    assert line["config"]["workload"] == "decode_gqa_b32_hq32_hkv8_l8192"
    assert line["config"]["parallelism"].startswith("dp2")
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
