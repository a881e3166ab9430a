"""bench.py's multi-rank host logic on CPU: two gloo ranks (one per GPU in a real run).

Every rank runs an independent replica of the layer; the only collectives are the barrier and
the max over ranks of the timed milliseconds, from which rank 0 reports the whole job's rate."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # rank r timed (10 + r) ms in all for its steps, and (3 - r, 7 + 2r) for two other figures
        got = bench.max_over_ranks([10.0 + rank, 3.0 - rank, 7.0 + 2 * rank], torch.device("cpu"), world)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_on_two_gloo_ranks():
    import torch.multiprocessing as mp

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    assert codes == [0, 0], codes
    results = dict(q.get(timeout=10) for _ in range(world))
    for r in range(world):
        assert results[r] == [11.0, 3.0, 9.0]  # every rank sees the slowest rank's figures

    sys.path.insert(0, ROOT)
    import bench

    # two replicas of 8192 tokens, 20 steps each, the slowest rank took 200 ms: 1,638,400 tokens/s
    assert bench.whole_job_rate(2, 8192, 20, 200.0) == pytest.approx(2 * 8192 * 20 / 0.2)
    assert bench.max_over_ranks([1.5, 2.5], None, 1) == [1.5, 2.5]  # one rank: no collective


def test_reference_arm_does_nothing_on_ranks_other_than_zero(capsys):
    sys.path.insert(0, ROOT)
    import bench
    import moe_inputs as mi

    class Args:
        steps, warmup, weights = 1, 3, "bf16"

    bench.run_reference(Args(), mi.WORKLOADS["tiny"], rank=1, world=2)
    assert capsys.readouterr().out == ""
