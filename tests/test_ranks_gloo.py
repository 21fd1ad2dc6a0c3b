"""Two ranks on the host (gloo): the benchmark's multi-rank logic.  Each rank
codes its own shard (weak scaling, no data-path collective); the only
collective is the max over ranks of the device-timed step, and the job value
counts every rank's tokens over that slowest time."""
import datetime
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q) -> None:
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench

        mine = 10.0 + 5.0 * rank  # this rank's step time (ms)
        slowest = bench.max_over_ranks(mine, world, "cpu")
        q.put((rank, slowest, bench.shard_seed(rank), bench.job_value(slowest, world, 30),
               bench.max_over_ranks(mine, 1, "cpu")))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_time_the_slowest_and_code_distinct_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = 15.0
    for rank, t, seed, value, alone in got:
        assert t == slowest  # both ranks see the slower rank's time
        assert alone == 10.0 + 5.0 * rank  # one rank: no collective
        assert value == 2 * 32760 * 30 * 2 / (slowest * 1e-3)  # both shards' tokens
    assert got[0][2] != got[1][2]  # distinct shards
