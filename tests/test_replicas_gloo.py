"""The multi-GPU path of the benchmark is N independent replicas (the decode
of one token does not shard): the only cross-rank step is the maximum of the
per-rank times.  Checked here with two gloo ranks on the CPU."""
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    local_ms = [12.5, 20.0][rank]
    ms = bench.max_over_ranks(local_ms, world, "cpu")
    value = bench.job_value(64, world, ms)
    q.put((rank, ms, value))
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[1] for g in got] == [20.0, 20.0]
    # 2 ranks x 64 tokens in the slowest rank's 20 ms
    assert all(abs(g[2] - 20.0 * 1000 / 128) < 1e-9 for g in got)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.job_value(10, 1, 5.0) == 500.0
