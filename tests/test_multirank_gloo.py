"""The benchmark's multi-GPU path on CPU: two `gloo` ranks run the same
aggregation the benchmark uses under torchrun (value = bytes of all ranks /
the slowest rank's time, "weak" scaling, no data-path collective)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    dev = torch.device("cpu")
    local_ms = 10.0 * (rank + 1)          # rank 1 is the slowest
    local_bytes = 1e9 * (rank + 1)
    bench.barrier(world)
    mx = bench.all_reduce_max(local_ms, world, dev)
    tot = bench.all_reduce_sum(local_bytes, world, dev)
    out.put((rank, mx, tot, tot / (mx * 1e-3) / 1e9))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_aggregation():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, tot, gbs in res:
        assert mx == 20.0                  # max over ranks
        assert tot == 3e9                  # sum over ranks
        assert gbs == pytest.approx(150.0) # 3 GB in 20 ms


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    import torch
    assert bench.all_reduce_max(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.all_reduce_sum(2.0, 1, torch.device("cpu")) == 2.0
