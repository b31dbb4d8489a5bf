"""The replica path of a multi-GPU bench run, on CPU with gloo (world size 2): every rank decodes
its own sequence; the only collective is the timing reduction (max time, summed tokens), and the
aggregate throughput is the summed tokens over the slowest rank's time."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = [12.5, 14.0][rank]
    tokens = [30.0, 34.0][rank]
    max_ms, = bench.reduce([ms], "max", world)
    tot, = bench.reduce([tokens], "sum", world)
    out[rank] = (max_ms, tot, tot / (max_ms / 1e3))
    dist.barrier()
    dist.destroy_process_group()


def test_replica_reduction_two_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        max_ms, tot, value = res[r]
        assert max_ms == 14.0 and tot == 64.0
        assert abs(value - 64.0 / 0.014) < 1e-6


def test_dist_setup_reads_torchrun_env(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "3")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.dist_setup() == (4, 3, 1)
