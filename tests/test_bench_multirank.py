"""Multi-process (world size 2, gloo on CPU) check of the benchmark's
multi-rank plumbing: each rank draws its own batch (seed offset by rank) and
the reported time is the max over ranks."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    w = bench.rank_workload("decode_128k", rank)
    t = bench.max_over_ranks([0.001 * (rank + 1), 0.5 - 0.1 * rank], world)
    out[rank] = torch.tensor([w.seed, t[0], t[1]], dtype=torch.float64)
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_max_and_distinct_batches():
    world = 2
    out = torch.zeros((world, 3), dtype=torch.float64).share_memory_()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    seeds = out[:, 0].tolist()
    assert seeds[0] != seeds[1]
    for r in range(world):
        assert abs(out[r, 1].item() - 0.002) < 1e-12     # max of 0.001, 0.002
        assert abs(out[r, 2].item() - 0.5) < 1e-12       # max of 0.5, 0.4
