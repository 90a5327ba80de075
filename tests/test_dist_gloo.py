"""Multi-rank host logic of the benchmark, on CPU with two gloo ranks: every
rank gets its own seeded layer (weak scaling, no data exchange) and timings
are reduced to the slowest rank's."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        t = torch.tensor([1.0 + rank, 10.0 - 3.0 * rank, 0.5], dtype=torch.float64)
        red = bench.max_over_ranks(t)
        w = bench.rank_workload(synth.workload(1), rank)
        q, _, _ = synth.head_tensors(w, 0)
        out[rank] = (red.tolist(), int(q[:8, :8].astype(np.int64).sum()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_reduction_and_distinct_layers():
    world = 2
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == [2.0, 10.0, 0.5]
    assert r0[1] != r1[1]                      # each rank runs its own layer


def test_single_process_reduction_is_identity():
    import bench
    t = torch.tensor([3.0, 4.0], dtype=torch.float64)
    assert bench.max_over_ranks(t).tolist() == [3.0, 4.0]
