"""Multi-rank host logic on CPU with gloo ranks (no GPU): one layer sharded
by head blocks (shard.py) -- every rank runs MC-Sparse on its own heads only,
with no exchange on the data path -- reassembles, in head order, to exactly
what one process computes for the whole layer; the benchmark's inputs are
seeded per global head, and its timings reduce to the slowest rank's.

On CPU the per-head computation is the fp64 oracle (the library needs a
GPU); what is under test is the partition: offsets, counts, uneven splits,
and the reassembly."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from oracle import mcs_oracle as orc
from sparse_attention_diffusion_mcs_b200 import shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(w):
    """(step-1 tensors, step-2 tensors) of the whole layer, uint16 [B,H,N,d]."""
    s1 = synth.layer_tensors(w, step=1)
    s2 = synth.layer_tensors(w, step=2)
    return s1, s2


def _mcs_heads(w, s1, s2):
    """Per head: plan on step 1, reused step on step 2 (fp64 oracle)."""
    out = []
    for b in range(s1[0].shape[0]):
        for h in range(s1[0].shape[1]):
            m = orc.plan_head(s1[0][b, h], s1[1][b, h], s1[2][b, h], w.G, w.k, w.scale)
            out.append(orc.reused_step_head(s2[0][b, h], s2[1][b, h], s2[2][b, h], w.scale,
                                            m["perm"], m["kv_idx"], m["residual"], w.G))
    return np.stack(out)


def _worker(rank, world, port, H, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        w = synth.workload(1).with_(H=H)
        s1, s2 = _layer(w)
        # this rank's heads: views of the layer at its head offset
        mine1 = [shard.shard(torch.from_numpy(x.astype(np.int32)), world, rank).numpy().astype(np.uint16)
                 for x in s1]
        mine2 = [shard.shard(torch.from_numpy(x.astype(np.int32)), world, rank).numpy().astype(np.uint16)
                 for x in s2]
        local = torch.from_numpy(_mcs_heads(w, mine1, mine2))[None]
        full = shard.gather_heads(local, w.BH, world)
        out[rank] = full.numpy()
        # the benchmark regenerates exactly its block from the global head index
        wb = synth.workload(1)
        heads = bench.rank_heads(wb, rank)
        start, count = shard.head_range(wb.BH * world, world, rank)
        assert heads == list(range(start, start + count))
        q_rank = synth.head_tensors(wb, heads[0])[0]
        assert np.array_equal(q_rank, synth.head_tensors(wb, start)[0])
        # timings reduce to the slowest rank's
        t = torch.tensor([1.0 + rank, 10.0 - 3.0 * rank], dtype=torch.float64)
        assert bench.max_over_ranks(t).tolist() == [float(world), 10.0]
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("H", [2, 3])   # even and uneven splits over two ranks
def test_head_sharded_layer_equals_single_process(H):
    world = 2
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, _free_port(), H, out), nprocs=world, join=True,
                       start_method="spawn")
    w = synth.workload(1).with_(H=H)
    s1, s2 = _layer(w)
    ref = _mcs_heads(w, s1, s2)
    for r in range(world):
        assert out[r].shape == ref.shape
        assert np.array_equal(out[r], ref), f"rank {r}: reassembled output differs"


def test_single_process_reduction_is_identity():
    import bench
    t = torch.tensor([3.0, 4.0], dtype=torch.float64)
    assert bench.max_over_ranks(t).tolist() == [3.0, 4.0]
