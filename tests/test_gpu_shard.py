"""Head-block sharding on the GPU: the library run on each rank's block of
heads -- a view of the layer at its head offset, as a rank holding only
those heads would pass it -- gives, block by block, bit for bit what one call
over the whole layer gives (every kernel works per head; nothing depends on
which other heads share a launch).  The ranks run one after another on one
GPU here; they never wait on each other."""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from sparse_attention_diffusion_mcs_b200 import shard
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_calls_equal_the_whole_layer(world):
    w = synth.workload(1).with_(B=2, H=3, grid=(1, 1, 700), d=64, G=128, k=150)   # 6 heads, uneven for 4
    Q1, K1, V1 = (dev_bf16(x) for x in synth.random_qkv(w.B, w.H, w.N, w.d, seed=21, q_std=2.0))
    Q2, K2, V2 = (dev_bf16(x) for x in synth.random_qkv(w.B, w.H, w.N, w.d, seed=22, q_std=2.0))
    meta, od = mcs.plan(Q1, K1, V1, w.G, w.k, return_dense=True)
    o_step = mcs.sparse_step(Q2, K2, V2, meta)
    o_dense = mcs.dense(Q2, K2, V2)
    torch.cuda.synchronize()
    flat = lambda t: t.reshape(w.BH, *t.shape[2:])
    for r in range(world):
        start, count = shard.head_range(w.BH, world, r)
        if count == 0:
            continue
        q1, k1, v1, q2, k2, v2 = (shard.shard(t, world, r) for t in (Q1, K1, V1, Q2, K2, V2))
        m_r, od_r = mcs.plan(q1, k1, v1, w.G, w.k, return_dense=True)
        step_r = mcs.sparse_step(q2, k2, v2, m_r)
        dense_r = mcs.dense(q2, k2, v2)
        torch.cuda.synchronize()
        assert mcs.last_device_status() == 0
        sl = slice(start, start + count)
        assert torch.equal(m_r.perm[0], flat(meta.perm)[sl])
        assert torch.equal(m_r.kv_idx[0], flat(meta.kv_idx)[sl])
        assert torch.equal(m_r.residual[0], flat(meta.residual)[sl])
        assert torch.equal(od_r[0], flat(od)[sl])
        assert torch.equal(step_r[0], flat(o_step)[sl])
        assert torch.equal(dense_r[0], flat(o_dense)[sl])
