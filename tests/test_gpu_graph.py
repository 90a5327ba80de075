"""The reused step (a6) inside a CUDA graph: a denoising loop reuses the same
metadata and buffers every step, so the step can be captured once and
replayed with new Q, K, V written into the captured input buffers.  The
replay must give exactly what an eager call gives on the same inputs, step
after step."""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def test_sparse_step_graph_replay_matches_eager():
    w = synth.workload("tiny").with_(grid=(1, 1, 1000), d=128, G=128, k=300)
    Q, K, V = synth.random_qkv(1, 2, 1000, 128, seed=8)
    perm = np.stack([synth.random_metadata_head(w, h)[0] for h in range(2)])[None]
    kv = np.stack([synth.random_metadata_head(w, h)[1] for h in range(2)])[None]
    res = np.stack([synth.random_metadata_head(w, h)[2] for h in range(2)])[None]
    meta = mcs.Meta.from_tensors(torch.from_numpy(perm).cuda(), torch.from_numpy(kv).cuda(),
                                 torch.from_numpy(res).cuda(), w.G)
    q, k, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    out = torch.empty_like(q)
    mcs.sparse_step(q, k, v, meta, out=out)          # eager warm-up (also sets up the library)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        mcs.sparse_step(q, k, v, meta, out=out)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        mcs.sparse_step(q, k, v, meta, out=out)
    for step in range(3):
        Qs, Ks, Vs = synth.random_qkv(1, 2, 1000, 128, seed=100 + step)
        q.copy_(dev_bf16(Qs))
        k.copy_(dev_bf16(Ks))
        v.copy_(dev_bf16(Vs))
        graph.replay()
        eager = mcs.sparse_step(dev_bf16(Qs), dev_bf16(Ks), dev_bf16(Vs), meta)
        torch.cuda.synchronize()
        assert mcs.last_device_status() == 0
        assert torch.equal(out, eager), f"replay {step} differs from the eager step"
