"""GPU parity of the ablation tools (the selection rules MC-Sparse replaces)
against the fp64 oracle's restatements, on seeded DiT-shaped inputs.

* block selection: the GPU's blocks (on its own group scores) agree with the
  oracle's blocks (on its exact group scores) except blocks whose score lies
  within 1e-4 relative of the kept threshold; then the residual and the
  reused step over the GPU's block keys match the oracle's on those keys;
* pooled scores element by element, and their top-k within the same band;
* the ablation driver's variants run end to end with finite fidelities and
  token selection beating the others at equal key budget on retained mass.
"""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from oracle import mcs_oracle as orc
from sparse_attention_diffusion_mcs_b200 import ablate
from tests.gpu_util import (COLSUM_ABS, COLSUM_REL, KV_THRESHOLD_REL, assert_out_close, assert_residual_close,
                            dev_bf16, host, kv_sets_agree)

pytestmark = pytest.mark.gpu


def block_sets_agree(got_keys, c, kb, block):
    """The GPU's kept blocks vs the oracle's block scores: differences only
    among blocks within KV_THRESHOLD_REL of the kb-th block score."""
    got_keys = np.asarray(got_keys)
    assert len(got_keys) == kb * block and np.all(np.diff(got_keys) > 0)
    assert np.all(got_keys.reshape(kb, block) % block == np.arange(block))      # whole aligned blocks
    nb = len(c) // block
    bs = c[:nb * block].reshape(nb, block).sum(axis=1)
    order = np.lexsort((np.arange(nb), -bs))
    thr = bs[order[kb - 1]]
    got = set((got_keys[::block] // block).tolist())
    for b in got.symmetric_difference(set(order[:kb].tolist())):
        assert abs(bs[b] - thr) <= KV_THRESHOLD_REL * abs(thr), (b, bs[b], thr)


@pytest.mark.parametrize("block", [64, 128])
def test_block_selection_and_its_residual_match_the_oracle(block):
    w = synth.workload(1).with_(grid=(4, 8, 32), G=128, k=300)            # N = 1024
    Q, K, V = synth.layer_tensors(w)
    q, kd, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    ws = mcs.alloc_workspace(w.B, w.H, w.N, w.d, w.G, w.k, q.device)
    meta = mcs.plan(q, kd, v, w.G, w.k, workspace=ws)
    colsum = mcs.workspace_views(ws, w.B, w.H, w.N, w.d, w.G, w.k)["colsum"]
    kb = w.k // block
    kv = mcs.select_blocks(colsum, kb, block)
    res = mcs.plan_residual(q, kd, v, meta.perm, kv, w.G, workspace=ws, stats_done=True)
    m2 = mcs.Meta.from_tensors(meta.perm, kv, res, w.G)
    Q2, K2, V2 = synth.layer_tensors(w, step=2)
    out = host(mcs.sparse_step(dev_bf16(Q2), dev_bf16(K2), dev_bf16(V2), m2))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    kv, res, perm = kv.cpu().numpy(), res.cpu().numpy().astype(np.float64), meta.perm.cpu().numpy()
    for h in range(w.H):
        assert np.array_equal(perm[0, h], orc.group_queries(Q[0, h]))
        c = orc.group_prob_sums(Q[0, h], K[0, h], w.scale, perm[0, h], w.G)
        for g in range(w.n_groups):
            block_sets_agree(kv[0, h, g], c[g], kb, block)
            ref_blocks = orc.select_blocks(c[g], kb, block)
            assert len(ref_blocks) == kb * block
            rows = orc.group_rows(perm[0, h], w.G, g)
            R, _, _ = orc.residual_group(Q[0, h][rows], K[0, h], V[0, h], w.scale, kv[0, h, g])
            assert_residual_close(res[0, h][rows], R, f"block{block} residual h{h} g{g}")
            o = orc.sparse_group(Q2[0, h][rows], K2[0, h], V2[0, h], w.scale, kv[0, h, g]) + R
            assert_out_close(out[0, h][rows], o, f"block{block} step h{h} g{g}")


def test_pooled_scores_and_selection_match_the_oracle():
    w = synth.workload(1).with_(grid=(4, 8, 32), G=64, k=200)
    Q, K, _ = synth.layer_tensors(w)
    perm = np.stack([orc.group_queries(Q[0, h]) for h in range(w.H)]).astype(np.int32)[None]
    p = mcs.pooled_scores(dev_bf16(Q), dev_bf16(K), torch.from_numpy(perm).cuda(), w.G)
    kv = mcs.select_topk(p, w.k)
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    p, kv = p.cpu().numpy().astype(np.float64), kv.cpu().numpy()
    for h in range(w.H):
        ref = orc.pooled_scores(Q[0, h], K[0, h], w.scale, perm[0, h], w.G)
        assert np.all(np.abs(p[0, h] - ref) <= COLSUM_REL * ref + COLSUM_ABS)
        for g in range(w.n_groups):
            kv_sets_agree(kv[0, h, g], ref[g], w.k)


def test_ablation_driver_runs_every_variant():
    w = synth.workload(1).with_(grid=(4, 8, 32), G=128, k=256)
    Q, K, V = (dev_bf16(x) for x in synth.layer_tensors(w))
    Q2, K2, V2 = (dev_bf16(x) for x in synth.layer_tensors(w, step=2))
    abl = ablate.Ablation(Q, K, V, w.G, w.k, blocks=(64, 128))
    res = abl.step(Q2, K2, V2, mcs.dense(Q2, K2, V2))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    assert set(res) == {"token", "block64", "token@k64", "block128", "token@k128", "pooled"}
    for name, r in res.items():
        assert np.isfinite(r["rel_l2"]) and np.isfinite(r["rel_l2_without_residual"]), name
        assert 0.0 < abl.alpha[name] <= 1.0 + 1e-6
    # exact token selection keeps the most mass for its budget
    assert abl.alpha["token@k64"] >= abl.alpha["block64"] - 1e-6
    assert abl.alpha["token"] >= abl.alpha["pooled"] - 1e-6
