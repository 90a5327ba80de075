"""GPU parity at the full workload sizes, through the same C entry points the
benchmark times, checked on sampled heads and query groups that the oracle
computes one by one (its full plan at these sizes would take hours).

Per workload: the GPU plans on the step-1 inputs, runs the reused step and
dense attention on the drifted step-2 inputs; then for two sampled heads:
  * the query order equals the oracle's (both decide it in fp64);
  * a2: for every row of the sampled groups, the row's log normaliser
    m + log2 l from the plan workspace matches the oracle's, and m lies in
    its documented band below the row maximum;
  * a3: the group scores colsum[g, :] of the sampled groups (first, middle,
    last-partial) match the oracle's sums of exact probabilities element by
    element;
  * a4: the KV index sets agree with the oracle's top-k except within 1e-4
    of the k-th score;
  * a5, a6: for EVERY sampled group the oracle recomputes the residual and
    the reused step on the GPU's own kv_idx (the protocol's step 2: once the
    sets agree within the band, the downstream comparison uses the GPU's
    selection), so no group is skipped;
  * sampled rows of both dense outputs agree with the oracle.
The number of groups and rows compared is asserted, never zero.
"""
import numpy as np
import pytest
import torch

import bench
import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from oracle import mcs_oracle as orc
from tests.gpu_util import (COLSUM_ABS, COLSUM_REL, LSE_ABS, assert_out_close, assert_residual_close,
                            kv_sets_agree)

pytestmark = pytest.mark.gpu

CASES = [
    ("video_short", 2, None, None),
    ("video_long", 3, None, None),
    ("asset3d", 4, None, None),
    ("sweep G64 1%", 5, 1310, 64),
    ("sweep G128 25%", 5, 32768, 128),
]


def _up(x):
    return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("name,cfg,k,G", CASES, ids=[c[0] for c in CASES])
def test_full_size_sampled_parity(name, cfg, k, G):
    w = synth.workload(cfg, k=k, G=G)
    s1, s2 = bench.make_inputs(w, 0)
    Q1, K1, V1 = (_up(x) for x in s1)
    Q2, K2, V2 = (_up(x) for x in s2)
    ws = mcs.alloc_workspace(w.B, w.H, w.N, w.d, w.G, w.k, Q1.device)
    meta, od1 = mcs.plan(Q1, K1, V1, w.G, w.k, workspace=ws, return_dense=True)
    o_step = mcs.sparse_step(Q2, K2, V2, meta)
    o_dense = mcs.dense(Q2, K2, V2)
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ok, code = mcs.validate_meta(meta)
    assert ok, code
    views = mcs.workspace_views(ws, w.B, w.H, w.N, w.d, w.G, w.k)
    kk = min(w.k, w.N)
    perm_all = meta.perm.view(w.BH, w.N)
    kv_all = meta.kv_idx.view(w.BH, w.n_groups, kk)
    res_all = meta.residual.view(w.BH, w.N, w.d)
    m_all = views["row_m"].reshape(w.BH, w.N)
    l_all = views["row_l"].reshape(w.BH, w.N)
    cs_all = views["colsum"].reshape(w.BH, w.n_groups, w.N)
    rng = np.random.default_rng(cfg * 1000 + (k or 0))
    heads = sorted({0, w.BH - 1})
    groups = sorted({0, w.n_groups // 2, w.n_groups - 1})
    n_groups_checked = n_rows_checked = 0
    for bh in heads:
        b, h = divmod(bh, w.H)
        q1, k1, v1 = (x[b, h] for x in s1)
        q2, k2, v2 = (x[b, h] for x in s2)
        perm = perm_all[bh].cpu().numpy()
        ref_perm = orc.group_queries(q1)
        assert np.array_equal(perm, ref_perm), f"{name} head {bh}: perm differs"
        kv = kv_all[bh][groups].cpu().numpy()
        res = res_all[bh].cpu().numpy().astype(np.float64)
        step_out = o_step[b, h].float().cpu().numpy()
        m_gpu = m_all[bh].cpu().numpy().astype(np.float64)
        l_gpu = l_all[bh].cpu().numpy().astype(np.float64)
        cs_gpu = cs_all[bh][groups].cpu().numpy().astype(np.float64)
        for gi, g in enumerate(groups):
            rows = orc.group_rows(ref_perm, w.G, g)
            # a2: log normaliser per row, m within its band
            m_ref, l_ref = orc.row_stats(q1[rows], k1, w.scale)
            lse_gpu = (m_gpu[rows] + np.log2(l_gpu[rows])) * np.log(2.0)
            lse_ref = m_ref + np.log(l_ref)
            assert np.abs(lse_gpu - lse_ref).max() <= LSE_ABS, f"{name} head {bh} group {g}: lse"
            mx = m_ref * np.log2(np.e)
            assert np.all(m_gpu[rows] <= mx + 1e-3) and np.all(m_gpu[rows] >= mx - 32 - 1e-3)
            # a3: group scores element by element
            c = orc.probabilities(q1[rows], k1, w.scale).sum(axis=0)
            err = np.abs(cs_gpu[gi] - c)
            assert np.all(err <= COLSUM_REL * c + COLSUM_ABS), (
                f"{name} head {bh} group {g}: colsum max rel err {float((err / np.maximum(c, 1e-30)).max()):.2e}")
            # a4
            kv_sets_agree(kv[gi], c, w.k)
            # a5, a6 on the GPU's own selection
            R, _, _ = orc.residual_group(q1[rows], k1, v1, w.scale, kv[gi])
            assert_residual_close(res[rows], R, f"{name} head {bh} group {g} residual")
            o_ref = orc.sparse_group(q2[rows], k2, v2, w.scale, kv[gi]) + R
            assert_out_close(step_out[rows], o_ref, f"{name} head {bh} group {g} reused step")
            n_groups_checked += 1
            n_rows_checked += len(rows)
        sample = rng.choice(w.N, size=64, replace=False)
        ref_d1 = orc.dense_rows(q1[sample], k1, v1, w.scale)
        assert_out_close(od1[b, h].float().cpu().numpy()[sample], ref_d1, f"{name} head {bh} plan dense")
        ref_d2 = orc.dense_rows(q2[sample], k2, v2, w.scale)
        assert_out_close(o_dense[b, h].float().cpu().numpy()[sample], ref_d2, f"{name} head {bh} dense")
    print(f"{name}: compared {n_groups_checked} groups, {n_rows_checked} rows (a2, a3, a4, a5, a6)")
    assert n_groups_checked == len(heads) * len(groups) and n_rows_checked > 0
    del meta, od1, o_step, o_dense, ws, views
    torch.cuda.empty_cache()
