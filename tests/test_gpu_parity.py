"""GPU parity of every hot-path step against the fp64 oracle, through the C ABI.

Sizes here finish in seconds in the oracle yet span several 128-row tiles and
ragged tails.  Each stage is also tested alone on oracle-made inputs (the
grouping the oracle chose, the selection the oracle made), so a failure
points at one kernel.
"""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from oracle import mcs_oracle as orc
from tests.gpu_util import (COLSUM_ABS, COLSUM_REL, LSE_ABS, assert_out_close, assert_residual_close,
                            dev_bf16, host, kv_sets_agree)

pytestmark = pytest.mark.gpu

# how far (log2 units) the sparse softmax lets a row's reference max trail the
# running max before it rescales what it has written
RAISE_LOG2 = 32


def _shape_workload(N, d, G, k):
    return synth.workload("tiny").with_(grid=(1, 1, N), d=d, G=G, k=k)


# ----------------------------------------------------------------------------- dense (a7)

DENSE_CASES = [(1, 1, 300, 128, 1.0), (1, 2, 1000, 64, 2.0), (1, 1, 129, 128, 1.0),
               (1, 1, 1, 64, 1.0), (2, 1, 777, 128, 3.0), (1, 1, 128, 64, 1.0)]


@pytest.mark.parametrize("B,H,N,d,qs", DENSE_CASES)
def test_dense_random_shapes(B, H, N, d, qs):
    Q, K, V = synth.random_qkv(B, H, N, d, seed=1, q_std=qs)
    out = host(mcs.dense(dev_bf16(Q), dev_bf16(K), dev_bf16(V)))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    for b in range(B):
        for h in range(H):
            ref = orc.dense_attention(Q[b, h], K[b, h], V[b, h], 1 / np.sqrt(d))
            assert_out_close(out[b, h], ref, f"dense b{b} h{h}")


@pytest.mark.parametrize("N,d", [(1000, 128), (777, 64)])
def test_dense_rising_scores(N, d):
    """Keys whose scale grows with the index: row maxima jump by more than
    2^RAISE_LOG2 between key tiles, so O and l are rescaled mid-row."""
    Q, K, V = synth.rising_qkv(1, 1, N, d, seed=6, growth=40.0)
    out = host(mcs.dense(dev_bf16(Q), dev_bf16(K), dev_bf16(V)))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ref = orc.dense_attention(Q[0, 0], K[0, 0], V[0, 0], 1 / np.sqrt(d))
    assert_out_close(out[0, 0], ref, f"dense rising N{N} d{d}")


def test_dense_tiny_workload():
    w = synth.workload(1)
    Q, K, V = synth.layer_tensors(w)
    out = host(mcs.dense(dev_bf16(Q), dev_bf16(K), dev_bf16(V)))
    for h in range(w.H):
        assert_out_close(out[0, h], orc.dense_attention(Q[0, h], K[0, h], V[0, h], w.scale), f"h{h}")


# ----------------------------------------------------------------------------- reused step (a6)

STEP_CASES = [(1000, 64, 64, 300), (1000, 128, 128, 129), (500, 128, 128, 500), (257, 64, 128, 1),
              (300, 64, 64, 5000), (1024, 128, 64, 257)]


@pytest.mark.parametrize("N,d,G,k", STEP_CASES)
def test_sparse_step_random_metadata(N, d, G, k):
    w = _shape_workload(N, d, G, k)
    Q, K, V = synth.random_qkv(1, 1, N, d, seed=2, q_std=2.0)
    perm, kv, res = synth.random_metadata_head(w, 0)
    meta = mcs.Meta.from_tensors(torch.from_numpy(perm)[None, None].cuda(),
                                 torch.from_numpy(kv)[None, None].cuda(),
                                 torch.from_numpy(res)[None, None].cuda(), G)
    out = host(mcs.sparse_step(dev_bf16(Q), dev_bf16(K), dev_bf16(V), meta))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ref = orc.reused_step_head(Q[0, 0], K[0, 0], V[0, 0], w.scale, perm, kv, res, G)
    assert_out_close(out[0, 0], ref, f"step N{N} d{d} G{G} k{k}")


@pytest.mark.parametrize("N,d,G,k", [(1000, 128, 128, 300), (1000, 64, 64, 600), (700, 128, 128, 700)])
def test_sparse_step_rising_scores(N, d, G, k):
    """Scores that rise steeply along each group's ascending key list: the
    running max is raised by more than 2^RAISE_LOG2 between tiles and inside
    them, so the P chunks a tile has already written get rescaled in place."""
    w = _shape_workload(N, d, G, k)
    Q, K, V = synth.rising_qkv(1, 1, N, d, seed=5, growth=40.0)
    perm, kv, res = synth.random_metadata_head(w, 0)
    # the inputs really do take the rescaling path: for the first group, some
    # 32-key chunk that is not the first of its 128-key tile has a max above
    # every earlier chunk's by more than 2^RAISE_LOG2
    s = orc.scores(Q[0, 0][perm[:G]], K[0, 0], w.scale) * np.log2(np.e)
    row = s[:, kv[0]]
    nch = -(-row.shape[1] // 32)
    padded = np.full((G, nch * 32), -np.inf)
    padded[:, :row.shape[1]] = row
    chunk_max = padded.reshape(G, nch, 32).max(axis=2)
    raised = chunk_max[:, 1:] > np.maximum.accumulate(chunk_max, axis=1)[:, :-1] + RAISE_LOG2
    assert raised[:, np.arange(1, nch) % 4 != 0].any()
    meta = mcs.Meta.from_tensors(torch.from_numpy(perm)[None, None].cuda(),
                                 torch.from_numpy(kv)[None, None].cuda(),
                                 torch.from_numpy(res)[None, None].cuda(), G)
    out = host(mcs.sparse_step(dev_bf16(Q), dev_bf16(K), dev_bf16(V), meta))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ref = orc.reused_step_head(Q[0, 0], K[0, 0], V[0, 0], w.scale, perm, kv, res, G)
    assert_out_close(out[0, 0], ref, f"rising step N{N} d{d} G{G} k{k}")


def test_sparse_step_on_oracle_plan_with_drift():
    """Tiny workload: the oracle plans at step 1; the GPU reuses that metadata
    on the drifted step-2 inputs."""
    w = synth.workload(1)
    Q1, K1, V1 = synth.layer_tensors(w, step=1)
    Q2, K2, V2 = synth.layer_tensors(w, step=2)
    metas = [orc.plan_head(Q1[0, h], K1[0, h], V1[0, h], w.G, w.k, w.scale) for h in range(w.H)]
    perm = np.stack([m["perm"] for m in metas]).astype(np.int32)[None]
    kv = np.stack([m["kv_idx"] for m in metas]).astype(np.int32)[None]
    res = np.stack([m["residual"] for m in metas]).astype(np.float32)[None]
    meta = mcs.Meta.from_tensors(torch.from_numpy(perm).cuda(), torch.from_numpy(kv).cuda(),
                                 torch.from_numpy(res).cuda(), w.G)
    out = host(mcs.sparse_step(dev_bf16(Q2), dev_bf16(K2), dev_bf16(V2), meta))
    for h in range(w.H):
        ref = orc.reused_step_head(Q2[0, h], K2[0, h], V2[0, h], w.scale, perm[0, h], kv[0, h],
                                   res[0, h], w.G)
        assert_out_close(out[0, h], ref, f"reused step h{h}")


# ----------------------------------------------------------------------------- grouping (a1)

@pytest.mark.parametrize("cfg_or_shape", [1, (1, 2, 1000, 64), (1, 1, 3000, 128), (1, 1, 1, 128)])
def test_plan_group_matches_oracle_order(cfg_or_shape):
    if isinstance(cfg_or_shape, int):
        w = synth.workload(cfg_or_shape)
        Q, _, _ = synth.layer_tensors(w)
    else:
        B, H, N, d = cfg_or_shape
        Q, _, _ = synth.random_qkv(B, H, N, d, seed=3)
    perm = mcs.plan_group(dev_bf16(Q)).cpu().numpy()
    B, H = Q.shape[:2]
    for b in range(B):
        for h in range(H):
            ref = orc.group_queries(Q[b, h])
            assert np.array_equal(np.sort(perm[b, h]), np.arange(Q.shape[2]))
            assert np.array_equal(perm[b, h], ref), f"b{b} h{h}: {np.sum(perm[b, h] != ref)} positions differ"


@pytest.mark.parametrize("N,d,BH", [(5000, 64, 1), (9000, 128, 2), (3100, 64, 3)])
def test_plan_group_stable_on_ties_across_sort_chunks(N, d, BH):
    """Runs of identical query rows give identical projections, so their
    order is decided by the sort's stability alone (ascending token index).
    At these sizes a head's sort is split over several CTAs (chunks of 1024
    keys, the last one ragged), so equal keys meet across chunk borders."""
    rng = np.random.default_rng(N + d)
    Q, _, _ = synth.random_qkv(1, BH, N, d, seed=9)
    for h in range(BH):
        src = rng.integers(0, N, size=N // 3)          # a third of the rows copy another row
        dst = rng.integers(0, N, size=N // 3)
        Q[0, h, dst] = Q[0, h, src]
    perm = mcs.plan_group(dev_bf16(Q)).cpu().numpy()
    for h in range(BH):
        ref = orc.group_queries(Q[0, h])
        assert np.array_equal(perm[0, h], ref), f"h{h}: {np.sum(perm[0, h] != ref)} positions differ"


# ----------------------------------------------------------------------------- selection (a2-a4)

@pytest.mark.parametrize("cfg,G,k", [(1, 64, 128), (1, 128, 300), (1, 64, 1), (1, 128, 1024)])
def test_plan_select_on_oracle_grouping(cfg, G, k):
    w = synth.workload(cfg, G=G, k=k)
    Q, K, V = synth.layer_tensors(w)
    perms = np.stack([orc.group_queries(Q[0, h]) for h in range(w.H)]).astype(np.int32)[None]
    kv = mcs.plan_select(dev_bf16(Q), dev_bf16(K), dev_bf16(V), torch.from_numpy(perms).cuda(), G,
                         k).cpu().numpy()
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    assert kv.shape == (1, w.H, w.n_groups, min(k, w.N))
    ndiff = 0
    for h in range(w.H):
        c = orc.group_prob_sums(Q[0, h], K[0, h], w.scale, perms[0, h], G)
        for g in range(w.n_groups):
            ndiff += kv_sets_agree(kv[0, h, g], c[g], k)
    assert ndiff <= 2 * w.H * w.n_groups


@pytest.mark.parametrize("N,d,G,k", [(1000, 128, 128, 100), (777, 64, 64, 50), (129, 128, 64, 16),
                                     (100, 64, 64, 10)])
def test_plan_stats_rising_scores(N, d, G, k):
    """Statistics pass on keys whose scale grows with the index, so row maxima
    jump by more than 2^RAISE_LOG2 inside and between key tiles (m, l, the
    output accumulators and P already written are rescaled): its dense output
    and the selection it drives match the oracle."""
    Q, K, V = synth.rising_qkv(1, 1, N, d, seed=7, growth=40.0)
    q, kd, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    scale = 1 / np.sqrt(d)
    perm = orc.group_queries(Q[0, 0]).astype(np.int32)
    ws, od = mcs.plan_stats(q, kd, v, G, k, return_dense=True)
    mcs.plan_scores(q, kd, torch.from_numpy(perm[None, None].copy()).cuda(), G, k, ws)
    kv = mcs.plan_topk(1, 1, N, d, G, k, ws).cpu().numpy()
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ref = orc.dense_attention(Q[0, 0], K[0, 0], V[0, 0], scale)
    assert_out_close(host(od)[0, 0], ref, f"plan dense rising N{N} d{d}")
    # the steepest rows put most keys' probabilities below fp32's range
    c = orc.group_prob_sums(Q[0, 0], K[0, 0], scale, perm, G)
    for g in range(c.shape[0]):
        kv_sets_agree(kv[0, 0, g], c[g], k, G=G)


# ----------------------------------------------------------------------------- residual (a5)

@pytest.mark.parametrize("cfg,G,k", [(1, 64, 128), (1, 128, 200)])
def test_plan_residual_on_oracle_metadata(cfg, G, k):
    w = synth.workload(cfg, G=G, k=k)
    Q, K, V = synth.layer_tensors(w)
    metas = [orc.plan_head(Q[0, h], K[0, h], V[0, h], G, k, w.scale) for h in range(w.H)]
    perm = np.stack([m["perm"] for m in metas]).astype(np.int32)[None]
    kv = np.stack([m["kv_idx"] for m in metas]).astype(np.int32)[None]
    res, od = mcs.plan_residual(dev_bf16(Q), dev_bf16(K), dev_bf16(V), torch.from_numpy(perm).cuda(),
                                torch.from_numpy(kv).cuda(), G, return_dense=True)
    res, od = res.cpu().numpy().astype(np.float64), host(od)
    for h in range(w.H):
        assert_residual_close(res[0, h], metas[h]["residual"], f"residual h{h}")
        assert_out_close(od[0, h], metas[h]["O_dense"], f"plan dense h{h}")


# ----------------------------------------------------------------------------- whole plan (a1-a5)

@pytest.mark.parametrize("cfg,G,k", [(1, 64, 128), (1, 128, 77)])
def test_plan_end_to_end(cfg, G, k):
    """The whole plan, then the comparison protocol: perm equal to the
    oracle's; every group's KV set within the 1e-4 band of the oracle's
    scores; then the residual of EVERY group recomputed by the oracle on the
    GPU's own selection; the dense output; and a reused step on the plan's
    own inputs, which must reproduce dense attention."""
    w = synth.workload(cfg, G=G, k=k)
    Q, K, V = synth.layer_tensors(w)
    q, kd, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    ws = mcs.alloc_workspace(w.B, w.H, w.N, w.d, G, k, q.device)
    meta, od = mcs.plan(q, kd, v, G, k, workspace=ws, return_dense=True)
    o_step = host(mcs.sparse_step(q, kd, v, meta))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ok, code = mcs.validate_meta(meta)
    assert ok, code
    views = mcs.workspace_views(ws, w.B, w.H, w.N, w.d, G, k)
    perm = meta.perm.cpu().numpy()
    kv = meta.kv_idx.cpu().numpy()
    res = meta.residual.cpu().numpy().astype(np.float64)
    cs = views["colsum"].cpu().numpy().astype(np.float64)
    od = host(od)
    n_groups = 0
    for h in range(w.H):
        ref = orc.plan_head(Q[0, h], K[0, h], V[0, h], G, k, w.scale)
        assert np.array_equal(perm[0, h], ref["perm"])
        c = orc.group_prob_sums(Q[0, h], K[0, h], w.scale, ref["perm"], G)
        assert np.all(np.abs(cs[0, h] - c) <= COLSUM_REL * c + COLSUM_ABS)
        for g in range(w.n_groups):
            kv_sets_agree(kv[0, h, g], c[g], k)
            rows = orc.group_rows(ref["perm"], G, g)
            R, _, _ = orc.residual_group(Q[0, h][rows], K[0, h], V[0, h], w.scale, kv[0, h, g])
            assert_residual_close(res[0, h][rows], R, f"plan residual h{h} g{g}")
            n_groups += 1
        assert_out_close(od[0, h], ref["O_dense"], f"plan O_dense h{h}")
        # a reused step on the plan's own inputs reproduces dense attention
        assert_out_close(o_step[0, h], ref["O_dense"], f"step on unchanged inputs h{h}")
    assert n_groups == w.H * w.n_groups


@pytest.mark.parametrize("N,d,G", [(1000, 128, 128), (777, 64, 64)])
def test_plan_statistics_elementwise(N, d, G):
    """a2 and a3 read back from the workspace: every row's log normaliser
    m + log2 l against the oracle's row statistics (m inside its documented
    band), and every group score against the oracle's sums of exact
    probabilities."""
    Q, K, V = synth.random_qkv(1, 1, N, d, seed=15, q_std=2.0)
    q, kd, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    k = 100
    perm = orc.group_queries(Q[0, 0]).astype(np.int32)
    ws = mcs.alloc_workspace(1, 1, N, d, G, k, q.device)
    mcs.plan_stats(q, kd, v, G, k, workspace=ws)
    mcs.plan_scores(q, kd, torch.from_numpy(perm[None, None].copy()).cuda(), G, k, ws)
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    views = mcs.workspace_views(ws, 1, 1, N, d, G, k)
    m_gpu = views["row_m"][0, 0].cpu().numpy().astype(np.float64)
    l_gpu = views["row_l"][0, 0].cpu().numpy().astype(np.float64)
    m_ref, l_ref = orc.row_stats(Q[0, 0], K[0, 0], 1 / np.sqrt(d))
    lse_gpu = (m_gpu + np.log2(l_gpu)) * np.log(2.0)
    assert np.abs(lse_gpu - (m_ref + np.log(l_ref))).max() <= LSE_ABS
    mx = m_ref * np.log2(np.e)
    assert np.all(m_gpu <= mx + 1e-3) and np.all(m_gpu >= mx - 32 - 1e-3)
    c = orc.group_prob_sums(Q[0, 0], K[0, 0], 1 / np.sqrt(d), perm, G)
    cs = views["colsum"][0, 0].cpu().numpy().astype(np.float64)
    assert cs.shape == c.shape
    assert np.all(np.abs(cs - c) <= COLSUM_REL * c + COLSUM_ABS)
    # O32, the plan's fp32 dense output, against the oracle's dense attention
    o32 = views["O32"][0, 0].cpu().numpy().astype(np.float64)
    ref = orc.dense_attention(Q[0, 0], K[0, 0], V[0, 0], 1 / np.sqrt(d))
    assert_residual_close(o32, ref, "plan fp32 dense output")


@pytest.mark.parametrize("N,d,G", [(1000, 128, 128), (700, 64, 64)])
def test_plan_with_k_equal_n(N, d, G):
    """k = N keeps every key: the residual vanishes (up to the fp32 rounding
    of two equal sums) and a reused step, on these or on drifted inputs,
    equals dense attention of its own inputs."""
    Q, K, V = synth.random_qkv(1, 1, N, d, seed=16, q_std=2.0)
    q, kd, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    meta, od = mcs.plan(q, kd, v, G, N, return_dense=True)
    torch.cuda.synchronize()
    assert meta.k == N
    res = meta.residual.cpu().numpy().astype(np.float64)
    ref = orc.dense_attention(Q[0, 0], K[0, 0], V[0, 0], 1 / np.sqrt(d))
    assert np.linalg.norm(res[0, 0]) <= 1e-3 * np.linalg.norm(ref)
    assert_out_close(host(mcs.sparse_step(q, kd, v, meta))[0, 0], ref, "k = N step, plan inputs")
    Q2, K2, V2 = synth.random_qkv(1, 1, N, d, seed=17, q_std=2.0)
    o2 = host(mcs.sparse_step(dev_bf16(Q2), dev_bf16(K2), dev_bf16(V2), meta))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ref2 = orc.dense_attention(Q2[0, 0], K2[0, 0], V2[0, 0], 1 / np.sqrt(d))
    assert_out_close(o2[0, 0], ref2, "k = N step, other inputs")


# ----------------------------------------------------------------------------- failure handling

def test_bounded_wait_times_out_and_context_survives():
    mcs.last_device_status()                 # clear
    mcs.selftest_wait_timeout(2_000_000)     # 2 ms on an mbarrier nothing arrives on
    assert mcs.last_device_status() == 5
    Q, K, V = synth.random_qkv(1, 1, 200, 64, seed=4)
    out = host(mcs.dense(dev_bf16(Q), dev_bf16(K), dev_bf16(V)))
    assert mcs.last_device_status() == 0
    assert_out_close(out[0, 0], orc.dense_attention(Q[0, 0], K[0, 0], V[0, 0], 0.125), "after timeout")


def _oracle_meta_tiny():
    w = synth.workload(1)
    Q, K, V = synth.layer_tensors(w)
    metas = [orc.plan_head(Q[0, h], K[0, h], V[0, h], w.G, w.k, w.scale) for h in range(w.H)]
    perm = np.stack([m["perm"] for m in metas]).astype(np.int32)[None]
    kv = np.stack([m["kv_idx"] for m in metas]).astype(np.int32)[None]
    res = np.stack([m["residual"] for m in metas]).astype(np.float32)[None]
    return w, (Q, K, V), perm, kv, res


def test_validate_meta_flags_each_corruption():
    w, _, perm, kv, res = _oracle_meta_tiny()
    mk = lambda p, k_, r: mcs.Meta.from_tensors(torch.from_numpy(p).cuda(), torch.from_numpy(k_).cuda(),
                                                torch.from_numpy(r).cuda(), w.G)
    assert mcs.validate_meta(mk(perm, kv, res)) == (True, 0)
    p2 = perm.copy(); p2[0, 1, 5] = p2[0, 1, 6]
    assert mcs.validate_meta(mk(p2, kv, res)) == (False, 1)
    k2 = kv.copy(); k2[0, 0, 3, 7] = w.N
    assert mcs.validate_meta(mk(perm, k2, res)) == (False, 2)
    k3 = kv.copy(); k3[0, 0, 3, 7] = k3[0, 0, 3, 6]
    assert mcs.validate_meta(mk(perm, k3, res)) == (False, 3)
    r2 = res.copy(); r2[0, 1, 10, 3] = np.nan
    assert mcs.validate_meta(mk(perm, kv, r2)) == (False, 4)


def test_out_of_range_index_is_reported_not_gathered():
    w, (Q, K, V), perm, kv, res = _oracle_meta_tiny()
    k2 = kv.copy()
    k2[0, 0, 2, -1] = w.N + 1000        # the kernel must mask it and report
    meta = mcs.Meta.from_tensors(torch.from_numpy(perm).cuda(), torch.from_numpy(k2).cuda(),
                                 torch.from_numpy(res).cuda(), w.G)
    mcs.last_device_status()
    mcs.sparse_step(dev_bf16(Q), dev_bf16(K), dev_bf16(V), meta)
    assert mcs.last_device_status() == 6
