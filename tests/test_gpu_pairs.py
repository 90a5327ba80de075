"""The reused step over pairs of adjacent query groups (pair_kernel.cuh).

The pair union lists are an execution order, not a new quantity: for groups
2p and 2p+1 the union of their kept keys, ordered [only 2p | both | only
2p+1] with each segment ascending.  They are checked entry for entry against
a plain restatement here, and the step that runs over them is checked against
the fp64 oracle's reused step, and against the one-group-at-a-time kernel, on
the same metadata: random key sets (little overlap), the oracle's own plans
(large overlap), k >= N (the two lists coincide), k = 1, odd numbers of
groups (a lone last group), partial last groups and G = 64.
"""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from oracle import mcs_oracle as orc
from tests.gpu_util import assert_out_close, dev_bf16, host

pytestmark = pytest.mark.gpu


def union_lists(kv: np.ndarray):
    """[n_pairs] lists: keys only group 2p keeps, then keys both keep, then keys
    only 2p+1 keeps, each in ascending order (a lone last group: its own list)."""
    out = []
    ng = kv.shape[0]
    for p in range((ng + 1) // 2):
        A = kv[2 * p].tolist()
        if 2 * p + 1 >= ng:
            out.append(A)
            continue
        B = kv[2 * p + 1].tolist()
        sa, sb = set(A), set(B)
        out.append([x for x in A if x not in sb] + [x for x in A if x in sb] + [x for x in B if x not in sa])
    return out


def _meta(perm, kv, res, G, pairs=True):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return mcs.Meta.from_tensors(t(perm)[None, None], t(kv)[None, None], t(res)[None, None], G, pairs=pairs)


def _shape_workload(N, d, G, k):
    return synth.workload("tiny").with_(grid=(1, 1, N), d=d, G=G, k=k)


LIST_CASES = [(1000, 64, 128, 300), (1000, 128, 64, 129), (300, 64, 64, 5000), (257, 64, 128, 1),
              (900, 128, 128, 450), (129, 64, 64, 128)]


@pytest.mark.parametrize("N,d,G,k", LIST_CASES)
def test_pair_lists_match_their_definition(N, d, G, k):
    w = _shape_workload(N, d, G, k)
    perm, kv, res = synth.random_metadata_head(w, 0)
    meta = _meta(perm, kv, res, G)
    torch.cuda.synchronize()
    kk = min(k, N)
    ref = union_lists(kv)
    got_idx = meta.pair_idx[0, 0].cpu().numpy()
    got_len = meta.pair_len[0, 0].cpu().numpy()
    assert len(ref) == meta.n_pairs
    for p, lst in enumerate(ref):
        assert got_len[p] == len(lst), (p, got_len[p], len(lst))
        assert np.array_equal(got_idx[p, :len(lst)], np.asarray(lst)), p
        # group 2p's keys are positions [0, k), group 2p+1's [u - k, u)
        assert set(got_idx[p, :kk].tolist()) == set(kv[2 * p].tolist())
        if 2 * p + 1 < w.n_groups:
            u = int(got_len[p])
            assert set(got_idx[p, u - kk:u].tolist()) == set(kv[2 * p + 1].tolist())
    ok, code = mcs.validate_meta(meta)
    assert ok, code


def test_pair_lists_on_oracle_plans_overlap():
    """On the oracle's plans of the tiny DiT layer adjacent groups keep mostly
    the same keys, so the unions are short: the case the pair kernel is for."""
    w = synth.workload(1)
    Q, K, V = synth.layer_tensors(w)
    for h in range(w.H):
        m = orc.plan_head(Q[0, h], K[0, h], V[0, h], w.G, w.k, w.scale)
        meta = _meta(m["perm"].astype(np.int32), m["kv_idx"].astype(np.int32),
                     m["residual"].astype(np.float32), w.G)
        got_len = meta.pair_len[0, 0].cpu().numpy()
        ref = union_lists(m["kv_idx"])
        assert [len(x) for x in ref] == got_len.tolist()
        assert got_len.mean() < 1.6 * w.k      # measured: about 1.25 k


STEP_CASES = [(1000, 64, 64, 300), (1000, 128, 128, 129), (500, 128, 128, 500), (257, 64, 128, 1),
              (300, 64, 64, 5000), (1024, 128, 64, 257), (900, 128, 128, 700), (2000, 128, 128, 1000),
              (129, 64, 64, 64)]


@pytest.mark.parametrize("N,d,G,k", STEP_CASES)
def test_pair_step_matches_oracle_and_single_group_kernel(N, d, G, k):
    w = _shape_workload(N, d, G, k)
    Q, K, V = synth.random_qkv(1, 1, N, d, seed=12, q_std=2.0)
    perm, kv, res = synth.random_metadata_head(w, 0)
    q, kd, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    meta = _meta(perm, kv, res, G)
    out_pairs = host(mcs.sparse_step(q, kd, v, meta))
    out_single = host(mcs.sparse_step(q, kd, v, meta.without_pairs()))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ref = orc.reused_step_head(Q[0, 0], K[0, 0], V[0, 0], w.scale, perm, kv, res, G)
    assert_out_close(out_pairs[0, 0], ref, f"pair step N{N} d{d} G{G} k{k}")
    assert_out_close(out_single[0, 0], ref, f"single-group step N{N} d{d} G{G} k{k}")
    # both kernels carry ~2^-17 relative error in the sparse output before the
    # bf16 rounding of O, so they agree to within one bf16 rounding step
    assert np.abs(out_pairs - out_single).max() <= 2 ** -7 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("N,d,G,k", [(1000, 128, 128, 300), (1000, 64, 64, 600)])
def test_pair_step_rising_scores(N, d, G, k):
    """Scores that rise steeply along the key lists: running maxima move by
    more than 2^32 inside and between tiles, so P chunks already written and
    O are rescaled in place."""
    w = _shape_workload(N, d, G, k)
    Q, K, V = synth.rising_qkv(1, 1, N, d, seed=5, growth=40.0)
    perm, kv, res = synth.random_metadata_head(w, 0)
    out = host(mcs.sparse_step(dev_bf16(Q), dev_bf16(K), dev_bf16(V), _meta(perm, kv, res, G)))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    ref = orc.reused_step_head(Q[0, 0], K[0, 0], V[0, 0], w.scale, perm, kv, res, G)
    assert_out_close(out[0, 0], ref, f"rising pair step N{N} d{d} G{G} k{k}")


def test_pair_step_multi_head_multi_batch():
    """Items cross head boundaries on the persistent CTAs: B = 2, H = 3."""
    B, H, N, d, G, k = 2, 3, 700, 64, 128, 200
    w = _shape_workload(N, d, G, k)
    Q, K, V = synth.random_qkv(B, H, N, d, seed=13, q_std=2.0)
    heads = [synth.random_metadata_head(w, bh) for bh in range(B * H)]
    perm = np.stack([x[0] for x in heads]).reshape(B, H, N)
    kv = np.stack([x[1] for x in heads]).reshape(B, H, w.n_groups, k)
    res = np.stack([x[2] for x in heads]).reshape(B, H, N, d)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    meta = mcs.Meta.from_tensors(t(perm), t(kv), t(res), G)
    out = host(mcs.sparse_step(dev_bf16(Q), dev_bf16(K), dev_bf16(V), meta))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    for b in range(B):
        for h in range(H):
            ref = orc.reused_step_head(Q[b, h], K[b, h], V[b, h], w.scale, perm[b, h], kv[b, h], res[b, h], G)
            assert_out_close(out[b, h], ref, f"b{b} h{h}")


def test_corrupt_pair_length_is_reported_not_read_past():
    w = _shape_workload(1000, 64, 128, 300)
    Q, K, V = synth.random_qkv(1, 1, 1000, 64, seed=14)
    perm, kv, res = synth.random_metadata_head(w, 0)
    meta = _meta(perm, kv, res, 128)
    meta.pair_len[0, 0, 1] = 10 ** 6          # far past the list's 2k entries
    assert mcs.validate_meta(meta) == (False, 5)
    mcs.last_device_status()
    mcs.sparse_step(dev_bf16(Q), dev_bf16(K), dev_bf16(V), meta)
    assert mcs.last_device_status() == 6
    meta.build_pairs()                         # rebuilt from kv_idx: valid again
    assert mcs.validate_meta(meta) == (True, 0)
