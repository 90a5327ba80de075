"""The reused step over a block-granular selection (mcs_sparse_step_blocks),
the coarse-block pattern MC-Sparse's individual KV selection replaces
(cctest.ai article, "Individual KV selection").

* block indices: `select_block_indices` names exactly the blocks whose keys
  `select_blocks` lists;
* pair lists over block indices match their definition entry for entry;
* the block step writes the same bits as the token step given the expanded
  keys of the same blocks (same union order, same tiles), with and without
  a residual, on ragged N, odd group counts, G = 64 and 128, d = 64 and 128,
  blocks of 64 and 128;
* on planned DiT-shaped inputs it matches the fp64 oracle's sparse attention
  over the blocks' keys plus the oracle's residual of those keys;
* an out-of-range block index is reported (MCS_ERR_BAD_META), never loaded.
"""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from oracle import mcs_oracle as orc
from tests.gpu_util import assert_out_close, assert_residual_close, dev_bf16, host
from tests.test_gpu_pairs import union_lists

pytestmark = pytest.mark.gpu

BAD_META = 6


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _expand(blk: np.ndarray, block: int) -> np.ndarray:
    """[..., kb] block indices -> [..., kb * block] ascending keys."""
    return (blk[..., :, None] * block + np.arange(block)).reshape(*blk.shape[:-1], -1).astype(np.int32)


def test_block_indices_name_the_listed_blocks():
    rng = np.random.default_rng(5)
    for N, block, kb in [(1000, 64, 7), (4096, 128, 32), (333, 64, 5), (8192, 64, 1)]:
        scores = _t(rng.random((3, 5, N), dtype=np.float32))
        keys = mcs.select_blocks(scores, kb, block)
        blk = mcs.select_block_indices(scores, kb, block)
        torch.cuda.synchronize()
        keys, blk = keys.cpu().numpy(), blk.cpu().numpy()
        assert np.all(np.diff(blk, axis=-1) > 0) and blk.min() >= 0 and blk.max() < N // block
        assert np.array_equal(_expand(blk, block), keys)


@pytest.mark.parametrize("N,G,block,kb", [(1000, 64, 64, 5), (4096, 128, 128, 9), (1280, 128, 64, 20)])
def test_block_pair_lists_match_their_definition(N, G, block, kb):
    w = synth.workload("tiny").with_(grid=(1, 1, N), G=G)
    blk = np.stack([synth.random_blocks_head(w, h, block, kb) for h in range(2)])[None]
    pidx, plen = mcs.union_pairs(_t(blk))
    torch.cuda.synchronize()
    pidx, plen = pidx.cpu().numpy(), plen.cpu().numpy()
    for h in range(2):
        for p, ref in enumerate(union_lists(blk[0, h])):
            assert plen[0, h, p] == len(ref)
            assert pidx[0, h, p, :len(ref)].tolist() == ref


STEP_CASES = [
    # N, d, G, block, kb
    (1000, 64, 64, 64, 5),      # ragged N (15 full blocks), ragged last group, odd group count
    (1024, 128, 128, 64, 16),   # every block kept (k = N)
    (4096, 128, 128, 128, 7),
    (2500, 128, 64, 128, 3),
    (1100, 64, 128, 64, 1),     # one block per group
]


@pytest.mark.parametrize("N,d,G,block,kb", STEP_CASES)
@pytest.mark.parametrize("with_residual", [True, False])
def test_block_step_equals_token_step_on_expanded_keys(N, d, G, block, kb, with_residual):
    w = synth.workload("tiny").with_(grid=(1, 1, N), d=d, G=G)
    Q, K, V = (dev_bf16(x) for x in synth.layer_tensors(w, step=2))
    perm = np.stack([synth.random_metadata_head(w, h)[0] for h in range(w.H)])[None]
    res = np.stack([synth.random_metadata_head(w, h)[2] for h in range(w.H)])[None]
    blk = np.stack([synth.random_blocks_head(w, h, block, kb) for h in range(w.H)])[None]
    res_t = _t(res) if with_residual else torch.zeros((1, w.H, N, d), dtype=torch.float32, device="cuda")
    meta = mcs.Meta.from_tensors(_t(perm), _t(_expand(blk, block)), res_t, G)
    bm = mcs.BlockMeta.build(_t(perm), _t(blk), G, block, _t(res) if with_residual else None)
    o_tok = mcs.sparse_step(Q, K, V, meta)
    o_blk = mcs.sparse_step_blocks(Q, K, V, bm)
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    assert torch.equal(o_blk, o_tok)       # -0 and +0 compare equal (a zero residual may flip a sign)


@pytest.mark.parametrize("block", [64, 128])
def test_block_step_matches_the_oracle(block):
    w = synth.workload(1).with_(grid=(4, 8, 32), G=128, k=512)          # N = 1024
    Q, K, V = synth.layer_tensors(w)
    q, kd, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    ws = mcs.alloc_workspace(w.B, w.H, w.N, w.d, w.G, w.k, q.device)
    meta = mcs.plan(q, kd, v, w.G, w.k, workspace=ws)
    colsum = mcs.workspace_views(ws, w.B, w.H, w.N, w.d, w.G, w.k)["colsum"]
    kb = w.k // block
    blk = mcs.select_block_indices(colsum, kb, block)
    keys = mcs.select_blocks(colsum, kb, block)
    res = mcs.plan_residual(q, kd, v, meta.perm, keys, w.G, workspace=ws, stats_done=True)
    Q2, K2, V2 = synth.layer_tensors(w, step=2)
    q2, k2, v2 = dev_bf16(Q2), dev_bf16(K2), dev_bf16(V2)
    out = host(mcs.sparse_step_blocks(q2, k2, v2, mcs.BlockMeta.build(meta.perm, blk, w.G, block, res)))
    out_nr = host(mcs.sparse_step_blocks(q2, k2, v2, mcs.BlockMeta.build(meta.perm, blk, w.G, block)))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    blk, perm = blk.cpu().numpy(), meta.perm.cpu().numpy()
    res = res.cpu().numpy().astype(np.float64)
    for h in range(w.H):
        for g in range(w.n_groups):
            kv = _expand(blk[0, h, g], block)
            rows = orc.group_rows(perm[0, h], w.G, g)
            R, _, _ = orc.residual_group(Q[0, h][rows], K[0, h], V[0, h], w.scale, kv)
            assert_residual_close(res[0, h][rows], R, f"block{block} residual h{h} g{g}")
            s = orc.sparse_group(Q2[0, h][rows], K2[0, h], V2[0, h], w.scale, kv)
            assert_out_close(out_nr[0, h][rows], s, f"block{block} step without residual h{h} g{g}")
            assert_out_close(out[0, h][rows], s + R, f"block{block} step h{h} g{g}")


def test_out_of_range_block_index_is_reported():
    N, d, G, block, kb = 1024, 128, 128, 64, 4
    w = synth.workload("tiny").with_(grid=(1, 1, N), d=d, G=G)
    Q, K, V = (dev_bf16(x) for x in synth.layer_tensors(w))
    perm = np.stack([synth.random_metadata_head(w, h)[0] for h in range(w.H)])[None]
    blk = np.stack([synth.random_blocks_head(w, h, block, kb) for h in range(w.H)])[None]
    bm = mcs.BlockMeta.build(_t(perm), _t(blk), G, block)
    mcs.sparse_step_blocks(Q, K, V, bm)
    assert mcs.last_device_status() == 0
    good = bm.pair_idx[0, 1, 1, 0].item()
    bm.pair_idx[0, 1, 1, 0] = N // block          # one past the last block: the kernel loads block 0 instead
    mcs.sparse_step_blocks(Q, K, V, bm)
    assert mcs.last_device_status() == BAD_META
    bm.pair_idx[0, 1, 1, 0] = good
    bm.pair_len[0, 0, 2] = 3 * kb                 # longer than two lists: clamped, never read past
    mcs.sparse_step_blocks(Q, K, V, bm)
    assert mcs.last_device_status() == BAD_META
