"""The compact (bf16) cached residual: its conversion and the reused step
that reads it (mcs_residual_compact, mcs_sparse_step_compact).

* conversion: bit for bit the oracle's round-to-nearest-even of every
  float32 input (random magnitudes, exact ties, overflow, subnormals,
  infinities; NaN stays NaN), at ragged lengths;
* the compact step writes the same bits as the fp32 step given the widened
  bf16 residual (the epilogue adds the same float32 values);
* on planned DiT-shaped inputs it matches the fp64 oracle's sparse attention
  plus the oracle's bf16 rounding of the plan's residual.
"""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
import synth
from oracle import mcs_oracle as orc
from tests.gpu_util import assert_out_close, dev_bf16, host

pytestmark = pytest.mark.gpu


def _inputs(n, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(n) * np.exp2(rng.integers(-30, 30, n))).astype(np.float32)
    bits = x.view(np.uint32)
    bits[: n // 8] = (bits[: n // 8] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)   # exact ties
    special = np.array([np.inf, -np.inf, 3.4e38, -3.4e38, 1e-40, -3e-39, 0.0, -0.0], dtype=np.float32)
    m = min(len(special), n - n // 8)
    x[n // 8: n // 8 + m] = special[:m]
    return x


@pytest.mark.parametrize("n", [1, 7, 8, 1000003, 4 * 1024 * 1024 + 5])
def test_conversion_is_round_to_nearest_even(n):
    x = _inputs(n, n)
    got = mcs.compact_residual(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    got = got.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, orc.round_bf16(x))
    nan = np.array([np.nan, 1.0] * 4, dtype=np.float32)
    g = mcs.compact_residual(torch.from_numpy(nan).cuda()).float().cpu().numpy()
    assert np.isnan(g[0::2]).all() and (g[1::2] == 1.0).all()


@pytest.mark.parametrize("N,d,G,k", [(1000, 64, 64, 300), (2048, 128, 128, 700), (777, 128, 128, 1)])
def test_compact_step_equals_fp32_step_on_the_rounded_residual(N, d, G, k):
    w = synth.workload("tiny").with_(grid=(1, 1, N), d=d, G=G, k=k)
    Q, K, V = (dev_bf16(x) for x in synth.layer_tensors(w, step=2))
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    md = [synth.random_metadata_head(w, h, r_scale=3.0) for h in range(w.H)]
    perm, kv, res = (t(np.stack([m[i] for m in md])[None]) for i in range(3))
    r16 = mcs.compact_residual(res)
    meta = mcs.Meta.from_tensors(perm, kv, r16.float(), G)
    o32 = mcs.sparse_step(Q, K, V, meta)
    o16 = mcs.sparse_step_compact(Q, K, V, mcs.Meta.from_tensors(perm, kv, res, G), r16)
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    assert torch.equal(o16, o32)


def test_compact_step_matches_the_oracle():
    w = synth.workload(1).with_(grid=(4, 8, 32), G=128, k=256)          # N = 1024
    Q, K, V = synth.layer_tensors(w)
    ws = mcs.alloc_workspace(w.B, w.H, w.N, w.d, w.G, w.k, "cuda")
    meta = mcs.plan(dev_bf16(Q), dev_bf16(K), dev_bf16(V), w.G, w.k, workspace=ws)
    r16 = mcs.compact_residual(meta.residual)
    Q2, K2, V2 = synth.layer_tensors(w, step=2)
    out = host(mcs.sparse_step_compact(dev_bf16(Q2), dev_bf16(K2), dev_bf16(V2), meta, r16))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    perm, kv = meta.perm.cpu().numpy(), meta.kv_idx.cpu().numpy()
    R = orc.widen_bf16(orc.round_bf16(meta.residual.cpu().numpy()))
    for h in range(w.H):
        for g in range(w.n_groups):
            rows = orc.group_rows(perm[0, h], w.G, g)
            o = orc.sparse_group(Q2[0, h][rows], K2[0, h], V2[0, h], w.scale, kv[0, h, g]) + R[0, h][rows]
            assert_out_close(out[0, h][rows], o, f"compact step h{h} g{g}")
