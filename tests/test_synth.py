"""The seeded input generator: determinism, structure, bf16 rounding."""
import numpy as np
import torch

import synth
from synth import dit_inputs as di


def test_workload_shapes_and_k():
    c = synth.WORKLOADS
    assert (c[1].N, c[1].k, c[1].n_groups) == (1024, 128, 16)
    assert (c[2].N, c[2].k, c[2].n_groups) == (15600, 1560, 122)
    assert (c[3].N, c[3].k, c[3].n_groups) == (32760, 1638, 256)
    assert (c[4].N, c[4].k, c[4].BH) == (65536, 1966, 32)
    assert c[5].N == 131072
    ks = sorted({w.k for _, _, w in synth.sweep_points()})
    assert ks == [1310, 2621, 6553, 13107, 32768]
    assert c[3].N - (c[3].n_groups - 1) * c[3].G == 120
    assert c[2].N - (c[2].n_groups - 1) * c[2].G == 112


def test_bf16_round_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10,
                        np.array([1.00390625, 1.01171875, -1.00390625, 0.0, 65504.0],
                                 dtype=np.float32)])
    got = di.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_heads_deterministic_and_independently_regenerable():
    w = synth.workload("tiny")
    Q, K, V = synth.layer_tensors(w)
    assert Q.shape == (1, 2, 1024, 64) and Q.dtype == np.uint16
    q1, k1, v1 = synth.head_tensors(w, 1)
    assert np.array_equal(Q[0, 1], q1) and np.array_equal(K[0, 1], k1)
    Q2, _, _ = synth.layer_tensors(w)
    assert np.array_equal(Q, Q2)
    assert not np.array_equal(Q[0, 0], Q[0, 1])


def test_q_and_k_share_cluster_structure():
    w = synth.workload("tiny")
    q, k, v = synth.head_tensors(w, 0)
    f = lambda u: (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    q, k, v = f(q), f(k), f(v)
    # Q_n - K_n is only the two noise terms: var 2 * 0.3^2 per element
    assert abs((q - k).var() - 2 * 0.09) < 0.01
    assert abs(v.var() - 1.0) < 0.02
    # a query is much closer to its own key than to a random key
    own = np.einsum("nd,nd->n", q, k).mean()
    other = np.einsum("nd,nd->n", q, np.roll(k, 7, axis=0)).mean()
    assert own > other + 1.0


def test_position_embedding_layout():
    w = synth.workload("tiny")           # d = 64 -> chunks 24 / 20 / 20
    pe = di.position_embedding(w)
    assert pe.shape == (1024, 64)
    # token 0 is (t,y,x)=(0,0,0): sin terms 0, cos terms 1 in every chunk
    want = np.concatenate([np.r_[np.zeros(12), np.ones(12)],
                           np.r_[np.zeros(10), np.ones(10)],
                           np.r_[np.zeros(10), np.ones(10)]])
    np.testing.assert_allclose(pe[0], want, atol=1e-7)
    # token 1 is x = 1: only the x chunk changes
    assert np.allclose(pe[1, :44], pe[0, :44])
    np.testing.assert_allclose(pe[1, 44], np.sin(1.0), atol=1e-6)


def test_drift_magnitude():
    w = synth.workload("tiny")
    q1, _, _ = synth.head_tensors(w, 0, step=1)
    q2, _, _ = synth.head_tensors(w, 0, step=2)
    f = lambda u: (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    dq = f(q2) - f(q1)
    assert abs(dq.std() - w.drift) < 0.01


def test_random_metadata_valid():
    w = synth.workload("tiny")
    perm, kv, r = synth.random_metadata_head(w, 0)
    assert sorted(perm) == list(range(w.N))
    assert kv.shape == (w.n_groups, w.k)
    assert np.all(np.diff(kv, axis=1) > 0) and kv.min() >= 0 and kv.max() < w.N
    assert r.shape == (w.N, w.d) and r.dtype == np.float32


def test_workloads_by_name_and_id_agree():
    for wid, w in synth.WORKLOADS.items():
        assert synth.workload(w.name) == w == synth.workload(wid)
    assert synth.workload("video_long", k=100, G=64).k == 100
