"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a closed form, brute force, an invariant
the method's definitions fix, or an independent textbook routine, chosen so a
plausible slip (dropped centring, wrong sign convention, transposed operand,
missing renormalisation, wrong tie rule, off-by-one group) fails at least one.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import mcs_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(n, d, seed, scale=1.0):
    return scale * np.random.default_rng(seed).standard_normal((n, d))


# --- dense attention ---------------------------------------------------------

@pytest.mark.parametrize("n,d", [(1, 3), (5, 4), (17, 8), (32, 5)])
def test_dense_matches_naive_loops(n, d):
    Q, K, V = _rand(n, d, 1), _rand(n, d, 2), _rand(n, d, 3)
    scale = 0.37
    got = orc.dense_attention(Q, K, V, scale)
    for i in range(n):
        s = [scale * sum(Q[i, c] * K[j, c] for c in range(d)) for j in range(n)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        z = sum(e)
        for c in range(d):
            want = sum(e[j] * V[j, c] for j in range(n)) / z
            assert abs(got[i, c] - want) < 1e-12


@pytest.mark.parametrize("n,m,d", [(64, 64, 16), (100, 37, 64), (130, 130, 128)])
def test_dense_matches_torch_sdpa_f64(n, m, d):
    Q, K, V = _rand(n, d, 4), _rand(m, d, 5), _rand(m, d, 6)
    scale = 1.0 / math.sqrt(d)
    got = orc.dense_attention(Q, K, V, scale, block=17)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        scale=scale)[0].numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_probability_rows_sum_to_one_and_stats():
    Q, K = _rand(40, 8, 7, 3.0), _rand(300, 8, 8, 3.0)
    P = orc.probabilities(Q, K, 0.5)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    m, l = orc.row_stats(Q, K, 0.5)
    S = 0.5 * Q @ K.T
    np.testing.assert_allclose(np.exp(S - m[:, None]) / l[:, None], P, rtol=1e-12, atol=1e-15)
    assert np.all(np.isclose(m, S.max(axis=1)))


# --- grouping -----------------------------------------------------------------

def test_principal_direction_rank_one_closed_form_needs_centring():
    rng = np.random.default_rng(11)
    d, n = 6, 50
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    i = int(np.argmax(np.abs(u)))
    if u[i] < 0:
        u = -u                       # largest component positive: v must equal u
    mu = 5.0 * rng.standard_normal(d)   # large offset, not parallel to u
    t = rng.standard_normal(n)
    Q = mu[None, :] + t[:, None] * u[None, :]
    mu_o, C, v, lam = orc.principal_direction(Q)
    np.testing.assert_allclose(mu_o, mu + t.mean() * u, atol=1e-12)
    np.testing.assert_allclose(v, u, atol=1e-10)
    np.testing.assert_allclose(lam[-1], t.var(), rtol=1e-10)
    # the projection order is the order of t
    assert np.array_equal(orc.group_queries(Q), np.argsort(t, kind="stable"))
    # flipping the data direction flips nothing in v (sign rule), and reverses the order
    Q2 = mu[None, :] - t[:, None] * u[None, :]
    assert np.array_equal(orc.group_queries(Q2), np.argsort(-t, kind="stable"))


def test_sign_rule_uses_largest_magnitude_component():
    # direction (0.6, -0.8): largest magnitude component is negative -> v = (-0.6, 0.8)
    t = np.linspace(-1.0, 1.0, 9)
    Q = t[:, None] * np.array([0.6, -0.8])[None, :]
    _, _, v, _ = orc.principal_direction(Q)
    np.testing.assert_allclose(v, [-0.6, 0.8], atol=1e-12)
    # projections increase with -t, so the first query in order is the last t
    assert orc.group_queries(Q)[0] == 8


def test_principal_direction_vs_independent_power_iteration():
    rng = np.random.default_rng(3)
    A = rng.standard_normal((8, 8))
    Q = rng.standard_normal((500, 8)) @ A
    mu, C, v, lam = orc.principal_direction(Q)
    X = Q - Q.mean(axis=0)
    M = sum(np.outer(x, x) for x in X) / len(X)      # covariance by explicit sum
    w = np.ones(8)
    for _ in range(5000):
        w = M @ w
        w /= np.linalg.norm(w)
    assert min(np.linalg.norm(w - v), np.linalg.norm(w + v)) < 1e-8
    np.testing.assert_allclose(M @ v, lam[-1] * v, atol=1e-9)
    for _ in range(50):
        z = rng.standard_normal(8)
        assert z @ M @ z / (z @ z) <= lam[-1] * (1 + 1e-12)


def test_group_queries_ties_keep_index_order():
    base = np.array([[1.0, 0.0], [2.0, 0.0], [3.0, 0.0]])
    Q = np.concatenate([base, base, base])           # rows 0,3,6 tie, etc.
    perm = orc.group_queries(Q)
    assert list(perm) == [0, 3, 6, 1, 4, 7, 2, 5, 8]


@pytest.mark.parametrize("N,d", [(9000, 128), (5000, 64)])
def test_group_queries_equal_rows_keep_index_order_at_size(N, d):
    """Equal query rows have equal projections, so the stable sort keeps each
    set of equal rows in token order, wherever the rows lie in the array (a
    blocked or threaded matrix-vector product can round equal rows apart)."""
    rng = np.random.default_rng(N + d)
    Q = rng.standard_normal((N, d))
    src = rng.integers(0, N, size=N // 3)
    dst = rng.integers(0, N, size=N // 3)
    Q[dst] = Q[src]
    perm = orc.group_queries(Q)
    where = np.empty(N, np.int64)
    where[perm] = np.arange(N)
    _, inv = np.unique(Q, axis=0, return_inverse=True)
    inv = inv.ravel()
    order = np.lexsort((np.arange(N), inv))           # tokens by set, ascending inside each set
    same_set = inv[order][1:] == inv[order][:-1]
    assert same_set.sum() > N // 5                    # many sets of equal rows
    a, b = order[:-1][same_set], order[1:][same_set]
    assert np.all(where[a] < where[b])                # lower token first ...
    assert np.all(where[b] - where[a] == 1)           # ... and adjacent: nothing sorts between equal rows


def test_groups_partition_with_partial_tail():
    perm = np.arange(10)[::-1]
    groups = [orc.group_rows(perm, 4, g) for g in range(3)]
    assert [len(g) for g in groups] == [4, 4, 2]
    assert sorted(np.concatenate(groups)) == list(range(10))


# --- selection ----------------------------------------------------------------

def test_select_kv_brute_force_with_ties():
    rng = np.random.default_rng(5)
    for trial in range(200):
        n = int(rng.integers(1, 13))
        k = int(rng.integers(1, 6))
        c = rng.integers(0, 4, size=n).astype(float)   # many exact ties
        kk = min(k, n)
        best = None
        for sub in itertools.combinations(range(n), kk):
            key = (sum(c[list(sub)]), -sum(sub))
            if best is None or key > best[0]:
                best = (key, sub)
        assert list(orc.select_kv(c, k)) == list(best[1]), (c, k)


def test_selection_maximises_group_retained_mass():
    rng = np.random.default_rng(9)
    for trial in range(20):
        n, d, G, k = 12, 4, 3, 3
        Q, K = rng.standard_normal((n, d)) * 2, rng.standard_normal((n, d)) * 2
        perm = orc.group_queries(Q)
        c = orc.group_prob_sums(Q, K, 0.7, perm, G)
        for g in range(4):
            rows = orc.group_rows(perm, G, g)
            P = orc.probabilities(Q[rows], K, 0.7)
            best = max(P[:, list(s)].sum() for s in itertools.combinations(range(n), k))
            got = P[:, orc.select_kv(c[g], k)].sum()
            assert got >= best - 1e-12


def test_group_sums_total_equals_group_size():
    Q, K = _rand(70, 8, 12), _rand(90, 8, 13)
    perm = orc.group_queries(Q)
    c = orc.group_prob_sums(Q, K, 0.4, perm, 16)
    np.testing.assert_allclose(c.sum(axis=1), [16, 16, 16, 16, 6], atol=1e-12)


def test_k_larger_than_n_is_clamped():
    assert list(orc.select_kv(np.array([0.1, 0.5, 0.2]), 10)) == [0, 1, 2]


# --- sparse output and residual ------------------------------------------------

def test_sparse_group_matches_masked_sdpa():
    Q, K, V = _rand(9, 16, 21), _rand(50, 16, 22), _rand(50, 16, 23)
    idx = np.array([1, 4, 5, 17, 30, 49])
    got = orc.sparse_group(Q, K, V, 0.25, idx)
    mask = torch.full((9, 50), float("-inf"), dtype=torch.float64)
    mask[:, idx] = 0.0
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        attn_mask=mask[None], scale=0.25)[0].numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_k_equals_n_gives_zero_residual():
    Q, K, V = _rand(48, 8, 31), _rand(48, 8, 32), _rand(48, 8, 33)
    meta = orc.plan_head(Q, K, V, G=16, k=48, scale=0.3)
    assert np.abs(meta["residual"]).max() < 1e-13
    O_sp = orc.sparse_attention(Q, K, V, 0.3, meta["perm"], meta["kv_idx"], 16)
    np.testing.assert_allclose(O_sp, orc.dense_attention(Q, K, V, 0.3), atol=1e-13)


def test_reused_step_on_unchanged_inputs_reproduces_dense():
    Q, K, V = _rand(100, 8, 41, 2.0), _rand(100, 8, 42, 2.0), _rand(100, 8, 43)
    meta = orc.plan_head(Q, K, V, G=16, k=10, scale=0.35)
    O = orc.reused_step_head(Q, K, V, 0.35, meta["perm"], meta["kv_idx"], meta["residual"], 16)
    dense = orc.dense_attention(Q, K, V, 0.35)
    np.testing.assert_allclose(O, dense, rtol=0, atol=1e-12)
    np.testing.assert_allclose(meta["O_dense"], dense, rtol=0, atol=1e-12)
    # with sparse selection the residual is not trivially zero
    assert np.abs(meta["residual"]).max() > 1e-3


def test_residual_two_formulas_agree():
    Q, K, V = _rand(20, 8, 51, 2.0), _rand(200, 8, 52, 2.0), _rand(200, 8, 53)
    idx = np.sort(np.random.default_rng(0).choice(200, 30, replace=False))
    R, R_alt, alpha = orc.residual_group(Q, K, V, 0.4, idx)
    np.testing.assert_allclose(R, R_alt, rtol=1e-12, atol=1e-14)
    assert np.all((alpha > 0) & (alpha < 1))


def test_constant_values_give_zero_residual():
    Q, K = _rand(30, 8, 61), _rand(30, 8, 62)
    V = np.tile(np.array([[0.5, -2.0, 3.0]]), (30, 1))
    meta = orc.plan_head(Q, K, V, G=8, k=3, scale=0.5)
    assert np.abs(meta["residual"]).max() < 1e-13


def test_single_query_groups_single_key_is_argmax():
    Q, K, V = _rand(25, 6, 71, 2.0), _rand(25, 6, 72, 2.0), _rand(25, 6, 73)
    meta = orc.plan_head(Q, K, V, G=1, k=1, scale=0.5)
    perm = meta["perm"]
    S = Q @ K.T
    O_sp = orc.sparse_attention(Q, K, V, 0.5, perm, meta["kv_idx"], 1)
    for i in range(25):
        np.testing.assert_allclose(O_sp[i], V[int(np.argmax(S[i]))], atol=1e-14)


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_example.json")))
    a = np.array(g["a"], dtype=float)
    n = len(a)
    Q = np.tile([[1.0, 0.0]], (n, 1))
    K = np.stack([np.log(a), np.zeros(n)], axis=1)
    V = np.array(g["V"], dtype=float)
    ex = {k: v for k, v in g["expected"].items()}
    f = lambda s: float(Fraction(s))
    P = orc.probabilities(Q, K, g["scale"])
    np.testing.assert_allclose(P[0], [f(x) for x in ex["P_row"]], atol=1e-15)
    meta = orc.plan_head(Q, K, V, g["G"], g["k"], g["scale"])
    c = orc.group_prob_sums(Q, K, g["scale"], meta["perm"], g["G"])
    np.testing.assert_allclose(c[0], [f(x) for x in ex["group_score"]], atol=1e-14)
    assert list(meta["kv_idx"][0]) == ex["kv_idx"]
    np.testing.assert_allclose(meta["O_dense"][0], [f(x) for x in ex["O_dense"]], atol=1e-15)
    np.testing.assert_allclose(meta["residual"], np.tile([f(x) for x in ex["residual"]], (n, 1)),
                               atol=1e-15)
    R, R_alt, alpha = orc.residual_group(Q, K, V, g["scale"], ex["kv_idx"])
    np.testing.assert_allclose(alpha, f(ex["alpha"]), atol=1e-15)
    np.testing.assert_allclose(R_alt, R, atol=1e-15)
    O_sp = orc.sparse_group(Q, K, V, g["scale"], ex["kv_idx"])
    np.testing.assert_allclose(O_sp[0], [f(x) for x in ex["O_sparse"]], atol=1e-15)


def test_page_speedup_context_numbers_are_consistent():
    g = json.load(open(os.path.join(GOLDEN, "page_speedups.json")))
    v = g["video_dit_minimax_h3_base_speedup"]
    a = g["asset3d_generation_speedup"]
    assert abs((1 - 1 / v) - g["derived_claims"]["video_step_time_reduction_about"]) < 0.01
    assert 1 - 1 / a > g["derived_claims"]["asset3d_step_time_reduction_more_than"]


def test_widen_bf16_exact():
    u = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x7F7F], dtype=np.uint16)
    w = orc.widen_bf16(u)
    assert w[0] == 1.0 and w[1] == -1.0 and w[3] == 0.0
    assert w[2] == 3.140625
    assert w[4] == float(np.float32(3.3895313892515355e38))


# --- denoising schedule ----------------------------------------------------------

def _drifted(n, d, steps, seed, sigma):
    """(Q, K, V) per step: a random walk of the step-1 tensors."""
    rng = np.random.default_rng(seed)
    cur = [_rand(n, d, seed + 1, 2.0), _rand(n, d, seed + 2, 2.0), _rand(n, d, seed + 3)]
    out = [tuple(cur)]
    for _ in range(steps - 1):
        cur = [x + sigma * rng.standard_normal(x.shape) for x in cur]
        out.append(tuple(cur))
    return out


def test_rel_l2_closed_forms():
    ref = np.array([[3.0, 4.0]])
    assert orc.rel_l2(ref, ref) == 0.0
    assert orc.rel_l2(2 * ref, ref) == pytest.approx(1.0, abs=1e-15)
    assert orc.rel_l2(ref + np.array([[0.0, 0.5]]), ref) == pytest.approx(0.1, abs=1e-15)


def test_schedule_on_unchanged_inputs_is_dense_at_every_step():
    st = _drifted(80, 8, 4, 100, 0.0)
    r = orc.schedule_head(st, [1], G=16, k=8, scale=0.35)
    assert [x["kind"] for x in r] == ["plan", "reused", "reused", "reused"]
    dense = orc.dense_attention(*st[0], 0.35)
    for x in r:
        assert x["rel_l2"] < 1e-12
        np.testing.assert_allclose(x["O"], dense, rtol=0, atol=1e-12)
    # the same cached metadata on the same inputs: the sparse-only error is the same each step
    assert r[0]["rel_l2_no_residual"] > 1e-3
    for x in r[1:]:
        assert x["rel_l2_no_residual"] == pytest.approx(r[0]["rel_l2_no_residual"], rel=1e-12)


def test_schedule_with_k_equal_n_is_dense_with_or_without_residual():
    st = _drifted(64, 8, 3, 200, 0.1)
    for x in orc.schedule_head(st, [1], G=16, k=64, scale=0.35):
        assert x["rel_l2"] < 1e-12 and x["rel_l2_no_residual"] < 1e-12


def test_schedule_plan_steps_output_dense_of_their_own_inputs():
    st = _drifted(64, 8, 4, 300, 0.2)
    r = orc.schedule_head(st, [1, 3], G=16, k=6, scale=0.35)
    assert [x["kind"] for x in r] == ["plan", "reused", "plan", "reused"]
    for t in (0, 2):
        np.testing.assert_allclose(r[t]["O"], orc.dense_attention(*st[t], 0.35), rtol=0, atol=1e-12)
        assert r[t]["rel_l2"] < 1e-12
    # drift moves the reused steps away from dense; the residual still helps
    for t in (1, 3):
        assert r[t]["rel_l2"] > 1e-6
        assert r[t]["rel_l2"] < r[t]["rel_l2_no_residual"]


def test_schedule_constant_values_exact_under_drift():
    st = _drifted(48, 6, 3, 400, 0.3)
    c = np.array([[1.5, -0.25, 2.0, 0.0, -1.0, 3.0]])
    st = [(q, k, np.tile(c, (48, 1))) for q, k, _ in st]
    for x in orc.schedule_head(st, [1], G=8, k=4, scale=0.4):
        assert x["rel_l2"] < 1e-13 and x["rel_l2_no_residual"] < 1e-13


# --- ablations of the three failure modes -------------------------------------

def test_select_blocks_of_one_key_is_token_selection():
    c = np.random.default_rng(40).random(37)
    for k in (1, 5, 37):
        assert np.array_equal(orc.select_blocks(c, k, 1), orc.select_kv(c, k))


def test_select_blocks_brute_force_and_ragged_tail():
    rng = np.random.default_rng(41)
    block, n = 4, 22                       # 5 full blocks, a ragged tail of 2 keys
    for trial in range(20):
        c = rng.integers(0, 3, size=n).astype(np.float64)    # many exact ties
        c[20:] = 100.0                                       # the tail is never a candidate
        for kb in (1, 2, 3, 5, 9):
            got = orc.select_blocks(c, kb, block)
            kk = min(kb, n // block)
            sums = [c[b * block:(b + 1) * block].sum() for b in range(n // block)]
            best = max(sum(sums[b] for b in comb) for comb in itertools.combinations(range(n // block), kk))
            chosen = sorted(set((got // block).tolist()))
            assert len(got) == kk * block and np.all(np.diff(got) > 0)
            assert sum(sums[b] for b in chosen) == best
            # among subsets of equal total the lowest block indices win
            first = min(itertools.combinations(range(n // block), kk),
                        key=lambda comb: (-sum(sums[b] for b in comb), comb))
            assert chosen == list(first)
            assert np.all(got < 20)


def test_pooled_score_of_single_query_groups_is_its_probability_row():
    Q, K = _rand(9, 4, 42), _rand(13, 4, 43)
    perm = np.arange(9)
    got = orc.pooled_scores(Q, K, 0.5, perm, 1)
    assert np.allclose(got, orc.probabilities(Q, K, 0.5), rtol=0, atol=1e-15)
    assert np.allclose(got.sum(axis=1), 1.0)


def test_pooled_score_uses_the_mean_query():
    Q, K = _rand(8, 5, 44), _rand(11, 5, 45)
    perm = np.array([3, 1, 7, 0, 2, 6, 5, 4])
    got = orc.pooled_scores(Q, K, 0.3, perm, 4)
    for g in range(2):
        qbar = Q[perm[4 * g:4 * g + 4]].sum(axis=0) / 4
        s = [0.3 * float(qbar @ K[j]) for j in range(11)]
        e = np.exp(np.array(s) - max(s))
        assert np.allclose(got[g], e / e.sum(), rtol=1e-13)


def test_ungrouped_rows_closed_forms():
    Q, K, V = _rand(6, 4, 46, 2.0), _rand(10, 4, 47), _rand(10, 3, 48)
    assert np.allclose(orc.ungrouped_rows(Q, K, V, 0.5, 10), orc.dense_rows(Q, K, V, 0.5), atol=1e-14)
    top1 = orc.ungrouped_rows(Q, K, V, 0.5, 1)
    P = orc.probabilities(Q, K, 0.5)
    assert np.allclose(top1, V[np.argmax(P, axis=1)], atol=0)


def test_retained_mass_closed_forms():
    Q, K = _rand(5, 4, 49), _rand(12, 4, 50)
    c = orc.probabilities(Q, K, 0.7).sum(axis=0)
    assert abs(orc.retained_mass(c, np.arange(12), 5) - 1.0) < 1e-14
    idx = orc.select_kv(c, 4)
    other = np.setdiff1d(np.arange(12), idx)
    assert abs(orc.retained_mass(c, idx, 5) + orc.retained_mass(c, other, 5) - 1.0) < 1e-14


# --------------------------------------------------------------------------- compact residual storage

def _all_finite_bf16():
    u = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        v = orc.widen_bf16(u)
    keep = np.isfinite(v)
    return u[keep], v[keep]


def test_round_bf16_is_the_nearest_bf16_value_by_exhaustive_search():
    """Every sample against all 65280 finite bf16 values: the result is at
    minimal distance; among two at equal distance, the even-mantissa one."""
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2 ** 32, size=1500, dtype=np.uint64).astype(np.uint32)
    ties = (bits[:500] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)     # exactly half-way cases
    x = np.concatenate([bits, ties]).view(np.float32)
    x = x[np.isfinite(x)]
    x = x[np.abs(x.astype(np.float64)) < 3.38e38]
    got = orc.round_bf16(x)
    u_all, v_all = _all_finite_bf16()
    for chunk in np.array_split(np.arange(len(x)), 20):
        xs = x[chunk].astype(np.float64)
        dist = np.abs(xs[:, None] - v_all[None, :])
        best = dist.min(axis=1)
        g = orc.widen_bf16(got[chunk])
        assert np.array_equal(np.abs(xs - g), best)
        for i, row in zip(chunk, dist):
            cands = u_all[row == row.min()]
            cands = cands[~((cands == 0x8000) & (x[i] >= 0)) & ~((cands == 0) & (x[i] < 0))]  # signed zero of x
            if len(cands) > 1:          # a tie: the even mantissa wins
                even = cands[(cands & 1) == 0]
                assert got[i] in even, (x[i], cands, got[i])


def test_round_bf16_keeps_bf16_values_and_special_values():
    u_all, v_all = _all_finite_bf16()
    assert np.array_equal(orc.round_bf16(v_all.astype(np.float32)), u_all)      # every bf16 value is kept
    assert orc.round_bf16(np.float32(np.inf))[()] == 0x7F80
    assert orc.round_bf16(np.float32(-np.inf))[()] == 0xFF80
    assert np.isnan(orc.widen_bf16(orc.round_bf16(np.float32(np.nan))))
    top = orc.widen_bf16(np.uint16(0x7F7F))                 # largest finite bf16, odd mantissa
    half_ulp = 2.0 ** (127 - 8)
    assert orc.round_bf16(np.float32(top + half_ulp))[()] == 0x7F80               # the tie goes to even: infinity
    assert orc.round_bf16(np.nextafter(np.float32(top + half_ulp), np.float32(0)))[()] == 0x7F7F
    assert orc.round_bf16(np.float32(1.0 + 2.0 ** -8))[()] == 0x3F80               # tie between 1 and 1 + 2^-7
    assert orc.round_bf16(np.float32(1.0 + 3 * 2.0 ** -8))[()] == 0x3F82           # tie: 1 + 2^-6 is even
    assert orc.round_bf16(np.float32(-(1.0 + 2.0 ** -8)))[()] == 0xBF80
