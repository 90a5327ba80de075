"""GPU parity of the top-k selection (step a4) on score rows built to reach
every branch of the kernel, checked index for index against the oracle's
select_kv (ties to the lower key index, output ascending):

  * rows whose scores take only a few distinct values (ties across the
    threshold, equal keys spread over many warps' slices);
  * constant rows and all-zero rows (the candidate list overflows and the
    remaining digits are resolved over the whole row);
  * lengths not a multiple of 4 (scalar loads), short and long rows, a
    ragged last warp slice;
  * k = 1, k = N - 1 and k >= N;
  * many rows at once, repeatedly, whose candidates all need the second and
    third digits (a clear of one digit's histogram racing the next digit's
    counts would lose counts in some row, some time);
  * long runs of rows per CTA, mixing rows alike their predecessor (the
    first walk's guess of the threshold's first digit holds), rows whose
    scale jumps by 2^10 either way (the guess misses: the keys are listed
    again, or the first list overflows), rows with ties at the threshold and
    constant rows;
  * rows longer than the output bitmap (N > 131072).
"""
import numpy as np
import pytest
import torch

import sparse_attention_diffusion_mcs_b200 as mcs
from oracle import mcs_oracle as orc

pytestmark = pytest.mark.gpu


def _rows(kind, rows, N, rng):
    if kind == "lognormal":
        return rng.lognormal(-9.0, 2.0, size=(rows, N)).astype(np.float32)
    if kind == "few_values":
        return rng.choice(np.array([0.0, 1e-6, 2.5e-3, 2.5e-3 * (1 + 2 ** -20), 0.125], np.float32),
                          size=(rows, N), p=[0.4, 0.3, 0.2, 0.05, 0.05])
    if kind == "constant":
        return np.full((rows, N), 3.0e-4, np.float32)
    if kind == "zeros":
        return np.zeros((rows, N), np.float32)
    if kind == "near_constant":
        # one first-digit bin holds every key; the rest differ in the low bits
        base = np.float32(1.0e-3).view(np.uint32)
        return (base + rng.integers(0, 1 << 14, size=(rows, N), dtype=np.uint32)).view(np.float32)
    raise ValueError(kind)


CASES = [
    ("lognormal", 6, 32760, 1638),      # the long-video row length
    ("lognormal", 3, 65536, 1966),      # too long to cache
    ("lognormal", 4, 4099, 123),        # N % 4 != 0: scalar loads, ragged slices
    ("lognormal", 4, 40960, 2048),
    ("lognormal", 2, 40964, 2048),
    ("few_values", 5, 15600, 1560),
    ("few_values", 3, 4097, 1000),
    ("constant", 3, 32760, 1638),
    ("zeros", 2, 15600, 7),
    ("near_constant", 3, 32760, 1638),
    ("near_constant", 2, 131072, 6553),
    ("lognormal", 3, 1000, 1),
    ("few_values", 3, 1000, 999),
    ("lognormal", 2, 37, 64),           # k >= N: every key
    ("lognormal", 2, 1, 1),
    ("lognormal", 3, 131076, 500),      # longer than the output bitmap
    ("lognormal", 2, 262144, 20000),
]


@pytest.mark.parametrize("kind,rows,N,k", CASES, ids=[f"{c[0]}-N{c[2]}-k{c[3]}" for c in CASES])
def test_select_topk_matches_oracle(kind, rows, N, k):
    rng = np.random.default_rng(N * 31 + k)
    s = _rows(kind, rows, N, rng)
    got = mcs.select_topk(torch.from_numpy(s).cuda(), k).cpu().numpy()
    assert got.shape == (rows, min(k, N))
    for r in range(rows):
        ref = orc.select_kv(s[r].astype(np.float64), k)
        assert np.array_equal(got[r], ref), f"{kind} row {r}: {np.sum(got[r] != ref)} indices differ"


def test_select_topk_many_rows_repeatably():
    rng = np.random.default_rng(77)
    rows, N, k = 2000, 6000, 3000
    s = _rows("near_constant", rows, N, rng)         # every key a candidate; passes 3 and 4 decide
    ref = np.stack([orc.select_kv(s[r].astype(np.float64), k) for r in range(rows)])
    dev = torch.from_numpy(s).cuda()
    for rep in range(5):
        got = mcs.select_topk(dev, k).cpu().numpy()
        bad = np.nonzero((got != ref).any(axis=1))[0]
        assert len(bad) == 0, f"repetition {rep}: {len(bad)} rows differ, first {bad[:5]}"


def _mixed_rows(rng, rows, N):
    s = rng.lognormal(-9.0, 2.0, size=(rows, N)).astype(np.float32)
    kind = rng.integers(0, 12, size=rows)
    for r in range(rows):
        if kind[r] == 0:
            s[r] *= np.float32(2.0 ** 10)
        elif kind[r] == 1:
            s[r] *= np.float32(2.0 ** -10)
        elif kind[r] == 2:
            s[r] = rng.choice(np.array([0.0, 1e-6, 2.5e-3, 0.125], np.float32), size=N, p=[0.4, 0.3, 0.25, 0.05])
        elif kind[r] == 3:
            s[r] = np.float32(3.0e-4)
    return s, kind


@pytest.mark.parametrize("rows,N,k", [(3000, 4096, 200), (1500, 32760, 1638), (700, 4099, 300)])
def test_select_topk_runs_of_mixed_rows(rows, N, k):
    """More rows than CTAs, so each CTA walks a run of rows and guesses each
    row's threshold digit from the row before; every row index-exact."""
    rng = np.random.default_rng(rows + N + k)
    s, kind = _mixed_rows(rng, rows, N)
    assert rows > 3 * 148 and len(set(kind.tolist())) == 12
    got = mcs.select_topk(torch.from_numpy(s).cuda(), k).cpu().numpy()
    bad = [r for r in range(rows) if not np.array_equal(got[r], orc.select_kv(s[r].astype(np.float64), k))]
    assert not bad, f"{len(bad)} rows differ, first {bad[:5]} (kinds {[int(kind[r]) for r in bad[:5]]})"


def test_select_topk_batched_shape_and_empty():
    s = torch.rand(2, 3, 5, 777, device="cuda")
    out = mcs.select_topk(s, 50)
    assert out.shape == (2, 3, 5, 50)
    host = s.cpu().numpy().reshape(-1, 777)
    o = out.cpu().numpy().reshape(-1, 50)
    for r in range(host.shape[0]):
        assert np.array_equal(o[r], orc.select_kv(host[r].astype(np.float64), 50))
    empty = mcs.select_topk(torch.empty(0, 100, device="cuda"), 10)
    assert empty.shape == (0, 10)


# ---------------------------------------------------------------------------
# The plan's selection on the group scores it has just made: exactly what the
# selection gives when called on those scores, including rows whose ties
# overflow the candidate list.

import synth  # noqa: E402
from tests.gpu_util import dev_bf16  # noqa: E402


def _plan_and_scores(Q, K, V, G, k):
    B, H, N, d = Q.shape
    q, kd, v = dev_bf16(Q), dev_bf16(K), dev_bf16(V)
    ws = mcs.alloc_workspace(B, H, N, d, G, k, q.device)
    meta = mcs.plan(q, kd, v, G, k, workspace=ws)
    colsum = mcs.workspace_views(ws, B, H, N, d, G, k)["colsum"]
    ref = mcs.select_topk(colsum, min(k, N))
    torch.cuda.synchronize()
    assert mcs.last_device_status() == 0
    return meta.kv_idx.cpu().numpy(), ref.cpu().numpy(), colsum.cpu().numpy()


@pytest.mark.parametrize("N,d,G,k", [(999, 64, 64, 100), (1024, 128, 128, 300), (2500, 128, 64, 1),
                                     (777, 64, 128, 777), (1300, 128, 128, 5000)])
def test_plan_selection_equals_select_topk_on_its_scores(N, d, G, k):
    Q, K, V = synth.random_qkv(1, 2, N, d, seed=21, q_std=2.0)
    got, ref, _ = _plan_and_scores(Q, K, V, G, k)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("N,d", [(1000, 128), (16384, 128), (13000, 64)])
def test_plan_selection_on_constant_rows(N, d):
    """K = 0 makes every score 0 and every group's probabilities uniform, so
    each group-score row is constant: the selection is keys 0 .. k-1 (ties to
    the lower index).  At N = 16384 and 13000 the whole row overflows the
    candidate list and the remaining digits are resolved over the row."""
    Q, _, V = synth.random_qkv(1, 1, N, d, seed=22)
    K = np.zeros_like(Q)
    k = 700
    got, ref, cs = _plan_and_scores(Q, K, V, 128, k)
    assert np.all(cs[0, 0] == cs[0, 0, :, :1])          # each group's row is constant
    assert np.array_equal(got, ref)
    assert np.array_equal(got[0, 0], np.broadcast_to(np.arange(k, dtype=np.int32), got[0, 0].shape))
