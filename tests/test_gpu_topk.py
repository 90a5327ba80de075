"""GPU parity of the top-k selection (step a4) on score rows built to reach
every branch of the kernel, checked index for index against the oracle's
select_kv (ties to the lower key index, output ascending):

  * rows whose scores take only a few distinct values (ties across the
    threshold, equal keys spread over many warps' slices);
  * constant rows and all-zero rows (the candidate list overflows and the
    remaining digits are resolved over the whole row);
  * lengths not a multiple of 4 (scalar loads), rows that fit in shared
    memory and rows that do not (re-read from L2), a ragged last warp slice;
  * k = 1, k = N - 1 and k >= N.
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
    ("lognormal", 6, 32760, 1638),      # the long-video row length, cached in shared memory
    ("lognormal", 3, 65536, 1966),      # too long to cache
    ("lognormal", 4, 4099, 123),        # N % 4 != 0: scalar loads, ragged slices
    ("lognormal", 4, 40960, 2048),      # the longest cached row
    ("lognormal", 2, 40964, 2048),      # one vector past it
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
