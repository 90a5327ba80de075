"""Helpers shared by the GPU parity tests: device upload of bf16 bit patterns
and the comparisons the tolerances are stated for."""
import numpy as np
import torch

# Tolerances (bf16 outputs; fp32 residual), stated once.
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 1e-2
RES_REL_L2 = 1e-3
KV_THRESHOLD_REL = 1e-4
# Plan statistics (a2) and group scores (a3), read from the plan workspace.
# s_ij comes out of fp32 tensor-core accumulation of exact bf16 products, and
# l_i is an fp32 sum of N terms; rounding in both behaves like sqrt(N) * 2^-24
# (about 1e-5 for N up to 131072), so the row's log normaliser m + log l
# (natural units) is held to 2e-4 absolute.  Each group score is a sum of G
# probabilities each carrying that relative error plus ex2.approx's 2^-22, so
# it is held to 1e-4 relative -- the same margin the KV-set rule grants at
# the k-th score -- plus an absolute floor for terms below fp32's smallest
# normal value, which the kernels flush to zero (at most G * 2^-126 per score).
LSE_ABS = 2e-4
COLSUM_REL = 1e-4
COLSUM_ABS = 128 * 2.0 ** -126


def dev_bf16(u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_out_close(got: np.ndarray, ref: np.ndarray, what: str):
    err = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert err <= OUT_MAX_ABS and rel <= OUT_REL_L2, f"{what}: max-abs {err:.3e} rel-L2 {rel:.3e}"
    return err, rel


def assert_residual_close(got: np.ndarray, ref: np.ndarray, what: str):
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert rel <= RES_REL_L2, f"{what}: residual rel-L2 {rel:.3e}"
    return rel


def kv_sets_agree(got_idx: np.ndarray, score_row: np.ndarray, k: int, G: int = 0) -> int:
    """GPU kv set vs the oracle score row: the sets may differ only in keys
    whose score lies within KV_THRESHOLD_REL of the k-th largest score.
    With G (the group size) given, scores at or below G * FLT_MIN -- sums of
    G probabilities each below fp32's smallest normal value, which the
    kernel's fp32 arithmetic flushes to zero -- count as ties at zero: the
    sets may differ in such keys when the k-th score is itself that small.
    Also checks the GPU list is strictly ascending.  Returns #differences."""
    got_idx = np.asarray(got_idx)
    assert np.all(np.diff(got_idx) > 0), "kv indices not strictly ascending"
    n = score_row.shape[0]
    kk = min(k, n)
    order = np.lexsort((np.arange(n), -score_row))
    ref = set(order[:kk].tolist())
    thr = score_row[order[kk - 1]]
    floor = G * float(np.finfo(np.float32).tiny)
    diff = ref.symmetric_difference(set(got_idx.tolist()))
    for j in diff:
        if thr <= floor and score_row[j] <= floor:
            continue
        assert abs(score_row[j] - thr) <= KV_THRESHOLD_REL * abs(thr), (
            f"key {j}: score {score_row[j]:.6e} vs k-th {thr:.6e}")
    return len(diff)
