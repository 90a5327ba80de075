"""Controlled comparisons of the three failure modes MC-Sparse closes.

The aiqbench.com abstract ("MC-Sparse: Deconstructing and Closing the
Dense-Sparse Attention Gap in Diffusion Transformers") attributes the gap to
constraints imposed by token grouping, inaccurate interaction selection, and
the attention contributions lost; the cnshai.top post (section "MC-Sparse:
three failure modes, one fix") pairs each with the choice that fixes it.
This module takes one choice away at a time on the same layer and reports
the fidelity to dense attention:

* ``token``      MC-Sparse's own selection: individual keys by exact summed
                 probability (with and without the cached residual);
* ``blockB``     block-granular selection (aligned blocks of B keys scored by
                 summed exact probability), at ``k // B`` blocks;
* ``token@kB``   token selection with the block variant's key budget, so the
                 two differ only in granularity;
* ``pooled``     a heuristic score: the probability the group's mean query
                 gives each key, instead of the exact summed probabilities;
* the residual's own effect is every variant with and without its residual.

(The ungrouped per-query selection -- the grouping constraint removed -- has
no group of 64 or 128 rows to run on the library's tiles; it is computed by
the fp64 oracle on sampled queries, in ``bench.py --ablate``.)

Every selection, residual and reused step runs in the CUDA library; this
module sequences the calls and reduces the outputs for the report (host
fp64 arithmetic on copies, as in ``fidelity``).
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import torch

from . import api
from .denoise import fidelity


def retained_mass(colsum: torch.Tensor, kv_idx: torch.Tensor, G: int, N: int) -> torch.Tensor:
    """alpha_g per group [B, H, n_groups]: the share of the group's dense
    attention mass its kept keys hold, sum_{j in S_g} colsum[g, j] / |g|."""
    ng = colsum.shape[2]
    sizes = torch.full((ng,), float(G), device=colsum.device)
    sizes[-1] = float(N - (ng - 1) * G)
    kept = torch.gather(colsum, 3, kv_idx.long()).sum(dim=3)
    return kept / sizes


class Ablation:
    """The variants' metadata, planned once on one step's Q, K, V."""

    def __init__(self, Q, K, V, G: int, k: int, blocks: Iterable[int] = (64, 128),
                 scale: Optional[float] = None, pooled: bool = True):
        B, H, N, d = Q.shape
        self.G, self.k, self.N, self.scale = G, min(int(k), N), N, scale
        self.ws = api.alloc_workspace(B, H, N, d, G, k, Q.device)
        meta = api.plan(Q, K, V, G, k, scale, workspace=self.ws)
        colsum = api.workspace_views(self.ws, B, H, N, d, G, k)["colsum"]
        perm = meta.perm
        selections = {"token": meta.kv_idx}
        for b in blocks:
            kb = self.k // b
            if kb < 1 or N // b < kb:
                continue
            selections[f"block{b}"] = api.select_blocks(colsum, kb, b)
            selections[f"token@k{b}"] = api.select_topk(colsum, kb * b)
        if pooled:
            selections["pooled"] = api.select_topk(api.pooled_scores(Q, K, perm, G, scale), self.k)
        self.metas: Dict[str, api.Meta] = {"token": meta}
        self.alpha: Dict[str, float] = {}
        for name, kv in selections.items():
            self.alpha[name] = float(retained_mass(colsum, kv, G, N).mean())
            if name == "token":
                continue
            res = api.plan_residual(Q, K, V, perm, kv, G, scale, workspace=self.ws, stats_done=True)
            self.metas[name] = api.Meta.from_tensors(perm, kv, res, G)

    def step(self, Q, K, V, O_dense: torch.Tensor) -> Dict[str, Dict[str, float]]:
        """Each variant's reused step on this step's Q, K, V: rel-L2 to the
        dense output of the same inputs, with and without its residual."""
        out = {}
        for name, meta in self.metas.items():
            O = api.sparse_step(Q, K, V, meta, self.scale)
            rel, rel_nr = fidelity(O, O_dense, meta.residual)
            out[name] = {"rel_l2": rel, "rel_l2_without_residual": rel_nr, "keys": int(meta.k),
                         "alpha_mean": self.alpha[name]}
        return out
