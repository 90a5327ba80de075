"""MC-Sparse over a diffusion sampler's denoising loop.

The metadata -- query groups, KV indices and the residual between dense and
sparse attention -- are computed on plan steps and reused on the steps in
between (aiqbench.com, "MC-Sparse: Deconstructing and Closing the
Dense-Sparse Attention Gap in Diffusion Transformers", abstract; cnshai.top
post, section "MC-Sparse: three failure modes, one fix").  A plan step
outputs the dense attention of its own inputs (the plan computes it anyway);
a reused step outputs the sparse attention over the cached groups and
indices plus the cached residual.  All attention work runs in the CUDA
library; this module only sequences the calls and keeps the buffers.

``fidelity`` measures a step's output against dense attention of the same
inputs, with and without the residual, for reports (host fp64 arithmetic on
copies; not part of the attention path).
"""
from __future__ import annotations

from typing import Iterable, Optional, Tuple

import numpy as np
import torch

from . import api


class Schedule:
    """Plan on the steps in ``plan_steps`` (1-based; the first step always
    plans, as nothing is cached before it), reuse the metadata elsewhere.

    The plan workspace, the metadata and the output buffer are allocated on
    the first step and reused for every later step of the same shape.
    """

    def __init__(self, G: int, k: int, plan_steps: Iterable[int], scale: Optional[float] = None):
        self.G, self.k, self.scale = int(G), int(k), scale
        self.plan_steps = frozenset(int(t) for t in plan_steps)
        self.meta: Optional[api.Meta] = None
        self._planned = False                 # does self.meta hold a plan?
        self._ws: Optional[torch.Tensor] = None
        self._out: Optional[torch.Tensor] = None
        self._shape = None

    def is_plan_step(self, t: int) -> bool:
        return not self._planned or t in self.plan_steps

    def reset(self) -> None:
        """Forget the cached metadata (buffers stay): the next step plans."""
        self._planned = False

    def step(self, t: int, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor) -> Tuple[torch.Tensor, str]:
        """Denoising step t on this step's Q, K, V: (O bf16 [B, H, N, d], "plan" | "reused").
        The returned tensor is this schedule's output buffer, overwritten by the next step."""
        if self._shape != tuple(Q.shape):
            B, H, N, d = Q.shape
            self._shape = tuple(Q.shape)
            self._ws = api.alloc_workspace(B, H, N, d, self.G, self.k, Q.device)
            self.meta = api.Meta.empty(B, H, N, d, self.G, self.k, Q.device)
            self._out = torch.empty_like(Q)
            self._planned = False
        if self.is_plan_step(t):
            api.plan(Q, K, V, self.G, self.k, self.scale, workspace=self._ws, meta=self.meta,
                     out_dense=self._out)
            self._planned = True
            return self._out, "plan"
        api.sparse_step(Q, K, V, self.meta, self.scale, out=self._out)
        return self._out, "reused"


def fidelity(O: torch.Tensor, O_dense: torch.Tensor, residual: torch.Tensor) -> Tuple[float, float]:
    """(||O - D|| / ||D||, ||(O - R) - D|| / ||D||) over the whole tensor, D the
    dense output of the same inputs and R the residual the output carries."""
    num = num_nr = den = 0.0
    for b in range(O.shape[0]):
        for h in range(O.shape[1]):
            o = O[b, h].float().cpu().numpy().astype(np.float64)
            dref = O_dense[b, h].float().cpu().numpy().astype(np.float64)
            r = residual[b, h].cpu().numpy().astype(np.float64)
            num += float(np.sum((o - dref) ** 2))
            num_nr += float(np.sum((o - r - dref) ** 2))
            den += float(np.sum(dref ** 2))
    den = max(den, 1e-300)
    return float(np.sqrt(num / den)), float(np.sqrt(num_nr / den))
