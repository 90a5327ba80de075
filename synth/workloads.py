"""The five synthetic DiT attention-layer workloads.

Shapes follow the video / 3D-asset DiT settings that the MC-Sparse pages
describe in words (long-sequence attention at every denoising step; video and
3D asset generation; aiqbench.com entry "MC-Sparse: Deconstructing and Closing
the Dense-Sparse Attention Gap in Diffusion Transformers", abstract).  The
concrete grids, head dims, group sizes, sparsities and drift schedules are the
benchmark workloads this library is measured on; the pages print none of them.

k is the number of KV tokens kept per query group.  A percentage p of N is
turned into k = floor(p * N) with integer arithmetic.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int
    B: int
    H: int
    grid: Tuple[int, int, int]          # (T, Y, X), raster order t-major
    d: int
    G: int
    k: int
    centroids: int
    noise: str                          # "gauss" or "student_t3"
    locality: bool                      # random-Fourier locality component
    steps: int
    drift: float
    plan_steps: Tuple[int, ...]         # 1-based denoising steps that re-plan
    seed: int = 0

    @property
    def N(self) -> int:
        t, y, x = self.grid
        return t * y * x

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def n_groups(self) -> int:
        return -(-self.N // self.G)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    # Work per reused step / dense step, as used for effective TFLOP/s.
    @property
    def sparse_flops(self) -> int:
        return 4 * self.BH * self.N * min(self.k, self.N) * self.d

    @property
    def dense_flops(self) -> int:
        return 4 * self.BH * self.N * self.N * self.d


def _pct(n: int, pct: int) -> int:
    return (n * pct) // 100


def _mk_workloads():
    c1 = Workload("tiny", 1, 1, 2, (8, 8, 16), 64, 64, 128, 8, "gauss", False,
                  2, 0.05, (1,))
    n2 = 13 * 30 * 40
    c2 = Workload("video_short", 2, 1, 16, (13, 30, 40), 64, 128, _pct(n2, 10), 32,
                  "gauss", False, 4, 0.03, (1,))
    n3 = 21 * 30 * 52
    c3 = Workload("video_long", 3, 1, 24, (21, 30, 52), 128, 128, _pct(n3, 5), 64,
                  "gauss", True, 8, 0.02, (1, 5))
    n4 = 64 * 32 * 32
    c4 = Workload("asset3d", 4, 2, 16, (64, 32, 32), 64, 128, _pct(n4, 3), 128,
                  "student_t3", False, 10, 0.02, (1, 6))
    n5 = 32 * 64 * 64
    c5 = Workload("sweep", 5, 1, 24, (32, 64, 64), 128, 128, _pct(n5, 5), 64,
                  "gauss", True, 2, 0.02, (1,))
    return {1: c1, 2: c2, 3: c3, 4: c4, 5: c5}


WORKLOADS = _mk_workloads()

SWEEP_PCTS = (1, 2, 5, 10, 25)
SWEEP_GROUPS = (64, 128)


def workload(which, k: Optional[int] = None, G: Optional[int] = None) -> Workload:
    """A workload by id (1-5) or by name ("tiny", "video_short", "video_long",
    "asset3d", "sweep"), optionally with another k or G."""
    if isinstance(which, str):
        hits = [w for w in WORKLOADS.values() if w.name == which]
        if not hits:
            raise KeyError(which)
        w = hits[0]
    else:
        w = WORKLOADS[which]
    if k is not None:
        w = w.with_(k=k)
    if G is not None:
        w = w.with_(G=G)
    return w


def sweep_points():
    """The sparsity sweep of the 131072-token workload: (G, pct, Workload)."""
    base = WORKLOADS[5]
    out = []
    for G in SWEEP_GROUPS:
        for p in SWEEP_PCTS:
            out.append((G, p, base.with_(G=G, k=_pct(base.N, p))))
    return out
