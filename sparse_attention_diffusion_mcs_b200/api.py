"""Torch-facing binding of the MC-Sparse C ABI.

Argument marshalling only: every step of the hot path runs in the CUDA
library.  Tensors must be CUDA, contiguous; Q/K/V/O are bf16 [B, H, N, d].
Each call makes the inputs' device current for its duration and runs
asynchronously on torch's current stream of that device.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
from typing import Optional, Tuple

import torch

from ._lib import McsMeta, check, lib


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _on(device):
    """The library resolves its status word, tensor maps and launches on the
    CURRENT device, so every call runs with its tensors' device current."""
    return torch.cuda.device(device)


def _check_qkv(*ts: torch.Tensor):
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4):
            raise ValueError("Q/K/V must be contiguous CUDA bf16 tensors [B, H, N, d]")
    if any(t.shape != ts[0].shape for t in ts):
        raise ValueError("Q/K/V shapes differ")
    if any(t.device != ts[0].device for t in ts):
        raise ValueError("Q/K/V are on different devices")


def _check_tensor(t: torch.Tensor, name: str, shape, dtype, device):
    """Buffers the library writes or reads by the sizes it is given must be
    exactly what those sizes describe: a mismatch would be an out-of-bounds
    access on the device, so it is refused here, before any launch."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.device != device or t.dtype != dtype or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {device}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def _check_meta(meta: "Meta", B: int, H: int, N: int, d: int, device, G: Optional[int] = None,
                k: Optional[int] = None):
    """meta's sizes match the layer [B, H, N, d] (and G, k when given) and
    its buffers are the sizes those describe."""
    if (meta.B, meta.H, meta.N, meta.d) != (B, H, N, d):
        raise ValueError(f"metadata is for [B, H, N, d] = {[meta.B, meta.H, meta.N, meta.d]}, "
                         f"the layer is {[B, H, N, d]}")
    if G is not None and meta.G != G:
        raise ValueError(f"metadata group size {meta.G} != {G}")
    if k is not None and meta.k != min(int(k), N):
        raise ValueError(f"metadata keeps {meta.k} keys per group, not min(k, N) = {min(int(k), N)}")
    ng = -(-N // meta.G)
    if meta.n_groups != ng:
        raise ValueError(f"metadata n_groups {meta.n_groups} != ceil(N / G) = {ng}")
    _check_tensor(meta.perm, "meta.perm", (B, H, N), torch.int32, device)
    _check_tensor(meta.kv_idx, "meta.kv_idx", (B, H, ng, meta.k), torch.int32, device)
    _check_tensor(meta.residual, "meta.residual", (B, H, N, d), torch.float32, device)
    if (meta.pair_idx is None) != (meta.pair_len is None):
        raise ValueError("meta.pair_idx and meta.pair_len come together")
    if meta.pair_idx is not None:
        npairs = (ng + 1) // 2
        _check_tensor(meta.pair_idx, "meta.pair_idx", (B, H, npairs, 2 * meta.k), torch.int32, device)
        _check_tensor(meta.pair_len, "meta.pair_len", (B, H, npairs), torch.int32, device)


def _scale(d: int, scale: Optional[float]) -> float:
    return float(scale) if scale is not None else 1.0 / math.sqrt(d)


@dataclasses.dataclass
class Meta:
    """Cached metadata of a plan: query order, KV indices, residual."""
    B: int
    H: int
    N: int
    d: int
    G: int
    k: int
    n_groups: int
    perm: torch.Tensor       # int32 [B, H, N]
    kv_idx: torch.Tensor     # int32 [B, H, n_groups, k]
    residual: torch.Tensor   # float32 [B, H, N, d]
    # union lists of adjacent group pairs, derived from kv_idx (include/mcs.h);
    # None: the reused step runs one group at a time
    pair_idx: Optional[torch.Tensor] = None   # int32 [B, H, n_pairs, 2k]
    pair_len: Optional[torch.Tensor] = None   # int32 [B, H, n_pairs]

    @property
    def n_pairs(self) -> int:
        return (self.n_groups + 1) // 2

    def c_struct(self) -> McsMeta:
        return McsMeta(self.B, self.H, self.N, self.d, self.G, self.k, self.n_groups,
                       self.perm.data_ptr(), self.kv_idx.data_ptr(), self.residual.data_ptr(),
                       self.pair_idx.data_ptr() if self.pair_idx is not None else 0,
                       self.pair_len.data_ptr() if self.pair_len is not None else 0)

    @staticmethod
    def empty(B: int, H: int, N: int, d: int, G: int, k: int, device="cuda", pairs: bool = True) -> "Meta":
        k = min(int(k), N)
        ng = -(-N // G)
        np_ = (ng + 1) // 2
        return Meta(B, H, N, d, G, k, ng,
                    torch.empty((B, H, N), dtype=torch.int32, device=device),
                    torch.empty((B, H, ng, k), dtype=torch.int32, device=device),
                    torch.empty((B, H, N, d), dtype=torch.float32, device=device),
                    torch.empty((B, H, np_, 2 * k), dtype=torch.int32, device=device) if pairs else None,
                    torch.empty((B, H, np_), dtype=torch.int32, device=device) if pairs else None)

    def build_pairs(self) -> "Meta":
        """(Re)build pair_idx / pair_len from kv_idx on the device (allocating
        them when absent); returns self."""
        dev = self.kv_idx.device
        if self.pair_idx is None or self.pair_len is None:
            self.pair_idx = torch.empty((self.B, self.H, self.n_pairs, 2 * self.k), dtype=torch.int32,
                                        device=dev)
            self.pair_len = torch.empty((self.B, self.H, self.n_pairs), dtype=torch.int32, device=dev)
        _check_meta(self, self.B, self.H, self.N, self.d, dev)
        cm = self.c_struct()
        with _on(dev):
            check(lib().mcs_meta_pairs(ctypes.byref(cm), _stream(dev)), "mcs_meta_pairs")
        return self

    def without_pairs(self) -> "Meta":
        """The same metadata with no pair lists (one group at a time)."""
        return dataclasses.replace(self, pair_idx=None, pair_len=None)

    def save(self, path) -> None:
        """Write the cached metadata (the state a denoising loop reuses) to
        `path` with torch.save; `Meta.load` restores it bit for bit."""
        torch.save({"format": "mcs-meta-1", "sizes": [self.B, self.H, self.N, self.d, self.G, self.k,
                                                      self.n_groups],
                    "perm": self.perm.cpu(), "kv_idx": self.kv_idx.cpu(), "residual": self.residual.cpu()},
                   path)

    @staticmethod
    def load(path, device="cuda", pairs: bool = True) -> "Meta":
        """Metadata written by `Meta.save`, on `device`; the pair lists (derived
        data, not saved) are rebuilt from kv_idx on a CUDA device."""
        blob = torch.load(path, map_location="cpu", weights_only=True)
        if blob.get("format") != "mcs-meta-1":
            raise ValueError(f"{path}: not saved metadata")
        B, H, N, d, G, k, ng = (int(x) for x in blob["sizes"])
        meta = Meta(B, H, N, d, G, k, ng, blob["perm"].to(device).contiguous(),
                    blob["kv_idx"].to(device).contiguous(), blob["residual"].to(device).contiguous())
        _check_meta(meta, B, H, N, d, meta.perm.device)
        if pairs and meta.kv_idx.is_cuda:
            meta.build_pairs()
        return meta

    @staticmethod
    def from_tensors(perm, kv_idx, residual, G: int, pairs: bool = True) -> "Meta":
        """Metadata from caller tensors; with `pairs` (CUDA tensors) the pair
        lists are built from kv_idx."""
        B, H, N, d = residual.shape
        ng, k = kv_idx.shape[2], kv_idx.shape[3]
        meta = Meta(B, H, N, d, G, k, ng, perm.contiguous(), kv_idx.contiguous(), residual.contiguous())
        if pairs and meta.kv_idx.is_cuda:
            meta.build_pairs()
        return meta


def workspace_size(B: int, H: int, N: int, d: int, G: int, k: int) -> int:
    n = lib().mcs_plan_workspace_size(B, H, N, d, G, k)
    if n == 0:
        raise ValueError("unsupported shape")
    return int(n)


def alloc_workspace(B: int, H: int, N: int, d: int, G: int, k: int, device="cuda") -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(workspace_size(B, H, N, d, G, k), dtype=torch.uint8, device=device)


def workspace_views(workspace: torch.Tensor, B: int, H: int, N: int, d: int, G: int, k: int):
    """Views of the plan workspace's statistics and group scores (no copies):
    {"row_m": [B,H,N] (log2 units), "row_l": [B,H,N], "O32": [B,H,N,d],
    "colsum": [B,H,n_groups,N]}, all float32 (layout in include/mcs.h)."""
    offs = [ctypes.c_size_t(0) for _ in range(4)]
    check(lib().mcs_plan_workspace_offsets(B, H, N, d, G, k, *[ctypes.byref(o) for o in offs]),
          "mcs_plan_workspace_offsets")
    ng = -(-N // G)
    shapes = {"row_m": (B, H, N), "row_l": (B, H, N), "O32": (B, H, N, d), "colsum": (B, H, ng, N)}
    out = {}
    for (name, shape), off in zip(shapes.items(), offs):
        n = 1
        for x in shape:
            n *= x
        start = int(off.value)
        if start + 4 * n > workspace.numel():
            raise ValueError("workspace smaller than the layout needs")
        out[name] = workspace[start:start + 4 * n].view(torch.float32).view(shape)
    return out


def _ws(ws: Optional[torch.Tensor], B, H, N, d, G, k, device):
    if ws is None:
        ws = alloc_workspace(B, H, N, d, G, k, device)
    return ws


def plan(Q, K, V, G: int, k: int, scale: Optional[float] = None,
         workspace: Optional[torch.Tensor] = None, meta: Optional[Meta] = None,
         out_dense: Optional[torch.Tensor] = None, return_dense: bool = False):
    """Metadata pass (steps a1-a5).  Returns Meta, or (Meta, O_dense bf16)."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    if meta is None:
        meta = Meta.empty(B, H, N, d, G, k, Q.device)
    else:
        _check_meta(meta, B, H, N, d, Q.device, G, k)
    if out_dense is not None:
        _check_tensor(out_dense, "out_dense", Q.shape, torch.bfloat16, Q.device)
    if return_dense and out_dense is None:
        out_dense = torch.empty_like(Q)
    ws = _ws(workspace, B, H, N, d, G, k, Q.device)
    cm = meta.c_struct()
    with _on(Q.device):
        check(lib().mcs_plan(_ptr(Q), _ptr(K), _ptr(V), B, H, N, d, G, k, _scale(d, scale),
                             ctypes.byref(cm), _ptr(out_dense), _ptr(ws), ws.numel(), _stream(Q.device)),
              "mcs_plan")
    meta.k, meta.n_groups = cm.k, cm.n_groups
    return (meta, out_dense) if (return_dense or out_dense is not None) else meta


def plan_group(Q, workspace: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Step a1 alone: int32 perm [B, H, N]."""
    _check_qkv(Q)
    B, H, N, d = Q.shape
    if out is not None:
        _check_tensor(out, "out", (B, H, N), torch.int32, Q.device)
    perm = out if out is not None else torch.empty((B, H, N), dtype=torch.int32, device=Q.device)
    ws = _ws(workspace, B, H, N, d, 128, 1, Q.device)
    with _on(Q.device):
        check(lib().mcs_plan_group(_ptr(Q), B, H, N, d, _ptr(perm), _ptr(ws), ws.numel(), _stream(Q.device)),
              "mcs_plan_group")
    return perm


def plan_stats(Q, K, V, G: int, k: int, scale: Optional[float] = None,
               workspace: Optional[torch.Tensor] = None, return_dense: bool = False,
               out_dense: Optional[torch.Tensor] = None):
    """Step a2 into the workspace (row statistics, fp32 dense output).
    Returns the workspace, or (workspace, O_dense bf16)."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    ws = _ws(workspace, B, H, N, d, G, k, Q.device)
    if out_dense is not None:
        _check_tensor(out_dense, "out_dense", Q.shape, torch.bfloat16, Q.device)
    od = out_dense if out_dense is not None else (torch.empty_like(Q) if return_dense else None)
    with _on(Q.device):
        check(lib().mcs_plan_stats(_ptr(Q), _ptr(K), _ptr(V), B, H, N, d, G, k, _scale(d, scale), _ptr(od),
                                   _ptr(ws), ws.numel(), _stream(Q.device)), "mcs_plan_stats")
    return (ws, od) if (return_dense or out_dense is not None) else ws


def plan_scores(Q, K, perm, G: int, k: int, workspace: torch.Tensor,
                scale: Optional[float] = None) -> None:
    """Step a3 into the workspace (needs plan_stats on the same workspace)."""
    _check_qkv(Q, K)
    B, H, N, d = Q.shape
    perm = perm.to(torch.int32).contiguous()
    _check_tensor(perm, "perm", (B, H, N), torch.int32, Q.device)
    _check_tensor(workspace, "workspace", (workspace.numel(),), torch.uint8, Q.device)
    with _on(Q.device):
        check(lib().mcs_plan_scores(_ptr(Q), _ptr(K), _ptr(perm), B, H, N, d, G, k, _scale(d, scale),
                                    _ptr(workspace), workspace.numel(), _stream(Q.device)), "mcs_plan_scores")


def plan_topk(B: int, H: int, N: int, d: int, G: int, k: int, workspace: torch.Tensor,
              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Step a4 (needs plan_scores on the same workspace): int32 kv_idx."""
    kk = min(int(k), N)
    if out is None:
        out = torch.empty((B, H, -(-N // G), kk), dtype=torch.int32, device=workspace.device)
    else:
        _check_tensor(out, "out", (B, H, -(-N // G), kk), torch.int32, workspace.device)
    with _on(workspace.device):
        check(lib().mcs_plan_topk(B, H, N, d, G, k, _ptr(out), _ptr(workspace), workspace.numel(),
                                  _stream(workspace.device)), "mcs_plan_topk")
    return out


def select_topk(scores: torch.Tensor, k: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Step a4 on any float32 score matrix [..., N]: int32 indices of the
    min(k, N) largest per row, ties to the lower index, ascending."""
    if scores.dtype != torch.float32 or not scores.is_cuda:
        raise TypeError("scores must be a float32 CUDA tensor")
    scores = scores.contiguous()
    N = scores.shape[-1]
    rows = scores.numel() // N if N else 0
    kk = min(int(k), N)
    if out is None:
        out = torch.empty((*scores.shape[:-1], kk), dtype=torch.int32, device=scores.device)
    else:
        _check_tensor(out, "out", (*scores.shape[:-1], kk), torch.int32, scores.device)
    if rows == 0:
        return out
    with _on(scores.device):
        check(lib().mcs_select_topk(_ptr(scores), rows, N, int(k), _ptr(out), _stream(scores.device)),
              "mcs_select_topk")
    return out


def select_blocks(scores: torch.Tensor, k_blocks: int, block: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Block-granular selection on a float32 score matrix [..., N] (an
    ablation of token-level selection): per row the k_blocks aligned blocks
    of `block` keys with the highest summed score (full blocks only), as
    their keys ascending: int32 [..., k_blocks * block]."""
    if scores.dtype != torch.float32 or not scores.is_cuda:
        raise TypeError("scores must be a float32 CUDA tensor")
    scores = scores.contiguous()
    N = scores.shape[-1]
    rows = scores.numel() // N if N else 0
    if not 1 <= k_blocks <= N // block:
        raise ValueError(f"k_blocks must be in [1, N // block] = [1, {N // block}]")
    if out is None:
        out = torch.empty((*scores.shape[:-1], k_blocks * block), dtype=torch.int32, device=scores.device)
    else:
        _check_tensor(out, "out", (*scores.shape[:-1], k_blocks * block), torch.int32, scores.device)
    n = lib().mcs_select_blocks_workspace_size(rows, N, block, k_blocks)
    ws = torch.empty(max(int(n), 1), dtype=torch.uint8, device=scores.device)
    with _on(scores.device):
        check(lib().mcs_select_blocks(_ptr(scores), rows, N, block, k_blocks, _ptr(out), _ptr(ws), ws.numel(),
                                      _stream(scores.device)), "mcs_select_blocks")
    return out


def select_block_indices(scores: torch.Tensor, k_blocks: int, block: int,
                         out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """As `select_blocks`, but the kept blocks' indices ascending: int32
    [..., k_blocks] (block b holds keys [b*block, (b+1)*block))."""
    if scores.dtype != torch.float32 or not scores.is_cuda:
        raise TypeError("scores must be a float32 CUDA tensor")
    scores = scores.contiguous()
    N = scores.shape[-1]
    rows = scores.numel() // N if N else 0
    if not 1 <= k_blocks <= N // block:
        raise ValueError(f"k_blocks must be in [1, N // block] = [1, {N // block}]")
    if out is None:
        out = torch.empty((*scores.shape[:-1], k_blocks), dtype=torch.int32, device=scores.device)
    else:
        _check_tensor(out, "out", (*scores.shape[:-1], k_blocks), torch.int32, scores.device)
    n = lib().mcs_select_blocks_workspace_size(rows, N, block, k_blocks)
    ws = torch.empty(max(int(n), 1), dtype=torch.uint8, device=scores.device)
    with _on(scores.device):
        check(lib().mcs_select_block_indices(_ptr(scores), rows, N, block, k_blocks, _ptr(out), _ptr(ws),
                                             ws.numel(), _stream(scores.device)), "mcs_select_block_indices")
    return out


def union_pairs(lists: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """Union lists of adjacent group pairs of ascending per-group lists
    (int32 [B, H, n_groups, k], keys or block indices): (pair_idx int32
    [B, H, n_pairs, 2k], pair_len int32 [B, H, n_pairs])."""
    if lists.dtype != torch.int32 or not lists.is_cuda or lists.dim() != 4:
        raise TypeError("lists must be an int32 CUDA tensor [B, H, n_groups, k]")
    lists = lists.contiguous()
    B, H, ng, k = lists.shape
    np_ = (ng + 1) // 2
    pair_idx = torch.empty((B, H, np_, 2 * k), dtype=torch.int32, device=lists.device)
    pair_len = torch.empty((B, H, np_), dtype=torch.int32, device=lists.device)
    with _on(lists.device):
        check(lib().mcs_union_pairs(_ptr(lists), B, H, ng, k, _ptr(pair_idx), _ptr(pair_len),
                                    _stream(lists.device)), "mcs_union_pairs")
    return pair_idx, pair_len


@dataclasses.dataclass
class BlockMeta:
    """A block-granular selection for `sparse_step_blocks`: the grouping, each
    group's kept block indices, their pair union lists, an optional residual."""
    G: int
    block: int
    perm: torch.Tensor                       # int32 [B, H, N]
    blk_idx: torch.Tensor                    # int32 [B, H, n_groups, k_blocks], ascending
    pair_idx: torch.Tensor                   # int32 [B, H, n_pairs, 2 k_blocks]
    pair_len: torch.Tensor                   # int32 [B, H, n_pairs]
    residual: Optional[torch.Tensor] = None  # float32 [B, H, N, d]

    @property
    def k_blocks(self) -> int:
        return self.blk_idx.shape[3]

    @staticmethod
    def build(perm, blk_idx, G: int, block: int, residual: Optional[torch.Tensor] = None) -> "BlockMeta":
        pair_idx, pair_len = union_pairs(blk_idx)
        return BlockMeta(G, block, perm.contiguous(), blk_idx.contiguous(), pair_idx, pair_len,
                         None if residual is None else residual.contiguous())


def sparse_step_blocks(Q, K, V, bm: BlockMeta, scale: Optional[float] = None,
                       out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The reused step over a block-granular selection (blocks of 64 or 128
    keys), with bm's residual added when it has one: bf16 O [B, H, N, d]."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    ng = -(-N // bm.G)
    np_ = (ng + 1) // 2
    _check_tensor(bm.perm, "perm", (B, H, N), torch.int32, Q.device)
    _check_tensor(bm.blk_idx, "blk_idx", (B, H, ng, bm.k_blocks), torch.int32, Q.device)
    _check_tensor(bm.pair_idx, "pair_idx", (B, H, np_, 2 * bm.k_blocks), torch.int32, Q.device)
    _check_tensor(bm.pair_len, "pair_len", (B, H, np_), torch.int32, Q.device)
    if bm.residual is not None:
        _check_tensor(bm.residual, "residual", (B, H, N, d), torch.float32, Q.device)
    if out is None:
        out = torch.empty_like(Q)
    else:
        _check_tensor(out, "out", Q.shape, torch.bfloat16, Q.device)
    with _on(Q.device):
        check(lib().mcs_sparse_step_blocks(_ptr(Q), _ptr(K), _ptr(V), B, H, N, d, bm.G, bm.block, bm.k_blocks,
                                           _ptr(bm.perm), _ptr(bm.pair_idx), _ptr(bm.pair_len),
                                           _ptr(bm.residual), _scale(d, scale), _ptr(out), _stream(Q.device)),
              "mcs_sparse_step_blocks")
    return out


def pooled_scores(Q, K, perm, G: int, scale: Optional[float] = None,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Pooled-query scores (an ablation of exact summed probabilities):
    float32 [B, H, n_groups, N], softmax_j(scale mean_{i in g}(Q_i) . K_j)."""
    _check_qkv(Q, K)
    B, H, N, d = Q.shape
    perm = perm.to(torch.int32).contiguous()
    _check_tensor(perm, "perm", (B, H, N), torch.int32, Q.device)
    ng = -(-N // G)
    if out is None:
        out = torch.empty((B, H, ng, N), dtype=torch.float32, device=Q.device)
    else:
        _check_tensor(out, "out", (B, H, ng, N), torch.float32, Q.device)
    with _on(Q.device):
        check(lib().mcs_pooled_scores(_ptr(Q), _ptr(K), _ptr(perm), B, H, N, d, G, _scale(d, scale), _ptr(out),
                                      _stream(Q.device)), "mcs_pooled_scores")
    return out


def plan_select(Q, K, V, perm, G: int, k: int, scale: Optional[float] = None,
                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Steps a2-a4 for a given grouping: int32 kv_idx [B, H, n_groups, min(k, N)].
    (a2 also leaves the dense output of Q, K, V in the workspace.)"""
    B, H, N, d = Q.shape
    ws = plan_stats(Q, K, V, G, k, scale, workspace)
    plan_scores(Q, K, perm, G, k, ws, scale)
    return plan_topk(B, H, N, d, G, k, ws)


def plan_residual(Q, K, V, perm, kv_idx, G: int, scale: Optional[float] = None,
                  workspace: Optional[torch.Tensor] = None, stats_done: bool = False,
                  return_dense: bool = False, out: Optional[torch.Tensor] = None):
    """Step a5 (running a2 first unless stats_done): float32 residual."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    perm = perm.to(torch.int32).contiguous()
    kv_idx = kv_idx.to(torch.int32).contiguous()
    k = kv_idx.shape[-1]
    _check_tensor(perm, "perm", (B, H, N), torch.int32, Q.device)
    _check_tensor(kv_idx, "kv_idx", (B, H, -(-N // G), min(k, N)), torch.int32, Q.device)
    if out is not None:
        _check_tensor(out, "out", (B, H, N, d), torch.float32, Q.device)
    od = None
    if stats_done:
        if workspace is None:
            raise ValueError("stats_done needs the workspace plan_stats filled")
        ws = workspace
    elif return_dense:
        ws, od = plan_stats(Q, K, V, G, k, scale, workspace, return_dense=True)
    else:
        ws = plan_stats(Q, K, V, G, k, scale, workspace)
    res = out if out is not None else torch.empty((B, H, N, d), dtype=torch.float32, device=Q.device)
    with _on(Q.device):
        check(lib().mcs_plan_residual(_ptr(Q), _ptr(K), _ptr(V), _ptr(perm), _ptr(kv_idx), B, H, N, d,
                                      G, k, _scale(d, scale), _ptr(res), _ptr(ws), ws.numel(),
                                      _stream(Q.device)),
              "mcs_plan_residual")
    return (res, od) if return_dense else res


def sparse_step(Q, K, V, meta: Meta, scale: Optional[float] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Reused denoising step (a6): bf16 O [B, H, N, d]."""
    _check_qkv(Q, K, V)
    _check_meta(meta, *Q.shape, Q.device)
    if out is None:
        out = torch.empty_like(Q)
    else:
        _check_tensor(out, "out", Q.shape, torch.bfloat16, Q.device)
    cm = meta.c_struct()
    with _on(Q.device):
        check(lib().mcs_sparse_step(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(cm),
                                    _scale(meta.d, scale), _ptr(out), _stream(Q.device)), "mcs_sparse_step")
    return out


def compact_residual(residual: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The cached residual as bf16 (round to nearest even), same shape: half
    the bytes the reused step reads and a cached plan keeps."""
    if residual.dtype != torch.float32 or not residual.is_cuda:
        raise TypeError("residual must be a float32 CUDA tensor")
    residual = residual.contiguous()
    if out is None:
        out = torch.empty(residual.shape, dtype=torch.bfloat16, device=residual.device)
    else:
        _check_tensor(out, "out", residual.shape, torch.bfloat16, residual.device)
    with _on(residual.device):
        check(lib().mcs_residual_compact(_ptr(residual), residual.numel(), _ptr(out), _stream(residual.device)),
              "mcs_residual_compact")
    return out


def sparse_step_compact(Q, K, V, meta: Meta, residual16: torch.Tensor, scale: Optional[float] = None,
                        out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The reused step with the residual read from its bf16 copy
    (`compact_residual`) instead of meta.residual: bf16 O [B, H, N, d].
    Needs meta's pair lists."""
    _check_qkv(Q, K, V)
    _check_meta(meta, *Q.shape, Q.device)
    if meta.pair_idx is None:
        raise ValueError("the compact-residual step needs the metadata's pair lists (Meta.build_pairs)")
    _check_tensor(residual16, "residual16", Q.shape, torch.bfloat16, Q.device)
    if out is None:
        out = torch.empty_like(Q)
    else:
        _check_tensor(out, "out", Q.shape, torch.bfloat16, Q.device)
    cm = meta.c_struct()
    with _on(Q.device):
        check(lib().mcs_sparse_step_compact(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(cm), _ptr(residual16),
                                            _scale(meta.d, scale), _ptr(out), _stream(Q.device)),
              "mcs_sparse_step_compact")
    return out


def dense(Q, K, V, scale: Optional[float] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Dense attention (a7): bf16 O [B, H, N, d]."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    if out is None:
        out = torch.empty_like(Q)
    else:
        _check_tensor(out, "out", Q.shape, torch.bfloat16, Q.device)
    with _on(Q.device):
        check(lib().mcs_dense(_ptr(Q), _ptr(K), _ptr(V), B, H, N, d, _scale(d, scale), _ptr(out),
                              _stream(Q.device)), "mcs_dense")
    return out


def validate_meta(meta: Meta) -> Tuple[bool, int]:
    """(valid, first failing check code); synchronous."""
    dev = meta.perm.device
    _check_meta(meta, meta.B, meta.H, meta.N, meta.d, dev)
    n = lib().mcs_validate_workspace_size(meta.B, meta.H, meta.N)
    ws = torch.empty(int(n), dtype=torch.uint8, device=dev)
    code = ctypes.c_int(0)
    cm = meta.c_struct()
    with _on(dev):
        st = lib().mcs_validate_meta(ctypes.byref(cm), _ptr(ws), ws.numel(), ctypes.byref(code), _stream(dev))
    if st == 6:
        return False, code.value
    check(st, "mcs_validate_meta")
    return True, 0


def last_device_status(device=None) -> int:
    """Read and clear the status word of `device` (default: the current one)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with _on(dev):
        return int(lib().mcs_last_device_status(_stream(dev)))


def set_wait_limit_ns(ns: int) -> None:
    lib().mcs_set_wait_limit_ns(int(ns))


def selftest_wait_timeout(limit_ns: int) -> None:
    check(lib().mcs_selftest_wait_timeout(int(limit_ns), _stream(None)), "mcs_selftest_wait_timeout")
