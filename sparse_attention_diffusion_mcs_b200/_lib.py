"""ctypes view of the C ABI in include/mcs.h (libmcs.so, built in-tree).

Loading needs no GPU: the library links the CUDA runtime statically and only
touches the driver on the first CUDA call.  Every function here is a plain
prototype; there is no fallback of any kind when the library is missing.
"""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libmcs.so")

MCS_OK = 0
STATUS_NAMES = {
    0: "MCS_OK", 1: "MCS_ERR_INVALID_ARG", 2: "MCS_ERR_UNSUPPORTED", 3: "MCS_ERR_WORKSPACE",
    4: "MCS_ERR_CUDA", 5: "MCS_ERR_TIMEOUT", 6: "MCS_ERR_BAD_META", 7: "MCS_ERR_TOO_LARGE",
}

# Every exported symbol and its prototype: (restype, argtypes).
c_int, c_size_t, c_float, c_vp, c_u64 = (ctypes.c_int, ctypes.c_size_t, ctypes.c_float,
                                        ctypes.c_void_p, ctypes.c_uint64)


class McsMeta(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("G", ctypes.c_int32), ("k", ctypes.c_int32),
                ("n_groups", ctypes.c_int32),
                ("perm", c_vp), ("kv_idx", c_vp), ("residual", c_vp),
                ("pair_idx", c_vp), ("pair_len", c_vp)]


PMETA = ctypes.POINTER(McsMeta)

PROTOTYPES = {
    "mcs_abi_version": (c_int, []),
    "mcs_status_string": (ctypes.c_char_p, [c_int]),
    "mcs_meta_init": (c_int, [PMETA, c_int, c_int, c_int, c_int, c_int, c_int]),
    "mcs_plan_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
    "mcs_plan": (c_int, [c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                         PMETA, c_vp, c_vp, c_size_t, c_vp]),
    "mcs_plan_workspace_offsets": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int,
                                           ctypes.POINTER(c_size_t), ctypes.POINTER(c_size_t),
                                           ctypes.POINTER(c_size_t), ctypes.POINTER(c_size_t)]),
    "mcs_plan_group": (c_int, [c_vp, c_int, c_int, c_int, c_int, c_vp, c_vp, c_size_t, c_vp]),
    "mcs_plan_stats": (c_int, [c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                               c_vp, c_vp, c_size_t, c_vp]),
    "mcs_plan_scores": (c_int, [c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                                c_vp, c_size_t, c_vp]),
    "mcs_plan_topk": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_vp, c_vp, c_size_t, c_vp]),
    "mcs_select_topk": (c_int, [c_vp, c_int, c_int, c_int, c_vp, c_vp]),
    "mcs_plan_residual": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int,
                                  c_int, c_float, c_vp, c_vp, c_size_t, c_vp]),
    "mcs_meta_pairs": (c_int, [PMETA, c_vp]),
    "mcs_sparse_step": (c_int, [c_vp, c_vp, c_vp, PMETA, c_float, c_vp, c_vp]),
    "mcs_dense": (c_int, [c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_float, c_vp, c_vp]),
    "mcs_residual_compact": (c_int, [c_vp, c_size_t, c_vp, c_vp]),
    "mcs_sparse_step_compact": (c_int, [c_vp, c_vp, c_vp, PMETA, c_vp, c_float, c_vp, c_vp]),
    "mcs_validate_workspace_size": (c_size_t, [c_int, c_int, c_int]),
    "mcs_validate_meta": (c_int, [PMETA, c_vp, c_size_t, ctypes.POINTER(c_int), c_vp]),
    "mcs_validate_meta_noalloc": (c_int, [PMETA, ctypes.POINTER(c_int), c_vp]),
    "mcs_select_blocks_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int]),
    "mcs_select_blocks": (c_int, [c_vp, c_int, c_int, c_int, c_int, c_vp, c_vp, c_size_t, c_vp]),
    "mcs_pooled_scores": (c_int, [c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_float, c_vp, c_vp]),
    "mcs_select_block_indices": (c_int, [c_vp, c_int, c_int, c_int, c_int, c_vp, c_vp, c_size_t, c_vp]),
    "mcs_union_pairs": (c_int, [c_vp, c_int, c_int, c_int, c_int, c_vp, c_vp, c_vp]),
    "mcs_sparse_step_blocks": (c_int, [c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                       c_vp, c_vp, c_vp, c_vp, c_float, c_vp, c_vp]),
    "mcs_last_device_status": (c_int, [c_vp]),
    "mcs_selftest_wait_timeout": (c_int, [c_u64, c_vp]),
    "mcs_set_wait_limit_ns": (None, [c_u64]),
}

_lib = None


class McsError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m sparse_attention_diffusion_mcs_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(code: int, where: str) -> None:
    if code != MCS_OK:
        raise McsError(code, where)
