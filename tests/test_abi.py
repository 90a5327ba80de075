"""The C ABI: the library loads without a GPU, exports every entry point the
header declares, and rejects bad arguments on the host with the documented
status codes before touching CUDA."""
import ctypes
import os
import re

import pytest

from sparse_attention_diffusion_mcs_b200 import _lib
from sparse_attention_diffusion_mcs_b200 import build as _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mcs.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = 0x10000   # 16-byte aligned non-null address; never dereferenced on these paths


@pytest.fixture(scope="module")
def L():
    _build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mcs_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported_and_bound(L):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.PROTOTYPES, n
    assert set(_lib.PROTOTYPES) == set(names)


def test_micro_library_exports_its_header():
    """libmcs_micro.so (include/mcs_micro.h) loads without a GPU, exports what
    its header declares, and refuses bad arguments before any launch."""
    from sparse_attention_diffusion_mcs_b200 import micro
    _build.build()
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "mcs_micro.h")).read(), flags=re.S)
    names = sorted(set(re.findall(r"\b(mcs_[a-z_0-9]+)\s*\(", text)))
    M = micro.lib()
    assert set(names) == set(micro.PROTOTYPES)
    for n in names:
        assert hasattr(M, n), n
    assert M.mcs_micro_gather(None, 1024, FAKE, 1, 1, 0, 1, None) == INVALID
    assert M.mcs_micro_gather(FAKE, 64, FAKE, 1, 1, 0, 1, None) == INVALID        # fewer rows than a tile
    assert M.mcs_micro_gather(FAKE, 1024, FAKE, 1, 1, 0, 9, None) == INVALID      # more than 8 warps
    assert M.mcs_micro_gather(FAKE, 1024, FAKE, 1, 1, 3, 1, None) == INVALID      # no such mode
    assert M.mcs_micro_gather(FAKE + 8, 1024, FAKE, 1, 1, 0, 1, None) == INVALID  # misaligned source
    assert M.mcs_micro_ex2(1, 8, 16, None, None) == INVALID
    assert M.mcs_micro_ex2(1, 33, 16, FAKE, None) == INVALID                      # more than 32 warps
    assert M.mcs_micro_mma(1, 3, 16, 0, 1, FAKE, None) == INVALID                  # no such shape
    assert M.mcs_micro_mma(1, 0, 16, 3, 1, FAKE, None) == INVALID                  # no such load
    assert M.mcs_micro_mma(1, 0, 0, 0, 1, FAKE, None) == INVALID
    assert M.mcs_micro_mma(1, 1, 16, 0, 3, FAKE, None) == INVALID                  # N = 128: two accumulators at most
    assert M.mcs_micro_mma(1, 0, 16, 0, 5, FAKE, None) == INVALID


def test_version_and_status_strings(L):
    assert L.mcs_abi_version() == 2
    for code, name in _lib.STATUS_NAMES.items():
        assert L.mcs_status_string(code).decode() == name


def test_meta_init_clamps_k_and_checks(L):
    m = _lib.McsMeta()
    assert L.mcs_meta_init(ctypes.byref(m), 1, 24, 32760, 128, 128, 1638) == OK
    assert (m.k, m.n_groups) == (1638, 256)
    assert L.mcs_meta_init(ctypes.byref(m), 1, 1, 100, 64, 64, 5000) == OK
    assert (m.k, m.n_groups) == (100, 2)
    assert L.mcs_meta_init(ctypes.byref(m), 1, 1, 100, 96, 64, 5) == UNSUPPORTED
    assert L.mcs_meta_init(ctypes.byref(m), 1, 1, 100, 64, 32, 5) == UNSUPPORTED
    assert L.mcs_meta_init(ctypes.byref(m), 1, 1, 0, 64, 64, 5) == INVALID
    assert L.mcs_meta_init(ctypes.byref(m), 1, 1, 100, 64, 64, 0) == INVALID
    assert L.mcs_meta_init(None, 1, 1, 100, 64, 64, 5) == INVALID


def test_workspace_size(L):
    assert L.mcs_plan_workspace_size(1, 24, 32760, 128, 128, 1638) > 24 * 256 * 32760 * 4
    assert L.mcs_plan_workspace_size(1, 1, 100, 96, 128, 5) == 0
    assert L.mcs_plan_workspace_size(0, 1, 100, 64, 128, 5) == 0
    assert L.mcs_validate_workspace_size(1, 2, 1024) >= 2 * 1024 // 8


def test_dense_argument_errors(L):
    s = None
    assert L.mcs_dense(None, FAKE, FAKE, 1, 1, 128, 64, 0.125, FAKE, s) == INVALID
    assert L.mcs_dense(FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, None, s) == INVALID
    assert L.mcs_dense(FAKE + 8, FAKE, FAKE, 1, 1, 128, 64, 0.125, FAKE, s) == INVALID
    assert L.mcs_dense(FAKE, FAKE, FAKE, 1, 1, 128, 96, 0.125, FAKE, s) == UNSUPPORTED
    assert L.mcs_dense(FAKE, FAKE, FAKE, 1, 1, 0, 64, 0.125, FAKE, s) == INVALID
    assert L.mcs_dense(FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.0, FAKE, s) == INVALID
    assert L.mcs_dense(FAKE, FAKE, FAKE, 1, 1, 128, 64, float("nan"), FAKE, s) == INVALID
    assert L.mcs_dense(FAKE, FAKE, FAKE, 70000, 1, 128, 64, 0.1, FAKE, s) == INVALID


def test_plan_argument_errors(L):
    m = _lib.McsMeta()
    m.perm, m.kv_idx, m.residual = FAKE, FAKE, FAKE
    need = L.mcs_plan_workspace_size(1, 2, 1024, 64, 64, 128)
    args = lambda ws, nbytes, G=64, d=64: (FAKE, FAKE, FAKE, 1, 2, 1024, d, G, 128, 0.125,
                                           ctypes.byref(m), None, ws, nbytes, None)
    assert L.mcs_plan(*args(None, need)) == WORKSPACE
    assert L.mcs_plan(*args(FAKE, need - 1)) == WORKSPACE
    assert L.mcs_plan(*args(FAKE + 16, need)) == WORKSPACE         # not 256-byte aligned
    assert L.mcs_plan(*args(FAKE, need, G=96)) == UNSUPPORTED
    assert L.mcs_plan(*args(FAKE, need, d=80)) == UNSUPPORTED
    m.residual = None
    assert L.mcs_plan(*args(FAKE, need)) == INVALID
    assert L.mcs_plan_group(None, 1, 1, 10, 64, FAKE, FAKE, 1 << 20, None) == INVALID
    assert L.mcs_plan_stats(FAKE, FAKE, FAKE, 1, 1, 10, 64, 64, 4, 0.1, None, None, 1 << 20,
                            None) == WORKSPACE
    assert L.mcs_plan_stats(FAKE, FAKE, FAKE, 1, 1, 10, 64, 64, 4, 0.1, FAKE + 8, FAKE, 1 << 20,
                            None) == INVALID
    assert L.mcs_plan_scores(FAKE, FAKE, None, 1, 1, 10, 64, 64, 4, 0.1, FAKE, 1 << 20, None) == INVALID
    assert L.mcs_plan_topk(1, 1, 10, 64, 64, 4, None, FAKE, 1 << 20, None) == INVALID
    assert L.mcs_plan_topk(1, 1, 10, 64, 64, 4, FAKE, FAKE, 16, None) == WORKSPACE
    assert L.mcs_select_topk(None, 4, 10, 3, FAKE, None) == INVALID
    assert L.mcs_select_topk(FAKE, 4, 10, 3, None, None) == INVALID
    assert L.mcs_select_topk(FAKE, -1, 10, 3, FAKE, None) == INVALID
    assert L.mcs_select_topk(FAKE, 4, 0, 3, FAKE, None) == INVALID
    assert L.mcs_select_topk(FAKE, 4, 10, 0, FAKE, None) == INVALID
    assert L.mcs_select_topk(FAKE, 0, 10, 3, FAKE, None) == OK          # no rows: nothing launched
    assert L.mcs_plan_residual(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 10, 64, 64, 4, 0.1, None,
                               FAKE, 1 << 20, None) == INVALID


def test_sparse_step_argument_errors(L):
    m = _lib.McsMeta()
    assert L.mcs_meta_init(ctypes.byref(m), 1, 2, 1024, 64, 64, 128) == OK
    m.perm, m.kv_idx, m.residual = FAKE, FAKE, FAKE
    assert L.mcs_sparse_step(FAKE, FAKE, FAKE, None, 0.125, FAKE, None) == INVALID
    assert L.mcs_sparse_step(FAKE, FAKE, FAKE, ctypes.byref(m), 0.125, None, None) == INVALID
    m.n_groups = 3
    assert L.mcs_sparse_step(FAKE, FAKE, FAKE, ctypes.byref(m), 0.125, FAKE, None) == INVALID
    m.n_groups = 16
    m.k = 2000
    assert L.mcs_sparse_step(FAKE, FAKE, FAKE, ctypes.byref(m), 0.125, FAKE, None) == INVALID
    m.k = 128
    m.G = 100
    assert L.mcs_sparse_step(FAKE, FAKE, FAKE, ctypes.byref(m), 0.125, FAKE, None) == UNSUPPORTED


def test_validate_argument_errors(L):
    m = _lib.McsMeta()
    assert L.mcs_meta_init(ctypes.byref(m), 1, 2, 1024, 64, 64, 128) == OK
    code = ctypes.c_int(-1)
    assert L.mcs_validate_meta(ctypes.byref(m), FAKE, 1 << 20, ctypes.byref(code), None) == INVALID
    m.perm, m.kv_idx, m.residual = FAKE, FAKE, FAKE
    assert L.mcs_validate_meta(ctypes.byref(m), None, 1 << 20, ctypes.byref(code), None) == WORKSPACE


def test_binding_refuses_to_run_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.lib()


def test_ablation_tool_argument_errors(L):
    s = None
    assert L.mcs_select_blocks_workspace_size(4, 1000, 64, 15) > 0
    assert L.mcs_select_blocks_workspace_size(4, 1000, 64, 16) == 0          # only 15 full blocks
    assert L.mcs_select_blocks(None, 4, 1000, 64, 2, FAKE, FAKE, 1 << 20, s) == INVALID
    assert L.mcs_select_blocks(FAKE, 4, 1000, 64, 0, FAKE, FAKE, 1 << 20, s) == INVALID
    assert L.mcs_select_blocks(FAKE, 4, 1000, 64, 16, FAKE, FAKE, 1 << 20, s) == INVALID
    assert L.mcs_select_blocks(FAKE, 4, 1000, 64, 2, FAKE, FAKE, 8, s) == WORKSPACE
    assert L.mcs_pooled_scores(FAKE, FAKE, None, 1, 1, 128, 64, 64, 0.125, FAKE, s) == INVALID
    assert L.mcs_pooled_scores(FAKE, FAKE, FAKE, 1, 1, 128, 64, 32, 0.125, FAKE, s) == UNSUPPORTED
    assert L.mcs_pooled_scores(FAKE, FAKE, FAKE, 1, 1, 128, 96, 64, 0.125, FAKE, s) == UNSUPPORTED


def test_block_step_argument_errors(L):
    s = None
    assert L.mcs_select_block_indices(None, 4, 1000, 64, 2, FAKE, FAKE, 1 << 20, s) == INVALID
    assert L.mcs_select_block_indices(FAKE, 4, 1000, 64, 16, FAKE, FAKE, 1 << 20, s) == INVALID
    assert L.mcs_select_block_indices(FAKE, 4, 1000, 64, 2, FAKE, FAKE, 8, s) == WORKSPACE
    assert L.mcs_union_pairs(None, 1, 1, 4, 8, FAKE, FAKE, s) == INVALID
    assert L.mcs_union_pairs(FAKE, 1, 1, 4, 0, FAKE, FAKE, s) == INVALID
    assert L.mcs_union_pairs(FAKE, 256, 257, 4, 8, FAKE, FAKE, s) == UNSUPPORTED
    args = lambda **kw: dict(dict(B=1, H=2, N=1024, d=128, G=128, block=64, kb=4, perm=FAKE, pidx=FAKE,
                                  plen=FAKE, res=None, scale=0.125, O=FAKE), **kw)
    step = lambda a: L.mcs_sparse_step_blocks(FAKE, FAKE, FAKE, a["B"], a["H"], a["N"], a["d"], a["G"], a["block"],
                                             a["kb"], a["perm"], a["pidx"], a["plen"], a["res"], a["scale"], a["O"], s)
    assert step(args(block=32)) == UNSUPPORTED
    assert step(args(G=96)) == UNSUPPORTED
    assert step(args(kb=0)) == INVALID
    assert step(args(kb=17)) == INVALID                   # only 16 blocks of 64 in 1024 keys
    assert step(args(block=128, kb=9)) == INVALID
    assert step(args(perm=None)) == INVALID
    assert step(args(pidx=None)) == INVALID
    assert step(args(res=FAKE + 4)) == INVALID   # a residual must be 16-byte aligned
    assert step(args(scale=0.0)) == INVALID


def test_compact_residual_argument_errors(L):
    s = None
    assert L.mcs_residual_compact(None, 0, None, s) == OK                  # nothing to convert
    assert L.mcs_residual_compact(None, 8, FAKE, s) == INVALID
    assert L.mcs_residual_compact(FAKE, 8, FAKE + 2, s) == INVALID         # misaligned output
    m = _lib.McsMeta()
    assert L.mcs_meta_init(ctypes.byref(m), 1, 2, 1024, 64, 64, 128) == OK
    m.perm, m.kv_idx = FAKE, FAKE
    assert L.mcs_sparse_step_compact(FAKE, FAKE, FAKE, ctypes.byref(m), FAKE, 0.125, FAKE, s) == INVALID  # no pairs
    m.pair_idx, m.pair_len = FAKE, FAKE
    assert L.mcs_sparse_step_compact(FAKE, FAKE, FAKE, ctypes.byref(m), None, 0.125, FAKE, s) == INVALID
    assert L.mcs_sparse_step_compact(FAKE, FAKE, FAKE, ctypes.byref(m), FAKE + 8, 0.125, FAKE, s) == INVALID
    assert L.mcs_sparse_step_compact(FAKE, FAKE, FAKE, None, FAKE, 0.125, FAKE, s) == INVALID
