"""The allocation-free validation entry point (mcs_validate_meta_noalloc).

Some callers of this library cannot allocate device memory when they want to
check cached metadata: a serving runtime that reserves all device memory at
start-up and forbids allocation afterwards, or a plugin whose host framework
owns all device memory and its allocator.  For them the library keeps a fixed
scratch array of its own (a call is synchronous, like mcs_validate_meta).
These tests call it through the C ABI and check that it reports exactly what
the workspace-based mcs_validate_meta reports, call after call, so leftovers
in the shared array never leak into a later answer.

This file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import mcs_oracle as orc
from sparse_attention_diffusion_mcs_b200 import _lib
from sparse_attention_diffusion_mcs_b200 import build as _build

OK, INVALID, BAD_META, TOO_LARGE = 0, 1, 6, 7


def _call_noalloc(L, cm):
    code = ctypes.c_int(-1)
    st = L.mcs_validate_meta_noalloc(ctypes.byref(cm), ctypes.byref(code),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, code.value


def _call_workspace(L, cm, B, H, N):
    n = L.mcs_validate_workspace_size(B, H, N)
    ws = torch.empty(int(n), dtype=torch.uint8, device="cuda")
    code = ctypes.c_int(-1)
    st = L.mcs_validate_meta(ctypes.byref(cm), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                             ctypes.byref(code), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, code.value


def test_noalloc_rejects_shapes_beyond_its_scratch():
    _build.build()
    L = _lib.lib()
    m = _lib.McsMeta()
    assert L.mcs_meta_init(ctypes.byref(m), 1, 128, 65537, 128, 128, 64) == OK   # 8,388,736 tokens
    m.perm, m.kv_idx, m.residual = 0x10000, 0x10000, 0x10000
    code = ctypes.c_int(-1)
    assert L.mcs_validate_meta_noalloc(ctypes.byref(m), ctypes.byref(code), None) == TOO_LARGE
    assert L.mcs_validate_meta_noalloc(None, ctypes.byref(code), None) == INVALID
    assert L.mcs_status_string(TOO_LARGE).decode() == "MCS_ERR_TOO_LARGE"


@pytest.mark.gpu
def test_noalloc_matches_workspace_validation_call_after_call():
    _build.build()
    L = _lib.lib()
    w = synth.workload(1)
    Q, K, V = synth.layer_tensors(w)
    metas = [orc.plan_head(Q[0, h], K[0, h], V[0, h], w.G, w.k, w.scale) for h in range(w.H)]
    perm = np.stack([m["perm"] for m in metas]).astype(np.int32)[None]
    kv = np.stack([m["kv_idx"] for m in metas]).astype(np.int32)[None]
    res = np.stack([m["residual"] for m in metas]).astype(np.float32)[None]

    bad_perm = perm.copy()
    bad_perm[0, 1, 5] = bad_perm[0, 1, 6]
    bad_kv = kv.copy()
    bad_kv[0, 0, 3, 7] = bad_kv[0, 0, 3, 6]
    bad_res = res.copy()
    bad_res[0, 1, 10, 3] = np.inf
    # valid, corrupt, valid again (the shared array must not carry the bad bits over), ...
    sequence = [(perm, kv, res), (bad_perm, kv, res), (perm, kv, res), (perm, bad_kv, res),
                (perm, kv, bad_res), (perm, kv, res)]
    expected = [(OK, 0), (BAD_META, 1), (OK, 0), (BAD_META, 3), (BAD_META, 4), (OK, 0)]
    for (p, k_, r), want in zip(sequence, expected):
        tp, tk, tr = (torch.from_numpy(x).cuda() for x in (p, k_, r))
        cm = _lib.McsMeta(w.B, w.H, w.N, w.d, w.G, w.k, w.n_groups, tp.data_ptr(), tk.data_ptr(),
                          tr.data_ptr())
        ref = _call_workspace(L, cm, w.B, w.H, w.N)
        first = _call_noalloc(L, cm)
        second = _call_noalloc(L, cm)          # two calls in a row on the same input
        assert ref == want
        assert first == ref and second == ref
