"""Binding of libmcs_micro.so (include/mcs_micro.h): the rate at which one SM
brings index-listed 256-byte rows into shared memory, measured on its own.
Measurement only; nothing on the hot path uses it."""
from __future__ import annotations

import ctypes
import os
from typing import Dict

import torch

from ._lib import PKG_DIR, check

MICRO_LIB_PATH = os.path.join(PKG_DIR, "libmcs_micro.so")
MODES = {"gather4": 0, "cp.async": 1, "tile": 2}
PROTOTYPES = {
    "mcs_micro_gather": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "mcs_micro_last_status": (ctypes.c_int, [ctypes.c_void_p]),
}
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(MICRO_LIB_PATH):
            raise ImportError(f"{MICRO_LIB_PATH} is missing: build with "
                              "`python -m sparse_attention_diffusion_mcs_b200.build`")
        L = ctypes.CDLL(MICRO_LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def gather_rate(mode: str, warps: int, rows: int = 65536, tiles: int = 256, reps: int = 5,
                seed: int = 0, device="cuda") -> Dict[str, float]:
    """Median bytes/s over `reps` launches of one CTA per SM streaming `tiles`
    tiles of 128 rows x 256 bytes each from a bf16 [rows, 128] source
    (16.8 MB at the default: one head's K and V at d = 128, L2-resident) with
    uniformly random row indices ("tile": contiguous 128-row tiles)."""
    dev = torch.device(device)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    g = torch.Generator(device="cpu").manual_seed(seed)
    src = torch.randn((rows, 128), generator=g).to(torch.bfloat16).to(dev)
    n = sms * tiles * 128
    if mode == "tile":
        starts = torch.randint(0, rows // 128, (sms * tiles,), generator=g) * 128
        idx = (starts[:, None] + torch.arange(128)[None, :]).reshape(-1).to(torch.int32)
    else:
        idx = torch.randint(0, rows, (n,), generator=g, dtype=torch.int32)
    idx = idx.to(dev)
    stream = torch.cuda.current_stream(dev)
    s = ctypes.c_void_p(stream.cuda_stream)
    L = lib()
    call = lambda: check(L.mcs_micro_gather(ctypes.c_void_p(src.data_ptr()), rows, ctypes.c_void_p(idx.data_ptr()),
                                            sms, tiles, MODES[mode], warps, s), "mcs_micro_gather")
    call()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        torch.cuda.synchronize(dev)
        times.append(a.elapsed_time(b) * 1e-3)
    check(L.mcs_micro_last_status(s), "mcs_micro_gather (device status)")
    t = sorted(times)[len(times) // 2]
    nbytes = sms * tiles * 128 * 256
    return {"mode": mode, "warps": warps, "bytes": nbytes, "seconds": t, "gbs": nbytes / t / 1e9,
            "gbs_per_sm": nbytes / t / 1e9 / sms}
