"""Binding of libmcs_micro.so (include/mcs_micro.h), each rate measured on its
own: the rate at which one SM brings index-listed 256-byte rows into shared
memory, its MUFU exponential rate, and its tcgen05 MMA rate for the reused
step's MMA shapes, alone and beside MUFU or FMA work.  Measurement only;
nothing on the hot path uses it."""
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
    "mcs_micro_ex2": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "mcs_micro_mma": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_void_p, ctypes.c_void_p]),
}
MMA_SHAPES = {"qk_ss_128x64": (0, 128 * 64 * 16 * 2), "pv_ts_128x128": (1, 128 * 128 * 16 * 2),
              "ss_128x128": (2, 128 * 128 * 16 * 2)}
MMA_LOADS = {"none": 0, "mufu": 1, "fma": 2}
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


def ex2_rate(warps: int = 16, iters: int = 4096, device="cuda") -> Dict[str, float]:
    """MUFU ex2.approx per SM cycle: one CTA per SM of `warps` warps, each
    thread 8 independent chains of `iters` exponentials (median CTA)."""
    dev = torch.device(device)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = torch.zeros(2 * sms, dtype=torch.int64, device=dev)
    s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for _ in range(2):   # the first launch warms up
        check(lib().mcs_micro_ex2(sms, warps, iters, ctypes.c_void_p(out.data_ptr()), s), "mcs_micro_ex2")
    torch.cuda.synchronize(dev)
    cyc = sorted(out[:sms].tolist())[sms // 2]
    n = warps * 32 * iters * 8
    return {"micro": "ex2", "warps": warps, "ex2_per_cta": n, "cycles": cyc, "ex2_per_sm_per_cycle": n / cyc}


def mma_rate(shape: str, load: str = "none", chains: int = 1, batches: int = 2048,
             device="cuda") -> Dict[str, float]:
    """Cycles per tcgen05 MMA of `shape` issued back to back by one warp per SM
    (one CTA per SM, median CTA) into `chains` interleaved accumulators, with
    the CTA's other warps keeping the MUFU or FMA pipe busy (`load`) or idle;
    FLOP per SM cycle beside it."""
    dev = torch.device(device)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    code, flop = MMA_SHAPES[shape]
    out = torch.zeros(3 * sms + 1, dtype=torch.int64, device=dev)
    s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for _ in range(2):
        check(lib().mcs_micro_mma(sms, code, batches, MMA_LOADS[load], chains, ctypes.c_void_p(out.data_ptr()), s),
              "mcs_micro_mma")
    torch.cuda.synchronize(dev)
    o = out[:3 * sms].view(sms, 3).cpu()
    if int(o[:, 2].sum()) != 0:
        raise RuntimeError("mcs_micro_mma: a completion wait ran out")
    cyc = sorted(o[:, 0].tolist())[sms // 2]
    n = int(o[0, 1])
    return {"micro": "mma", "shape": shape, "load": load, "chains": chains, "mmas": n, "cycles": cyc,
            "cycles_per_mma": cyc / n, "flop_per_sm_per_cycle": flop * n / cyc}

