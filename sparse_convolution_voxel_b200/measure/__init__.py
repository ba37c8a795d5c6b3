"""Device peak probes for the benchmark's roofline (libmeasure.so, include/lattice_measure.h).

Not part of the convolution path.  ``ffma_peak`` measures the fp32 FMA rate
of the CUDA cores, the compute ceiling of the fp32 convolutions.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmeasure.so")
_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmeasure.so not built ({LIB_PATH}); run sparse_convolution_voxel_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        lib.lat_measure_ffma.restype = ctypes.c_int
        lib.lat_measure_ffma.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                         ctypes.c_float, ctypes.c_void_p]
        lib.lat_measure_ffma_flops.restype = ctypes.c_double
        lib.lat_measure_ffma_flops.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        _lib = lib
    return _lib


def ffma_peak(device: torch.device, reps: int = 5, iters: int = 32768) -> dict:
    """Best-of-`reps` fp32 FMA throughput (TFLOP/s) on `device`, CUDA events on
    the launching stream: 8 blocks of 256 threads per SM, each thread 64 FMAs
    per loop trip."""
    lib = load()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    blocks, threads = 8 * sms, 256
    out = torch.empty(blocks * threads, dtype=torch.float32, device=device)
    s = torch.cuda.current_stream(device)
    flops = lib.lat_measure_ffma_flops(blocks, threads, iters)

    def launch():
        rc = lib.lat_measure_ffma(ctypes.c_void_p(out.data_ptr()), blocks, threads, iters, 1.0000001, 1e-7,
                                  ctypes.c_void_p(s.cuda_stream))
        if rc:
            raise RuntimeError(f"lat_measure_ffma failed ({rc})")

    launch()
    torch.cuda.synchronize(device)
    best = None
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        launch()
        b.record(s)
        b.synchronize()
        ms = a.elapsed_time(b)
        best = ms if best is None else min(best, ms)
    if not torch.isfinite(out).all():
        raise RuntimeError("ffma probe produced non-finite values")
    return {"tflops": flops / (best * 1e-3) / 1e12, "ms": best, "flops": flops, "blocks": blocks,
            "threads": threads, "iters": iters}
