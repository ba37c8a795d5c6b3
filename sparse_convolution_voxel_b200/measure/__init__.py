"""Device peak probes for the benchmark's roofline (libmeasure.so, include/lattice_measure.h).

Not part of the convolution path.  ``ffma_peak`` measures the fp32 FMA rate
of the CUDA cores, the compute ceiling of the fp32 convolutions;
``gather_peak`` the rate of copying rows in random order, the access pattern
of the convolutions' gathered operands and scattered output rows.
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
        lib.lat_measure_gather.restype = ctypes.c_int
        lib.lat_measure_gather.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                           ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
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


def gather_peak(device: torch.device, n: int = 500_000, row_bytes: int = 256, reps: int = 5, seed: int = 0) -> dict:
    """Best-of-`reps` throughput (GB/s of rows read + written) of copying `n`
    rows of `row_bytes` bytes from random rows to random rows (two seeded
    permutations), 8 blocks of 256 threads per SM.  The 2 * n * row_bytes
    bytes exceed the L2 cache at the default sizes, and a 256 MB write flushes
    it before every timed launch."""
    lib = load()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    blocks = 8 * sms
    g = torch.Generator().manual_seed(seed)
    in_idx = torch.randperm(n, generator=g).to(torch.int32).to(device)
    out_idx = torch.randperm(n, generator=g).to(torch.int32).to(device)
    src = torch.empty(n * row_bytes // 4, dtype=torch.float32, device=device).uniform_()
    dst = torch.empty_like(src)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    s = torch.cuda.current_stream(device)

    def launch():
        rc = lib.lat_measure_gather(ctypes.c_void_p(src.data_ptr()), ctypes.c_void_p(in_idx.data_ptr()),
                                    ctypes.c_void_p(out_idx.data_ptr()), n, row_bytes,
                                    ctypes.c_void_p(dst.data_ptr()), blocks, ctypes.c_void_p(s.cuda_stream))
        if rc:
            raise RuntimeError(f"lat_measure_gather failed ({rc})")

    launch()
    torch.cuda.synchronize(device)
    rows_per_row = row_bytes // 4
    check = torch.randint(0, n, (64,), generator=g)
    for i in check.tolist():  # dst row out_idx[i] holds src row in_idx[i]
        o, r = int(out_idx[i]), int(in_idx[i])
        if not torch.equal(dst[o * rows_per_row:(o + 1) * rows_per_row], src[r * rows_per_row:(r + 1) * rows_per_row]):
            raise RuntimeError("gather probe copied the wrong rows")
    best = None
    for _ in range(reps):
        flush.add_(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        launch()
        b.record(s)
        b.synchronize()
        ms = a.elapsed_time(b)
        best = ms if best is None else min(best, ms)
    nbytes = 2 * n * row_bytes + 8 * n
    return {"gbs": nbytes / (best * 1e-3) / 1e9, "ms": best, "bytes": nbytes, "rows": n, "row_bytes": row_bytes,
            "blocks": blocks, "pattern": "random permutation read, random permutation write"}
