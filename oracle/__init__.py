"""CPU oracle for sparse convolution over coordinate-indexed voxels.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference leg of ``bench.py`` may import this package.
The product library never loads it, and it never loads the product.

The arithmetic lives in ``oracle.cpp`` (plain C++, ``std::unordered_map``
kernel map, fp64 accumulation, OpenMP over output rows); this module builds
it with g++ on first use and wraps it with ctypes.  Each wrapper names the
passage of the pages it follows; see ``oracle.cpp`` for the readings taken
where the pages are silent.

Parity pins (see ``tests/test_oracle_pins.py``): dense fp64 ``conv3d`` /
``conv_transpose3d`` on tiny grids, brute-force all-pairs neighbour search,
the two-voxel worked example of the docs page, the k=1 matmul special case,
adjoint identities and kernel-map symmetries.  No page prints a numeric
feature value, so no output is pinned to a printed number.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

SUBM, STRIDED, TRANSPOSED = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile ``oracle.cpp`` into ``liboracle.so`` (g++ -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i64, i32 = ctypes.c_int64, ctypes.c_int
            lib.orc_version.restype = i32
            lib.orc_pack_key.restype = ctypes.c_uint64
            lib.orc_pack_key.argtypes = [ctypes.c_int32] * 4
            lib.orc_kmap.restype = i32
            lib.orc_kmap.argtypes = [P, i64, P, i64, P, P, P, i32, P, i32]
            lib.orc_downsample.restype = i64
            lib.orc_downsample.argtypes = [P, i64, P, P, P, P, i64]
            lib.orc_upsample.restype = i64
            lib.orc_upsample.argtypes = [P, i64, P, P, P, P, i64]
            lib.orc_conv_fwd.restype = None
            lib.orc_conv_fwd.argtypes = [P, i64, i32, P, i32, P, i64, i32, P, i32]
            lib.orc_conv_dgrad.restype = None
            lib.orc_conv_dgrad.argtypes = [P, i64, i32, P, i32, P, i32, P, i64, i32]
            lib.orc_conv_wgrad.restype = None
            lib.orc_conv_wgrad.argtypes = [P, i32, P, i32, P, i64, i32, P, i32]
            lib.orc_pool.restype = None
            lib.orc_pool.argtypes = [P, i64, i32, P, i64, i32, i32, P]
            lib.orc_to_dense.restype = i64
            lib.orc_to_dense.argtypes = [P, i64, P, i32, P, P, i32, P]
            lib.orc_max_threads.restype = i32
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _triple(v) -> np.ndarray:
    if np.isscalar(v):
        v = (v, v, v)
    return _i32(v).reshape(3)


class OracleError(RuntimeError):
    pass


def max_threads() -> int:
    return _load().orc_max_threads()


def pack_key(b: int, x: int, y: int, z: int) -> int:
    """Packed 64-bit key; unsigned order equals lexicographic (b, x, y, z)."""
    return int(_load().orc_pack_key(b, x, y, z))


def kmap(in_coords, out_coords, ksize, stride=1, pad=0, mode=SUBM, nthreads=0) -> np.ndarray:
    """Kernel map as an (n_out, K^3) table of input rows (-1 = no neighbour).

    Coordinate query and kernel-map construction ("Migrating from
    TorchSparse", "What remains familiar" and "Sparse tensor expectations");
    support semantics per "Convolution mapping"."""
    inc, outc = _i32(in_coords).reshape(-1, 4), _i32(out_coords).reshape(-1, 4)
    ks, st, pd = _triple(ksize), _triple(stride), _triple(pad)
    k3 = int(np.prod(ks))
    nbr = np.empty((len(outc), k3), np.int32)
    rc = _load().orc_kmap(_ptr(inc), len(inc), _ptr(outc), len(outc), _ptr(ks), _ptr(st), _ptr(pd),
                          int(mode), _ptr(nbr), int(nthreads))
    if rc != 0:
        raise OracleError({1: "bad argument", 2: "coordinate out of range",
                           3: "duplicate coordinate"}.get(rc, rc))
    return nbr


def subm_pad(ksize) -> np.ndarray:
    """Submanifold padding (K-1)/2 per axis (odd kernel sizes)."""
    return (_triple(ksize) - 1) // 2


def downsample(coords, ksize, stride, pad=0) -> np.ndarray:
    """Coarse support of a strided Conv3d, sorted by packed key ("Convolution
    mapping": strided forward convolution creates a downsampled support)."""
    c = _i32(coords).reshape(-1, 4)
    ks, st, pd = _triple(ksize), _triple(stride), _triple(pad)
    cap = max(1, len(c) * int(np.prod(ks)))
    out = np.empty((cap, 4), np.int32)
    m = _load().orc_downsample(_ptr(c), len(c), _ptr(ks), _ptr(st), _ptr(pd), _ptr(out), cap)
    if m < 0:
        raise OracleError("downsample failed")
    return out[:m].copy()


def upsample(coords, ksize, stride, pad=0) -> np.ndarray:
    """Support generated by a transposed convolution (GenerativeConvTranspose3d):
    every s*q + off - pad, sorted by packed key ("Convolution mapping")."""
    c = _i32(coords).reshape(-1, 4)
    ks, st, pd = _triple(ksize), _triple(stride), _triple(pad)
    cap = max(1, len(c) * int(np.prod(ks)))
    out = np.empty((cap, 4), np.int32)
    m = _load().orc_upsample(_ptr(c), len(c), _ptr(ks), _ptr(st), _ptr(pd), _ptr(out), cap)
    if m < 0:
        raise OracleError("upsample failed")
    return out[:m].copy()


def pairs(nbr: np.ndarray):
    """Per-offset pair lists from a kernel-map table, in canonical order
    (offset ascending, output row ascending).  Returns (offsets[K^3+1],
    in_rows, out_rows)."""
    k3 = nbr.shape[1]
    ins, outs, off = [], [], [0]
    for k in range(k3):
        j = np.nonzero(nbr[:, k] >= 0)[0]
        ins.append(nbr[j, k])
        outs.append(j)
        off.append(off[-1] + len(j))
    cat = (lambda v: np.concatenate(v).astype(np.int32)) if k3 else (lambda v: np.zeros(0, np.int32))
    return np.asarray(off, np.int64), cat(ins), cat(outs)


def conv_fwd(x, w, nbr, nthreads=0) -> np.ndarray:
    """y[j] = sum_k x[nbr[j,k]] . W[k] in fp64 (gather-scatter definition)."""
    x, w, nbr = _f64(x), _f64(w), _i32(nbr)
    n_in, cin = x.shape
    k3, wcin, cout = w.shape
    assert wcin == cin and nbr.shape[1] == k3
    y = np.empty((len(nbr), cout), np.float64)
    _load().orc_conv_fwd(_ptr(x), n_in, cin, _ptr(w), cout, _ptr(nbr), len(nbr), k3, _ptr(y),
                         int(nthreads))
    return y


def conv_dgrad(dy, w, nbr, n_in, nthreads=0) -> np.ndarray:
    """dx[i] = sum over pairs (i, j, k) of dy[j] . W[k]^T in fp64."""
    dy, w, nbr = _f64(dy), _f64(w), _i32(nbr)
    k3, cin, cout = w.shape
    dx = np.empty((n_in, cin), np.float64)
    _load().orc_conv_dgrad(_ptr(dy), len(dy), cout, _ptr(w), cin, _ptr(nbr), k3, _ptr(dx), n_in,
                           int(nthreads))
    return dx


def conv_wgrad(x, dy, nbr, nthreads=0) -> np.ndarray:
    """dW[k] = sum over pairs (i, j) of offset k of x[i]^T dy[j] in fp64."""
    x, dy, nbr = _f64(x), _f64(dy), _i32(nbr)
    k3 = nbr.shape[1]
    dw = np.empty((k3, x.shape[1], dy.shape[1]), np.float64)
    _load().orc_conv_wgrad(_ptr(x), x.shape[1], _ptr(dy), dy.shape[1], _ptr(nbr), len(nbr), k3,
                           _ptr(dw), int(nthreads))
    return dw


POOL_MAX, POOL_AVG = 0, 1


def pool(x, nbr, op=POOL_MAX) -> np.ndarray:
    """Max (op 0) or mean (op 1) of x over each output row's neighbours; 0 if none.  fp64."""
    x, nbr = _f64(x), _i32(nbr)
    n_out, k3 = nbr.shape
    y = np.empty((n_out, x.shape[1]), np.float64)
    _load().orc_pool(_ptr(x), len(x), x.shape[1], _ptr(nbr), n_out, k3, int(op), _ptr(y))
    return y


def to_dense(coords, feats, origin, shape, batch):
    """(grid [batch, sx, sy, sz, C] fp64, number of rows outside the box)."""
    coords, feats = _i32(coords).reshape(-1, 4), _f64(feats)
    o, sh = _triple(origin), _triple(shape)
    grid = np.empty((int(batch), int(sh[0]), int(sh[1]), int(sh[2]), feats.shape[1]), np.float64)
    outside = _load().orc_to_dense(_ptr(coords), len(coords), _ptr(feats), feats.shape[1], _ptr(o), _ptr(sh),
                                   int(batch), _ptr(grid))
    return grid, int(outside)
