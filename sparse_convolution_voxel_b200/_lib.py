"""ctypes binding of liblattice.so (argument marshalling only).

Every function here converts torch tensors into device pointers and sizes,
passes the current CUDA stream, and calls the C entry point of the same name
declared in ``include/lattice.h``.  All work runs in the library's kernels;
there is no Python or CPU fallback: if the shared library is missing the
import fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblattice.so")

LAT_OK = 0
LAT_F32, LAT_F16, LAT_BF16 = 0, 1, 2
LAT_SUBM, LAT_STRIDED, LAT_TRANSPOSED = 0, 1, 2
LAT_OP_FWD, LAT_OP_DGRAD, LAT_OP_WGRAD = 0, 1, 2
LAT_TILE_ROWS = 128
LAT_POOL_MAX, LAT_POOL_AVG = 0, 1

STATUS_BITS = {
    1: "LAT_ERR_ARG", 2: "LAT_ERR_COORD_RANGE", 4: "LAT_ERR_DUPLICATE", 8: "LAT_ERR_TABLE_FULL",
    16: "LAT_ERR_CAPACITY", 32: "LAT_ERR_UNSUPPORTED", 64: "LAT_ERR_CUDA", 128: "LAT_ERR_WORKSPACE",
    256: "LAT_ERR_BAD_MAP", 512: "LAT_ERR_TIMEOUT",
}

# every symbol include/lattice.h declares
EXPORTS = [
    "lat_hash_bytes", "lat_hash_build", "lat_kmap_ws_bytes", "lat_kmap_query",
    "lat_downsample_ws_bytes", "lat_downsample_coords", "lat_downsample_coords_async", "lat_upsample_ws_bytes",
    "lat_upsample_coords", "lat_kmap_from_parent_ws_bytes",
    "lat_kmap_from_parent",
    "lat_sconv_ws_bytes", "lat_sconv_fwd",
    "lat_sconv_dgrad", "lat_sconv_wgrad", "lat_sconv_wgrad_static", "lat_sparse_pool", "lat_to_dense",
    "lat_status_fetch", "lat_status_string", "lat_version", "lat_set_wait_limit_ns",
]


class LatticeError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        names = [n for b, n in STATUS_BITS.items() if self.status & b] or [str(status)]
        super().__init__(f"{where}: {'|'.join(names)}")


class lat_geom(ctypes.Structure):
    _fields_ = [("ksize", ctypes.c_int32 * 3), ("stride", ctypes.c_int32 * 3),
                ("pad", ctypes.c_int32 * 3), ("mode", ctypes.c_int32)]


class lat_kmap(ctypes.Structure):
    _fields_ = [("nbr", ctypes.c_void_p), ("mask", ctypes.c_void_p), ("perm", ctypes.c_void_p),
                ("tile_mask", ctypes.c_void_p), ("pair_off", ctypes.c_void_p),
                ("pair_in", ctypes.c_void_p), ("pair_out", ctypes.c_void_p),
                ("pair_capacity", ctypes.c_int64), ("n_in", ctypes.c_int64),
                ("n_out", ctypes.c_int64), ("k3", ctypes.c_int32), ("mode", ctypes.c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load liblattice.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"liblattice.so not built ({LIB_PATH}); run sparse_convolution_voxel_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    G, K = ctypes.POINTER(lat_geom), ctypes.POINTER(lat_kmap)
    sig = {
        "lat_hash_bytes": (SZ, [I64, ctypes.c_float]),
        "lat_hash_build": (I32, [P, I64, P, SZ, P, P]),
        "lat_kmap_ws_bytes": (SZ, [I64, I32]),
        "lat_kmap_query": (I32, [P, SZ, P, G, K, P, SZ, P, P]),
        "lat_downsample_ws_bytes": (SZ, [I64, G]),
        "lat_downsample_coords": (I32, [P, I64, G, P, I64, ctypes.POINTER(I64), P, P, SZ, P, P]),
        "lat_downsample_coords_async": (I32, [P, I64, G, P, I64, P, P, P, SZ, P, P]),
        "lat_upsample_ws_bytes": (SZ, [I64, G]),
        "lat_upsample_coords": (I32, [P, I64, G, P, I64, ctypes.POINTER(I64), P, SZ, P, P]),
        "lat_kmap_from_parent_ws_bytes": (SZ, [I64, I64, I32]),
        "lat_kmap_from_parent": (I32, [P, P, G, K, K, P, SZ, P, P]),
        "lat_sconv_ws_bytes": (SZ, [I32, I32, I32, K, I32]),
        "lat_sconv_fwd": (I32, [P, I32, P, I32, K, P, I32, P, SZ, P, P]),
        "lat_sconv_dgrad": (I32, [P, I32, P, I32, K, I32, P, I32, P, SZ, P, P]),
        "lat_sconv_wgrad": (I32, [P, I32, P, I32, K, P, I32, P, SZ, P, P]),
        "lat_sconv_wgrad_static": (I32, [P, I32, P, I32, K, P, I32, P, P]),
        "lat_sparse_pool": (I32, [P, I32, K, I32, P, I32, P, P]),
        "lat_to_dense": (I32, [P, I64, P, I32, I32, ctypes.POINTER(I32), ctypes.POINTER(I32), I32, P, P, P]),
        "lat_status_fetch": (I32, [P, P]),
        "lat_status_string": (ctypes.c_char_p, [I32]),
        "lat_version": (I32, []),
        "lat_set_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("liblattice takes device tensors")
    if not t.is_contiguous():
        raise ValueError("liblattice takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_cur_dev = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream=None):
    """The CUDA stream handle: `stream` (a torch.cuda.Stream or a raw handle), else
    the current stream of the current device (read without building a Stream object,
    which costs a few microseconds per call)."""
    if stream is None:
        if _raw_stream is not None and _cur_dev is not None:
            return ctypes.c_void_p(_raw_stream(_cur_dev()))
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream if isinstance(stream, int) else stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != LAT_OK:
        raise LatticeError(rc, where)


_DTYPE_CODE = {torch.float32: LAT_F32, torch.float16: LAT_F16, torch.bfloat16: LAT_BF16}


def dtype_code(dt: torch.dtype) -> int:
    return _DTYPE_CODE[dt]


def make_geom(ksize, stride=1, pad=0, mode=LAT_SUBM) -> lat_geom:
    t = lambda v: (v, v, v) if isinstance(v, int) else tuple(v)
    g = lat_geom()
    g.ksize[:] = t(ksize)
    g.stride[:] = t(stride)
    g.pad[:] = t(pad)
    g.mode = int(mode)
    return g


# ----------------------------------------------------------------------------- entry points
def lat_hash_bytes(n: int, rsv_ratio: float = 2.0) -> int:
    return int(load().lat_hash_bytes(int(n), float(rsv_ratio)))


def lat_hash_build(coords: torch.Tensor, table: torch.Tensor, d_status: torch.Tensor | None = None, stream=None):
    rc = load().lat_hash_build(_ptr(coords), coords.shape[0], _ptr(table), table.numel() * table.element_size(),
                               _ptr(d_status), _stream(stream))
    _check(rc, "lat_hash_build")


def lat_kmap_ws_bytes(n_out: int, k3: int) -> int:
    return int(load().lat_kmap_ws_bytes(int(n_out), int(k3)))


def lat_kmap_query(table: torch.Tensor, out_coords: torch.Tensor, geom: lat_geom, kmap: lat_kmap,
                   ws: torch.Tensor | None, d_status: torch.Tensor | None = None, stream=None):
    rc = load().lat_kmap_query(_ptr(table), table.numel() * table.element_size(), _ptr(out_coords),
                               ctypes.byref(geom), ctypes.byref(kmap), _ptr(ws),
                               0 if ws is None else ws.numel() * ws.element_size(), _ptr(d_status),
                               _stream(stream))
    _check(rc, "lat_kmap_query")


def lat_downsample_ws_bytes(n_in: int, geom: lat_geom) -> int:
    return int(load().lat_downsample_ws_bytes(int(n_in), ctypes.byref(geom)))


def lat_downsample_coords(coords: torch.Tensor, geom: lat_geom, out_coords: torch.Tensor, ws: torch.Tensor | None,
                          d_status: torch.Tensor | None = None, stream=None, parent: torch.Tensor | None = None) -> int:
    n = ctypes.c_int64(0)
    rc = load().lat_downsample_coords(_ptr(coords), coords.shape[0], ctypes.byref(geom), _ptr(out_coords),
                                      out_coords.shape[0], ctypes.byref(n), _ptr(parent), _ptr(ws),
                                      0 if ws is None else ws.numel() * ws.element_size(), _ptr(d_status),
                                      _stream(stream))
    _check(rc, "lat_downsample_coords")
    return int(n.value)


def lat_downsample_coords_async(coords: torch.Tensor, geom: lat_geom, out_coords: torch.Tensor,
                                ws: torch.Tensor | None, n_out_host: torch.Tensor, d_status: torch.Tensor | None = None,
                                stream=None, parent: torch.Tensor | None = None) -> None:
    """Enqueue the downsample; n_out_host (pinned host int64[1]) receives the count (-1: use the blocking call)."""
    if n_out_host.device.type != "cpu" or n_out_host.dtype != torch.int64 or n_out_host.numel() < 1:
        raise ValueError("n_out_host must be a host int64 tensor")
    rc = load().lat_downsample_coords_async(_ptr(coords), coords.shape[0], ctypes.byref(geom), _ptr(out_coords),
                                            out_coords.shape[0], ctypes.c_void_p(n_out_host.data_ptr()), _ptr(parent),
                                            _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                            _ptr(d_status), _stream(stream))
    _check(rc, "lat_downsample_coords_async")


def lat_upsample_ws_bytes(n_in: int, geom: lat_geom) -> int:
    return int(load().lat_upsample_ws_bytes(int(n_in), ctypes.byref(geom)))


def lat_upsample_coords(coords: torch.Tensor, geom: lat_geom, out_coords: torch.Tensor, ws: torch.Tensor | None,
                        d_status: torch.Tensor | None = None, stream=None) -> int:
    n = ctypes.c_int64(0)
    rc = load().lat_upsample_coords(_ptr(coords), coords.shape[0], ctypes.byref(geom), _ptr(out_coords),
                                    out_coords.shape[0], ctypes.byref(n), _ptr(ws),
                                    0 if ws is None else ws.numel() * ws.element_size(), _ptr(d_status),
                                    _stream(stream))
    _check(rc, "lat_upsample_coords")
    return int(n.value)


def lat_kmap_from_parent_ws_bytes(n_fine: int, n_coarse: int, k3: int) -> int:
    return int(load().lat_kmap_from_parent_ws_bytes(int(n_fine), int(n_coarse), int(k3)))


def lat_kmap_from_parent(fine_coords: torch.Tensor, parent: torch.Tensor, geom: lat_geom, down: lat_kmap | None,
                         up: lat_kmap | None, ws: torch.Tensor | None, d_status: torch.Tensor | None = None,
                         stream=None):
    rc = load().lat_kmap_from_parent(_ptr(fine_coords), _ptr(parent), ctypes.byref(geom),
                                     None if down is None else ctypes.byref(down),
                                     None if up is None else ctypes.byref(up), _ptr(ws),
                                     0 if ws is None else ws.numel() * ws.element_size(), _ptr(d_status),
                                     _stream(stream))
    _check(rc, "lat_kmap_from_parent")


def lat_sconv_ws_bytes(op: int, cin: int, cout: int, kmap: lat_kmap, dtype: torch.dtype) -> int:
    return int(load().lat_sconv_ws_bytes(int(op), int(cin), int(cout), ctypes.byref(kmap), dtype_code(dtype)))


def _ws_args(ws):
    return _ptr(ws), (0 if ws is None else ws.numel() * ws.element_size())


def lat_sconv_fwd(x, w, kmap: lat_kmap, y, ws=None, d_status=None, stream=None):
    cin, cout = w.shape[1], w.shape[2]
    p, n = _ws_args(ws)
    rc = load().lat_sconv_fwd(_ptr(x), cin, _ptr(w), cout, ctypes.byref(kmap), _ptr(y), dtype_code(x.dtype), p, n,
                              _ptr(d_status), _stream(stream))
    _check(rc, "lat_sconv_fwd")


def lat_sconv_dgrad(dy, w, kmap: lat_kmap, flip_offsets: bool, dx, ws=None, d_status=None, stream=None):
    cin, cout = w.shape[1], w.shape[2]
    p, n = _ws_args(ws)
    rc = load().lat_sconv_dgrad(_ptr(dy), cout, _ptr(w), cin, ctypes.byref(kmap), int(bool(flip_offsets)), _ptr(dx),
                                dtype_code(dy.dtype), p, n, _ptr(d_status), _stream(stream))
    _check(rc, "lat_sconv_dgrad")


def lat_sconv_wgrad(x, dy, kmap: lat_kmap, dw, ws=None, d_status=None, stream=None):
    cin, cout = x.shape[1], dy.shape[1]
    p, n = _ws_args(ws)
    rc = load().lat_sconv_wgrad(_ptr(x), cin, _ptr(dy), cout, ctypes.byref(kmap), _ptr(dw), dtype_code(x.dtype), p, n,
                                _ptr(d_status), _stream(stream))
    _check(rc, "lat_sconv_wgrad")


def lat_sconv_wgrad_static(x, dy, kmap: lat_kmap, dw, d_status=None, stream=None):
    """Weight gradient with the library's own static scratch (no workspace argument)."""
    rc = load().lat_sconv_wgrad_static(_ptr(x), x.shape[1], _ptr(dy), dy.shape[1], ctypes.byref(kmap), _ptr(dw),
                                       dtype_code(x.dtype), _ptr(d_status), _stream(stream))
    _check(rc, "lat_sconv_wgrad_static")


def lat_sparse_pool(x, kmap: lat_kmap, op: int, y, d_status=None, stream=None):
    rc = load().lat_sparse_pool(_ptr(x), x.shape[1], ctypes.byref(kmap), int(op), _ptr(y), dtype_code(x.dtype),
                                _ptr(d_status), _stream(stream))
    _check(rc, "lat_sparse_pool")


def lat_to_dense(coords, feats, origin, shape, batch: int, out, d_status=None, stream=None):
    o = (ctypes.c_int32 * 3)(*[int(v) for v in origin])
    sh = (ctypes.c_int32 * 3)(*[int(v) for v in shape])
    rc = load().lat_to_dense(_ptr(coords), coords.shape[0], _ptr(feats), feats.shape[1], dtype_code(feats.dtype), o,
                             sh, int(batch), _ptr(out), _ptr(d_status), _stream(stream))
    _check(rc, "lat_to_dense")


def lat_status_fetch(d_status: torch.Tensor, stream=None) -> int:
    return int(load().lat_status_fetch(_ptr(d_status), _stream(stream)))


def lat_status_string(status: int) -> str:
    return load().lat_status_string(int(status)).decode()


def lat_version() -> int:
    return int(load().lat_version())


def lat_set_wait_limit_ns(ns: int) -> int:
    """Limit of every barrier wait in the tensor-core kernels (ns); returns the previous limit."""
    return int(load().lat_set_wait_limit_ns(int(ns)))
