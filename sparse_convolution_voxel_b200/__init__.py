"""Sparse convolution over coordinate-indexed voxels on B200 (sm_100a).

The compute lives in ``liblattice.so`` (C ABI, ``include/lattice.h``).  This
package is its Python face: ``_lib`` binds every C entry point under the same
name, and the helpers below only allocate device buffers with torch and call
those entry points in order.  There is no CPU path.

Typical SubmConv3d forward (Torch Lattice docs, "Convolution mapping"):

    table = hash_table(coords)                       # lat_hash_build
    kmap = kernel_map(table, coords, coords, subm_geom(3))   # lat_kmap_query
    y = conv_fwd(x, w, kmap)                         # lat_sconv_fwd
"""
from __future__ import annotations

import torch

from ._lib import (  # noqa: F401  (re-exported C entry points and constants)
    EXPORTS, LAT_BF16, LAT_F16, LAT_F32, LAT_OK, LAT_OP_DGRAD, LAT_OP_FWD, LAT_OP_WGRAD, LAT_STRIDED, LAT_SUBM,
    LAT_POOL_AVG, LAT_POOL_MAX, LAT_TILE_ROWS, LAT_TRANSPOSED, LIB_PATH, LatticeError, lat_downsample_coords, lat_downsample_coords_async, lat_downsample_ws_bytes, lat_geom,
    lat_upsample_coords, lat_upsample_ws_bytes,
    lat_hash_build, lat_hash_bytes, lat_kmap, lat_kmap_from_parent, lat_kmap_from_parent_ws_bytes, lat_kmap_query,
    lat_kmap_ws_bytes, lat_sconv_dgrad, lat_sconv_fwd, lat_sparse_pool, lat_to_dense,
    lat_sconv_wgrad, lat_sconv_wgrad_static, lat_sconv_ws_bytes, lat_set_wait_limit_ns, lat_status_fetch,
    lat_status_string, lat_version, load, make_geom,
)

__all__ = [
    "KernelMap", "Workspace", "hash_table", "kernel_map", "downsample", "downsample_async", "PendingDownsample",
    "upsample", "maps_from_parent", "conv_fwd", "conv_dgrad", "conv_wgrad", "sparse_pool", "to_dense",
    "subm_geom", "strided_geom", "target_geom", "transposed_geom", "check_status", "new_status",
] + EXPORTS


def subm_geom(ksize=3):
    ks = (ksize,) * 3 if isinstance(ksize, int) else tuple(ksize)
    return make_geom(ks, 1, tuple((k - 1) // 2 for k in ks), LAT_SUBM)


def strided_geom(ksize=2, stride=2, pad=0):
    return make_geom(ksize, stride, pad, LAT_STRIDED)


def target_geom(ksize=3):
    """TargetConv3d: the stride-1 relation evaluated at caller output coordinates."""
    ks = (ksize,) * 3 if isinstance(ksize, int) else tuple(ksize)
    return make_geom(ks, 1, tuple((k - 1) // 2 for k in ks), LAT_STRIDED)


def transposed_geom(ksize=2, stride=2, pad=0):
    return make_geom(ksize, stride, pad, LAT_TRANSPOSED)


def new_status(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_status(d_status: torch.Tensor, where: str = "device status"):
    """Synchronise and raise LatticeError if a kernel flagged an error."""
    v = lat_status_fetch(d_status)
    if v:
        raise LatticeError(v, where)


class Workspace:
    """Grow-only device scratch buffer handed to the *_ws arguments."""

    def __init__(self, device="cuda"):
        self.device = torch.device(device)
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor | None:
        if nbytes <= 0:
            return None
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=self.device)
        return self.buf


class KernelMap:
    """Device buffers of one lat_kmap (see include/lattice.h) plus the C struct."""

    def __init__(self, n_in: int, n_out: int, k3: int, device="cuda", pair_capacity: int | None = None):
        dev = torch.device(device)
        cap = n_out * k3 if pair_capacity is None else int(pair_capacity)
        ntiles = (n_out + LAT_TILE_ROWS - 1) // LAT_TILE_ROWS
        self.n_in, self.n_out, self.k3 = int(n_in), int(n_out), int(k3)
        self.nbr = torch.empty(max(1, k3 * n_out), dtype=torch.int32, device=dev)
        self.mask = torch.empty(max(1, n_out), dtype=torch.int32, device=dev)
        self.perm = torch.empty(max(1, n_out), dtype=torch.int32, device=dev)
        self.tile_mask = torch.empty(max(1, ntiles), dtype=torch.int32, device=dev)
        self.pair_off = torch.empty(k3 + 1, dtype=torch.int64, device=dev)
        self.pair_in = torch.empty(max(1, cap), dtype=torch.int32, device=dev)
        self.pair_out = torch.empty(max(1, cap), dtype=torch.int32, device=dev)
        c = lat_kmap()
        c.nbr, c.mask, c.perm, c.tile_mask = (self.nbr.data_ptr(), self.mask.data_ptr(), self.perm.data_ptr(),
                                              self.tile_mask.data_ptr())
        c.pair_off, c.pair_in, c.pair_out = self.pair_off.data_ptr(), self.pair_in.data_ptr(), self.pair_out.data_ptr()
        c.pair_capacity, c.n_in, c.n_out, c.k3 = cap, self.n_in, self.n_out, self.k3
        self.c = c

    @property
    def ntiles(self) -> int:
        return (self.n_out + LAT_TILE_ROWS - 1) // LAT_TILE_ROWS

    def nbr_table(self) -> torch.Tensor:
        """(n_out, k3) view of the offset-major neighbour table."""
        return self.nbr[: self.k3 * self.n_out].view(self.k3, self.n_out).t()


def hash_table(coords: torch.Tensor, rsv_ratio: float = 4.0, d_status=None, stream=None) -> torch.Tensor:
    nbytes = lat_hash_bytes(coords.shape[0], rsv_ratio)
    if nbytes == 0:
        raise LatticeError(1, "lat_hash_bytes")
    table = torch.empty(nbytes // 8, dtype=torch.int64, device=coords.device)
    lat_hash_build(coords, table, d_status, stream)
    return table


def kernel_map(table: torch.Tensor, n_in: int, out_coords: torch.Tensor, geom: lat_geom, ws: Workspace | None = None,
               d_status=None, pair_capacity=None, stream=None) -> KernelMap:
    k3 = geom.ksize[0] * geom.ksize[1] * geom.ksize[2]
    km = KernelMap(n_in, out_coords.shape[0], k3, out_coords.device, pair_capacity)
    ws = ws or Workspace(out_coords.device)
    lat_kmap_query(table, out_coords, geom, km.c, ws.get(lat_kmap_ws_bytes(km.n_out, k3)), d_status, stream)
    return km


def upsample(coords: torch.Tensor, geom: lat_geom, ws: Workspace | None = None, d_status=None,
             capacity: int | None = None, stream=None) -> torch.Tensor:
    """Support a GenerativeConvTranspose3d generates from `coords` (geom: LAT_TRANSPOSED),
    in canonical order (synchronises)."""
    n = coords.shape[0]
    k3 = geom.ksize[0] * geom.ksize[1] * geom.ksize[2]
    cap = n * k3 if capacity is None else int(capacity)
    out = torch.empty((max(1, cap), 4), dtype=torch.int32, device=coords.device)
    ws = ws or Workspace(coords.device)
    m = lat_upsample_coords(coords, geom, out, ws.get(lat_upsample_ws_bytes(n, geom)), d_status, stream)
    return out[:m]


class PendingDownsample:
    """A downsample enqueued by downsample_async; result() waits for the coarse row count."""

    def __init__(self, coords, geom, out, parent, host, event, ws_t, d_status, stream):
        self._args = (coords, geom, out, parent, ws_t, d_status, stream)
        self._host, self._event = host, event

    def count(self) -> int:
        """Coarse row count (waits for the stream to pass the downsample)."""
        coords, geom, out, parent, ws_t, d_status, stream = self._args
        self._event.synchronize()
        m = int(self._host[0])
        if m < 0:  # coarse fields too wide for the bitmap: the blocking radix-sort path
            m = lat_downsample_coords(coords, geom, out, ws_t, d_status, stream, parent=parent)
            self._host[0] = m
        elif m > out.shape[0]:
            raise LatticeError(16, "lat_downsample_coords_async")
        return m

    def result(self):
        """(coarse coords, parent) like downsample(..., with_parent=True), or the coords alone."""
        m = self.count()
        coords, _, out, parent, _, _, _ = self._args
        return (out[:m], parent[:coords.shape[0]]) if parent is not None else out[:m]


def downsample_async(coords: torch.Tensor, geom: lat_geom, ws: Workspace | None = None, d_status=None,
                     capacity: int | None = None, stream=None, with_parent: bool = False) -> PendingDownsample:
    """Enqueue the coarse support (and parents) without waiting for the row count."""
    n = coords.shape[0]
    per = 1
    for a in range(3):
        per *= -(-geom.ksize[a] // geom.stride[a])
    cap = n * per if capacity is None else int(capacity)
    out = torch.empty((max(1, cap), 4), dtype=torch.int32, device=coords.device)
    parent = torch.empty(max(1, n), dtype=torch.int32, device=coords.device) if with_parent else None
    ws = ws or Workspace(coords.device)
    ws_t = ws.get(lat_downsample_ws_bytes(n, geom))
    host = torch.empty(1, dtype=torch.int64, pin_memory=True)
    lat_downsample_coords_async(coords, geom, out, ws_t, host, d_status, stream, parent=parent)
    event = torch.cuda.Event()
    event.record(stream if stream is not None else torch.cuda.current_stream())
    return PendingDownsample(coords, geom, out, parent, host, event, ws_t, d_status, stream)


def downsample(coords: torch.Tensor, geom: lat_geom, ws: Workspace | None = None, d_status=None,
               capacity: int | None = None, stream=None, with_parent: bool = False):
    """Coarse support of a strided Conv3d in canonical order (synchronises).
    With with_parent=True also returns the coarse row of every input row."""
    n = coords.shape[0]
    per = 1
    for a in range(3):
        per *= -(-geom.ksize[a] // geom.stride[a])
    cap = n * per if capacity is None else int(capacity)
    out = torch.empty((max(1, cap), 4), dtype=torch.int32, device=coords.device)
    parent = torch.empty(max(1, n), dtype=torch.int32, device=coords.device) if with_parent else None
    ws = ws or Workspace(coords.device)
    m = lat_downsample_coords(coords, geom, out, ws.get(lat_downsample_ws_bytes(n, geom)), d_status, stream,
                              parent=parent)
    return (out[:m], parent[:n]) if with_parent else out[:m]


def maps_from_parent(fine_coords: torch.Tensor, parent: torch.Tensor, n_coarse: int, geom: lat_geom,
                     ws: Workspace | None = None, d_status=None, stream=None):
    """(strided map, transposed map) of a ksize == stride, pad == 0 Conv3d from parent rows."""
    n = fine_coords.shape[0]
    k3 = geom.ksize[0] * geom.ksize[1] * geom.ksize[2]
    down = KernelMap(n, n_coarse, k3, fine_coords.device)
    up = KernelMap(n_coarse, n, k3, fine_coords.device)
    ws = ws or Workspace(fine_coords.device)
    lat_kmap_from_parent(fine_coords, parent, geom, down.c, up.c, ws.get(lat_kmap_from_parent_ws_bytes(n, n_coarse, k3)),
                         d_status, stream)
    return down, up


def conv_fwd(x, w, kmap: KernelMap, ws: Workspace | None = None, d_status=None, out=None, stream=None):
    y = out if out is not None else torch.empty((kmap.n_out, w.shape[2]), dtype=x.dtype, device=x.device)
    ws = ws or Workspace(x.device)
    lat_sconv_fwd(x, w, kmap.c, y, ws.get(lat_sconv_ws_bytes(LAT_OP_FWD, w.shape[1], w.shape[2], kmap.c, x.dtype)),
                  d_status, stream)
    return y


def conv_dgrad(dy, w, kmap: KernelMap, flip_offsets: bool, ws: Workspace | None = None, d_status=None, out=None,
               stream=None):
    dx = out if out is not None else torch.empty((kmap.n_out, w.shape[1]), dtype=dy.dtype, device=dy.device)
    ws = ws or Workspace(dy.device)
    lat_sconv_dgrad(dy, w, kmap.c, flip_offsets, dx,
                    ws.get(lat_sconv_ws_bytes(LAT_OP_DGRAD, w.shape[1], w.shape[2], kmap.c, dy.dtype)), d_status,
                    stream)
    return dx


def conv_wgrad(x, dy, kmap: KernelMap, ws: Workspace | None = None, d_status=None, out=None, stream=None):
    dw = out if out is not None else torch.empty((kmap.k3, x.shape[1], dy.shape[1]), dtype=torch.float32,
                                                 device=x.device)
    ws = ws or Workspace(x.device)
    lat_sconv_wgrad(x, dy, kmap.c, dw,
                    ws.get(lat_sconv_ws_bytes(LAT_OP_WGRAD, x.shape[1], dy.shape[1], kmap.c, x.dtype)), d_status,
                    stream)
    return dw


def sparse_pool(x, kmap: KernelMap, op: str = "max", d_status=None, out=None, stream=None):
    """Max or mean of x over each output row's neighbours in ``kmap`` (0 where it has none)."""
    codes = {"max": LAT_POOL_MAX, "avg": LAT_POOL_AVG, "mean": LAT_POOL_AVG}
    if op not in codes:
        raise ValueError(f"pooling op must be one of {sorted(codes)}, not {op!r}")
    code = codes[op]
    y = out if out is not None else torch.empty((kmap.n_out, x.shape[1]), dtype=x.dtype, device=x.device)
    lat_sparse_pool(x, kmap.c, code, y, d_status, stream)
    return y


def to_dense(coords, feats, origin, shape, batch: int, d_status=None, out=None, stream=None):
    """Channels-last dense grid [batch, shape[0], shape[1], shape[2], C] over the box at ``origin``."""
    size = (int(batch), int(shape[0]), int(shape[1]), int(shape[2]), feats.shape[1])
    grid = out if out is not None else torch.empty(size, dtype=feats.dtype, device=feats.device)
    lat_to_dense(coords, feats, origin, shape, batch, grid, d_status, stream)
    return grid
