"""The C-ABI library loads and exports every symbol include/lattice.h declares (CPU only).

Only host-side behaviour is exercised here: size queries, status strings and
argument checks that return before anything is enqueued on a GPU.
"""
import ctypes
import os
import re

import pytest

import sparse_convolution_voxel_b200 as scv
from sparse_convolution_voxel_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sparse_convolution_voxel_b200 import build
    build.build()
    return _lib.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "lattice.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lat_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_measure_library_exports_every_declared_symbol(lib):
    """libmeasure.so (include/lattice_measure.h): the probes bench.py uses for
    its rooflines; bad arguments return 1 before anything is launched."""
    from sparse_convolution_voxel_b200 import measure
    text = open(os.path.join(ROOT, "include", "lattice_measure.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = sorted(set(re.findall(r"\b(lat_[a-z0-9_]+)\s*\(", text)))
    assert names == ["lat_measure_ffma", "lat_measure_ffma_flops", "lat_measure_gather"]
    m = measure.load()
    for name in names:
        assert hasattr(m, name), name
    P = ctypes.c_void_p
    assert m.lat_measure_gather(None, P(16), None, 10, 256, P(16), 8, None) == 1      # no source
    assert m.lat_measure_gather(P(16), P(16), None, 10, 24, P(16), 8, None) == 1      # row not 16-byte multiple
    assert m.lat_measure_gather(P(8), P(16), None, 10, 256, P(16), 8, None) == 1      # misaligned source
    assert m.lat_measure_gather(P(16), P(16), None, 0, 256, P(16), 8, None) == 0      # nothing to copy
    assert m.lat_measure_ffma(None, 8, 256, 1, 1.0, 0.0, None) == 1
    assert m.lat_measure_ffma_flops(2, 64, 3) == 2.0 * 64 * 3 * 2 * 64


def test_size_queries(lib):
    assert scv.lat_hash_bytes(1000, 2.0) == 16 * 2048
    assert scv.lat_hash_bytes(10, 2.0) == 16 * 64
    assert scv.lat_hash_bytes(1000, 0.5) == 0
    assert scv.lat_kmap_ws_bytes(200_000, 27) > 0
    assert scv.lat_kmap_ws_bytes(10, 33) == 0
    g = scv.strided_geom(2, 2, 0)
    assert scv.lat_downsample_ws_bytes(1000, g) > 0
    assert scv.lat_downsample_ws_bytes(1000, scv.subm_geom(3)) == 0


def test_status_strings_and_version(lib):
    assert scv.lat_status_string(0) == "ok"
    assert "duplicate" in scv.lat_status_string(4)
    assert scv.lat_version() >= 100


def test_host_argument_checks_return_without_gpu(lib):
    P = ctypes.c_void_p
    # null coords with n > 0
    assert lib.lat_hash_build(None, 10, P(16), 16 * 64, None, None) == 1
    # table size not a power of two
    assert lib.lat_hash_build(P(16), 10, P(16), 16 * 65, None, None) == 1
    km = _lib.lat_kmap()
    km.k3 = 27
    km.n_out = 10
    km.n_in = 10
    bad = scv.make_geom(3, 1, 0, scv.LAT_SUBM)       # submanifold pad must be (K-1)/2
    assert lib.lat_kmap_query(P(16), 16 * 64, P(16), ctypes.byref(bad), ctypes.byref(km), None, 0, None, None) == 1
    km.k3 = 40
    assert lib.lat_sconv_fwd(P(16), 16, P(16), 16, ctypes.byref(km), P(16), 0, None, 0, None, None) == 1
    km.k3 = 27
    # channel counts must be multiples of 8
    assert lib.lat_sconv_fwd(P(16), 12, P(16), 16, ctypes.byref(km), P(16), 0, None, 0, None, None) == 1


def test_conv_workspace_query_and_check_without_gpu(lib):
    """Tensor-core fwd / dgrad need the 256-byte tile-counter workspace; the
    CUDA-core shapes need none; too little workspace fails before any launch."""
    P = ctypes.c_void_p
    km = _lib.lat_kmap()
    km.k3, km.n_out, km.n_in = 27, 10, 10
    km.nbr, km.perm, km.tile_mask = P(16), P(16), P(16)
    f32, f16 = 0, 1
    assert lib.lat_sconv_ws_bytes(0, 64, 64, ctypes.byref(km), f16) == 256
    assert lib.lat_sconv_ws_bytes(1, 64, 128, ctypes.byref(km), f16) == 256
    assert lib.lat_sconv_ws_bytes(0, 64, 64, ctypes.byref(km), f32) == 0
    assert lib.lat_sconv_ws_bytes(0, 16, 32, ctypes.byref(km), f16) == 0
    assert lib.lat_sconv_fwd(P(16), 64, P(16), 64, ctypes.byref(km), P(16), f16, None, 0, None, None) == 128
    assert lib.lat_sconv_fwd(P(16), 64, P(16), 64, ctypes.byref(km), P(16), f16, P(256), 16, None, None) == 128
    assert lib.lat_sconv_dgrad(P(16), 128, P(16), 64, ctypes.byref(km), 1, P(16), f16, None, 0, None, None) == 128


def test_pool_and_dense_argument_checks_without_gpu(lib):
    """Every rejected argument returns LAT_ERR_ARG before anything is enqueued."""
    P = ctypes.c_void_p
    km = _lib.lat_kmap()
    km.k3, km.n_out, km.n_in = 27, 10, 10
    km.nbr, km.mask = P(16), P(16)
    ok = (P(16), 16, ctypes.byref(km), 0, P(32), 0, None, None)
    assert lib.lat_sparse_pool(None, 16, None, 0, P(32), 0, None, None) == 1          # no map
    assert lib.lat_sparse_pool(P(16), 12, *ok[2:]) == 1                                # C % 8
    assert lib.lat_sparse_pool(*ok[:3], 2, *ok[4:]) == 1                               # unknown op
    assert lib.lat_sparse_pool(P(24), *ok[1:]) == 1                                    # x not 16-byte aligned
    km.k3 = 33
    assert lib.lat_sparse_pool(*ok) == 1
    km.k3, km.mask = 27, None
    assert lib.lat_sparse_pool(*ok) == 1                                               # no mask
    i3 = ctypes.c_int32 * 3
    o, sh = i3(0, 0, 0), i3(4, 4, 4)
    assert lib.lat_to_dense(P(16), 5, P(16), 8, 0, o, sh, 0, P(16), None, None) == 1   # batch 0
    assert lib.lat_to_dense(P(16), 5, P(16), 8, 0, o, i3(4, 0, 4), 1, P(16), None, None) == 1
    assert lib.lat_to_dense(P(16), 5, P(16), 10, 0, o, sh, 1, P(16), None, None) == 1  # C % 8
    assert lib.lat_to_dense(None, 5, P(16), 8, 0, o, sh, 1, P(16), None, None) == 1
    assert lib.lat_to_dense(P(8), 5, P(16), 8, 0, o, sh, 1, P(16), None, None) == 1    # coords alignment
    assert lib.lat_to_dense(P(16), 5, P(16), 8, 3, o, sh, 1, P(16), None, None) == 1   # dtype


def test_binding_rejects_host_tensors(lib):
    """The binding only marshals device pointers: a host tensor fails loudly
    (no CPU fallback) before anything reaches the library."""
    import torch
    km = scv.KernelMap.__new__(scv.KernelMap)  # the struct alone; no device buffers needed
    km.c = _lib.lat_kmap()
    km.c.k3, km.c.n_out, km.c.n_in = 27, 4, 4
    x = torch.zeros((4, 16))
    with pytest.raises(ValueError, match="device tensors"):
        _lib.lat_sparse_pool(x, km.c, 0, torch.zeros((4, 16)))
    with pytest.raises(ValueError, match="device tensors"):
        _lib.lat_sconv_fwd(x, torch.zeros((27, 16, 16)), km.c, torch.zeros((4, 16)))
    with pytest.raises(ValueError, match="device tensors"):
        _lib.lat_hash_build(torch.zeros((4, 4), dtype=torch.int32), torch.zeros(64, dtype=torch.int64))


def test_pool_helper_rejects_unknown_op(lib):
    import torch
    km = scv.KernelMap.__new__(scv.KernelMap)
    km.c = _lib.lat_kmap()
    km.n_out = 4
    with pytest.raises(ValueError, match="pooling op"):
        scv.sparse_pool(torch.zeros((4, 16)), km, "sum", out=torch.zeros((4, 16)))
