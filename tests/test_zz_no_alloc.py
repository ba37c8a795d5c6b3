"""The weight gradient that uses the library's static scratch instead of a caller buffer.

Callers that cannot allocate device memory (code running under stream
capture without memory nodes, real-time loops that must not call cudaMalloc
or cudaFree once running, hosts whose allocator belongs to another runtime)
use lat_sconv_wgrad_static.  It must give the same dW as lat_sconv_wgrad,
call after call, since every call reuses the one static array.  This file
is named so pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.util import assert_close, feats, rand_coords, with_terms

pytestmark = pytest.mark.gpu

scv = pytest.importorskip("sparse_convolution_voxel_b200")


def _map(coords):
    c = torch.from_numpy(coords).cuda()
    st = scv.new_status()
    km = scv.kernel_map(scv.hash_table(c, 2.0, st), len(coords), c, scv.subm_geom(3), d_status=st)
    scv.check_status(st)
    return km


def _static_wgrad(x, g, km, cin, cout, dtype):
    dw = torch.full((27, cin, cout), float("nan"), dtype=torch.float32, device="cuda")
    st = scv.new_status()
    rc = scv.load().lat_sconv_wgrad_static(ctypes.c_void_p(x.data_ptr()), cin, ctypes.c_void_p(g.data_ptr()), cout,
                                           ctypes.byref(km.c), ctypes.c_void_p(dw.data_ptr()),
                                           scv._lib.dtype_code(dtype), ctypes.c_void_p(st.data_ptr()),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, scv.lat_status_string(rc)
    scv.check_status(st)
    return dw


@pytest.mark.parametrize("dtype,cin,cout", [(torch.float16, 64, 64), (torch.bfloat16, 128, 128),
                                            (torch.float32, 16, 32), (torch.float32, 8, 32)])
def test_static_scratch_wgrad_matches_oracle_twice(dtype, cin, cout):
    """Two calls in a row, each against the fp64 oracle; on the shapes where
    lat_sconv_wgrad also runs on the CUDA cores (fp32 here) both entry points
    run the same kernels in the same order, so their dW must agree bit for bit."""
    scv.load()
    rng = np.random.default_rng(cin + cout)
    coords = rand_coords(rng, 4000, -12, 12, 2)
    km = _map(coords)
    ref_nbr = oracle.kmap(coords, coords, 3, 1, 1, oracle.SUBM)
    x, x64 = feats(len(coords), cin, dtype, seed=41)
    g, g64 = feats(len(coords), cout, dtype, seed=41, stream=1)
    ref = with_terms(oracle.conv_wgrad, x64, g64, ref_nbr)
    outs = []
    for _ in range(2):
        dw = _static_wgrad(x, g, km, cin, cout, dtype)
        outs.append(dw)
        assert_close(dw.double().cpu().numpy(), ref, dtype, "static-scratch wgrad")
    assert torch.equal(outs[0], outs[1]), "the second call differs from the first"
    if dtype == torch.float32:
        assert torch.equal(outs[0], scv.conv_wgrad(x, g, km)), "differs from lat_sconv_wgrad on CUDA-core shapes"


def test_static_scratch_wgrad_rejects_problems_above_its_limit():
    scv.load()
    rng = np.random.default_rng(3)
    coords = rand_coords(rng, 200, 0, 8)
    km = _map(coords)
    x = torch.zeros((len(coords), 256), dtype=torch.float16, device="cuda")
    dw = torch.zeros((27, 256, 256), dtype=torch.float32, device="cuda")
    # (296 + 27) partials of 256 x 256 fp32 need 84.7 MB, above the 32 MiB array
    rc = scv.load().lat_sconv_wgrad_static(ctypes.c_void_p(x.data_ptr()), 256, ctypes.c_void_p(x.data_ptr()), 256,
                                           ctypes.byref(km.c), ctypes.c_void_p(dw.data_ptr()), 1, None, None)
    assert rc == 128                                  # LAT_ERR_WORKSPACE, nothing enqueued
    # the limit is in channels only: 128 x 192 fits whatever the pair capacity
    big = scv.lat_kmap.from_buffer_copy(km.c)
    big.pair_capacity = 50_000_000
    assert scv.lat_sconv_ws_bytes(2, 128, 192, big, torch.float32) <= 32 << 20
