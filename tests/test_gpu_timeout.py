"""Bounded waits of the tensor-core kernels: a wait that runs out returns an
error status instead of hanging, and the context stays usable.

lat_set_wait_limit_ns(0) makes every barrier wait that is not complete at
its first test give up at once, so a tensor-core call gives up within
microseconds of its launch: the test checks that LAT_ERR_TIMEOUT reaches the
status word, restores the default limit, and checks that the next normal
call on the same stream matches the oracle.  Nothing faults, traps or hangs.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.util import assert_close, feats, rand_coords, weights, with_terms

pytestmark = pytest.mark.gpu

scv = pytest.importorskip("sparse_convolution_voxel_b200")

TIMEOUT = 512  # LAT_ERR_TIMEOUT


def _map(coords):
    c = torch.from_numpy(coords).cuda()
    st = scv.new_status()
    km = scv.kernel_map(scv.hash_table(c, 2.0, st), len(coords), c, scv.subm_geom(3), d_status=st)
    scv.check_status(st)
    return km


def _timed_out(run) -> int:
    """Status of `run(d_status)` made with a zero wait limit (the default limit is restored after)."""
    prev = scv.lat_set_wait_limit_ns(0)
    try:
        st = scv.new_status()
        run(st)
        return scv.lat_status_fetch(st)
    finally:
        assert scv.lat_set_wait_limit_ns(prev) == 0


def test_wait_limit_setter_returns_the_previous_limit():
    prev = scv.lat_set_wait_limit_ns(123)
    try:
        assert prev == 2_000_000_000
        assert scv.lat_set_wait_limit_ns(456) == 123
    finally:
        scv.lat_set_wait_limit_ns(prev)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_conv_wait_timeout_then_normal_call(dtype):
    rng = np.random.default_rng(11)
    coords = rand_coords(rng, 20000, -30, 30, 2)
    km = _map(coords)
    ref_nbr = oracle.kmap(coords, coords, 3, 1, 1, oracle.SUBM)
    x, x64 = feats(len(coords), 64, dtype, seed=11)
    w, w64 = weights(27, 64, 64, dtype, seed=11)
    status = _timed_out(lambda st: scv.conv_fwd(x, w, km, d_status=st))
    assert status & TIMEOUT, scv.lat_status_string(status)
    st = scv.new_status()
    y = scv.conv_fwd(x, w, km, d_status=st)
    scv.check_status(st, "the call after the timeout")
    assert_close(y.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr), dtype, "fwd after timeout")


def test_wgrad_wait_timeout_then_normal_call():
    dtype = torch.bfloat16
    rng = np.random.default_rng(12)
    coords = rand_coords(rng, 20000, -30, 30, 2)
    km = _map(coords)
    ref_nbr = oracle.kmap(coords, coords, 3, 1, 1, oracle.SUBM)
    x, x64 = feats(len(coords), 128, dtype, seed=12)
    g, g64 = feats(len(coords), 128, dtype, seed=12, stream=1)
    status = _timed_out(lambda st: scv.conv_wgrad(x, g, km, d_status=st))
    assert status & TIMEOUT, scv.lat_status_string(status)
    st = scv.new_status()
    dw = scv.conv_wgrad(x, g, km, d_status=st)
    scv.check_status(st, "the call after the timeout")
    assert_close(dw.double().cpu().numpy(), with_terms(oracle.conv_wgrad, x64, g64, ref_nbr), dtype,
                 "wgrad after timeout")
