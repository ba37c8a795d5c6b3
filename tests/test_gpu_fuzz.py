"""Seeded random small cases: the whole path on the GPU against the oracle.

Each case draws a row count, batch count, coordinate box (negative
coordinates included, dense or sparse), kernel shape, table ratio, dtype and
channel pair (8 to 128; the tensor-core shapes among them), then checks the
kernel map bit for bit and the forward, data-gradient and weight-gradient
passes within the dtype's tolerance.  Every fifth case also builds the
strided k2s2 support with its strided and transposed maps and checks them
and both convolutions over them.  Separate seeds put a repeated coordinate
in (LAT_ERR_DUPLICATE) or give the table too few slots (LAT_ERR_TABLE_FULL).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.util import assert_close, check_kmap, rand_coords, with_terms

pytestmark = pytest.mark.gpu

scv = pytest.importorskip("sparse_convolution_voxel_b200")

DTYPES = [torch.float32, torch.float16, torch.bfloat16]
CHANNELS = [8, 16, 24, 32, 64, 128]
KERNELS = [(3, 3, 3), (3, 3, 3), (3, 3, 1), (1, 1, 3), (3, 1, 5), (5, 3, 1), (1, 1, 1)]
N_CASES = 200


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _draw(rng, n, dt, c):
    t = torch.from_numpy(rng.standard_normal((n, c)).astype(np.float32)).to(dt)
    return t.cuda(), t.double().numpy()


def _case(seed):
    rng = np.random.default_rng(seed)
    batch = int(rng.integers(1, 4))
    span = int(rng.choice([6, 10, 20, 40]))
    lo = int(rng.integers(-span, span // 2))
    n = int(min(rng.integers(1, 1200), span ** 3))
    coords = rand_coords(rng, n, lo, lo + span, batch)
    ks = KERNELS[int(rng.integers(len(KERNELS)))]
    ratio = float(rng.choice([2.0, 4.0]))
    dt = DTYPES[int(rng.integers(3))]
    cin, cout = (int(rng.choice(CHANNELS)) for _ in range(2))
    return rng, coords, ks, ratio, dt, cin, cout


@pytest.mark.parametrize("block", range(4))
def test_fuzz_subm_path(block):
    for seed in range(block * N_CASES // 4, (block + 1) * N_CASES // 4):
        rng, coords, ks, ratio, dt, cin, cout = _case(seed)
        k3 = int(np.prod(ks))
        what = f"seed {seed}: n={len(coords)} ks={ks} {dt} {cin}->{cout}"
        c = _dev(coords)
        st = scv.new_status()
        km = scv.kernel_map(scv.hash_table(c, ratio, st), len(coords), c, scv.subm_geom(ks), d_status=st)
        scv.check_status(st, what)
        ref_nbr = oracle.kmap(coords, coords, ks, 1, oracle.subm_pad(ks), oracle.SUBM)
        check_kmap(km, ref_nbr)
        x, x64 = _draw(rng, len(coords), dt, cin)
        g, g64 = _draw(rng, len(coords), dt, cout)
        w_t = torch.from_numpy((rng.standard_normal((k3, cin, cout)) / np.sqrt(k3 * cin)).astype(np.float32)).to(dt)
        w, w64 = w_t.cuda(), w_t.double().numpy()
        y = scv.conv_fwd(x, w, km, d_status=st)
        dx = scv.conv_dgrad(g, w, km, True, d_status=st)
        dw = scv.conv_wgrad(x, g, km, d_status=st)
        scv.check_status(st, what)
        assert_close(y.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr), dt, what + " fwd")
        assert_close(dx.double().cpu().numpy(), with_terms(oracle.conv_dgrad, g64, w64, ref_nbr, len(coords)), dt,
                     what + " dgrad")
        assert_close(dw.double().cpu().numpy(), with_terms(oracle.conv_wgrad, x64, g64, ref_nbr), dt, what + " wgrad")
        if seed % 5:
            continue
        # strided k2s2 support, its strided and transposed maps, and both convolutions over them
        g2 = scv.strided_geom(2, 2, 0)
        coarse, parent = scv.downsample(c, g2, with_parent=True, d_status=st)
        ref_coarse = oracle.downsample(coords, 2, 2, 0)
        assert np.array_equal(coarse.cpu().numpy(), ref_coarse), what
        down, up = scv.maps_from_parent(c, parent.contiguous(), len(ref_coarse), g2, d_status=st)
        scv.check_status(st, what)
        ref_down = oracle.kmap(coords, ref_coarse, 2, 2, 0, oracle.STRIDED)
        ref_up = oracle.kmap(ref_coarse, coords, 2, 2, 0, oracle.TRANSPOSED)
        check_kmap(down, ref_down)
        check_kmap(up, ref_up)
        wd_t = torch.from_numpy((rng.standard_normal((8, cin, cout)) / np.sqrt(8 * cin)).astype(np.float32)).to(dt)
        yc = scv.conv_fwd(x, wd_t.cuda(), down, d_status=st)
        z = scv.conv_dgrad(yc, wd_t.cuda(), up, False, d_status=st)
        scv.check_status(st, what)
        yc64 = yc.double().cpu().numpy()
        assert_close(yc64, with_terms(oracle.conv_fwd, x64, wd_t.double().numpy(), ref_down), dt, what + " down")
        assert_close(z.double().cpu().numpy(),
                     with_terms(oracle.conv_dgrad, yc64, wd_t.double().numpy(), ref_down, len(coords)), dt,
                     what + " down dgrad")


@pytest.mark.parametrize("seed", range(8))
def test_fuzz_duplicate_rows_are_flagged(seed):
    rng = np.random.default_rng(1000 + seed)
    coords = rand_coords(rng, int(rng.integers(10, 500)), -8, 8, 2)
    dup = np.concatenate([coords, coords[rng.integers(len(coords), size=int(rng.integers(1, 5)))]])
    dup = np.ascontiguousarray(dup[rng.permutation(len(dup))])
    st = scv.new_status()
    scv.hash_table(_dev(dup), 2.0, st)
    assert scv.lat_status_fetch(st) & 4  # LAT_ERR_DUPLICATE


@pytest.mark.parametrize("seed", range(4))
def test_fuzz_full_table_is_flagged(seed):
    rng = np.random.default_rng(2000 + seed)
    n = int(rng.integers(65, 300))
    coords = rand_coords(rng, n, -10, 10, 1)
    table = torch.empty(2 * 64, dtype=torch.int64, device="cuda")   # 64 slots < n rows
    st = scv.new_status()
    scv.lat_hash_build(_dev(coords), table, st)
    assert scv.lat_status_fetch(st) & 8  # LAT_ERR_TABLE_FULL
