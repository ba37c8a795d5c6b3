"""Sparse pooling and dense materialization on the GPU (through the C ABI) against the oracle.

Max pooling returns one of its inputs, so it is compared bit for bit.  Mean
pooling sums in fp32 and rounds once to the output type: per element
|err| <= u * |ref| + 2^-19 * max|x| (u = 2^-24, 2^-11, 2^-8 for fp32, fp16,
bf16; the second term bounds the fp32 sum of at most 32 terms and the
division).  Dense materialization is a copy and is compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.util import TORCH_DT, feats, rand_coords

pytestmark = pytest.mark.gpu

scv = pytest.importorskip("sparse_convolution_voxel_b200")

DTYPES = [torch.float32, torch.float16, torch.bfloat16]
UNIT = {torch.float32: 2.0 ** -24, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}
OPS = {"max": oracle.POOL_MAX, "avg": oracle.POOL_AVG}


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check_pool(got, ref, x64, dtype, op):
    got = got.double().cpu().numpy()
    assert got.shape == ref.shape
    if op == "max":
        assert np.array_equal(got, ref), "max pool differs"
        return
    bound = UNIT[dtype] * np.abs(ref) + 2.0 ** -19 * np.abs(x64).max(initial=0.0)
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"avg pool: worst err {err.max():.3e}"


def _subm(coords, ks=3):
    c = _dev(coords)
    km = scv.kernel_map(scv.hash_table(c), len(coords), c, scv.subm_geom(ks))
    return km, oracle.kmap(coords, coords, ks, 1, oracle.subm_pad(ks), oracle.SUBM)


def _strided(coords, ks, st_, pd):
    c = _dev(coords)
    g = scv.strided_geom(ks, st_, pd)
    coarse = scv.downsample(c, g).contiguous()
    km = scv.kernel_map(scv.hash_table(c), len(coords), coarse, g)
    rc = coarse.cpu().numpy()
    return km, oracle.kmap(coords, rc, ks, st_, pd, oracle.STRIDED)


# --------------------------------------------------------------------------- pooling
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("c", [8, 16, 64, 128])
@pytest.mark.parametrize("op", ["max", "avg"])
def test_subm_pool_small(dtype, c, op):
    rng = np.random.default_rng(c + 3)
    coords = rand_coords(rng, 700, -6, 6, 2)
    km, ref_nbr = _subm(coords)
    x, x64 = feats(len(coords), c, dtype, seed=c)
    st = scv.new_status()
    y = scv.sparse_pool(x, km, op, d_status=st)
    scv.check_status(st)
    _check_pool(y, oracle.pool(x64, ref_nbr, OPS[op]), x64, dtype, op)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("ks,st_,pd", [(2, 2, 0), (3, 2, 1), ((3, 2, 1), (2, 1, 3), (0, 1, 0))])
@pytest.mark.parametrize("op", ["max", "avg"])
def test_strided_pool(dtype, ks, st_, pd, op):
    rng = np.random.default_rng(17)
    coords = rand_coords(rng, 2500, -9, 9, 2)
    km, ref_nbr = _strided(coords, ks, st_, pd)
    x, x64 = feats(len(coords), 32, dtype, seed=5)
    y = scv.sparse_pool(x, km, op)
    _check_pool(y, oracle.pool(x64, ref_nbr, OPS[op]), x64, dtype, op)


@pytest.mark.parametrize("op", ["max", "avg"])
def test_pool_rows_without_neighbours_are_zero(op):
    """Transposed map with K < stride on one axis: most fine rows have no coarse neighbour."""
    rng = np.random.default_rng(23)
    coords = rand_coords(rng, 2500, -9, 9, 2)
    ks, st_, pd = (3, 2, 1), (2, 1, 3), (0, 1, 0)
    c = _dev(coords)
    coarse = scv.downsample(c, scv.strided_geom(ks, st_, pd)).contiguous()
    rc = coarse.cpu().numpy()
    up = scv.kernel_map(scv.hash_table(coarse), len(rc), c, scv.transposed_geom(ks, st_, pd))
    ref_up = oracle.kmap(rc, coords, ks, st_, pd, oracle.TRANSPOSED)
    assert (ref_up < 0).all(1).sum() >= 256
    x, x64 = feats(len(rc), 64, torch.float16, seed=29)
    y = scv.sparse_pool(x, up, op, out=torch.full((len(coords), 64), 3.0, dtype=torch.float16, device="cuda"))
    _check_pool(y, oracle.pool(x64, ref_up, OPS[op]), x64, torch.float16, op)


def test_pool_empty_and_errors():
    coords = np.zeros((0, 4), np.int32)
    km, _ = _subm(coords)
    y = scv.sparse_pool(torch.zeros((0, 16), device="cuda"), km, "max")
    torch.cuda.synchronize()
    assert y.shape == (0, 16)
    km, _ = _subm(rand_coords(np.random.default_rng(1), 50, 0, 5, 1))
    x = torch.zeros((50, 12), device="cuda")
    with pytest.raises(scv.LatticeError):
        scv.sparse_pool(x, km, "max")                     # C not a multiple of 8
    with pytest.raises(scv.LatticeError):
        scv.lat_sparse_pool(torch.zeros((50, 16), device="cuda"), km.c, 7, torch.empty((50, 16), device="cuda"))


@pytest.mark.parametrize("name,op", [("lidar_subm", "max"), ("lidar_subm", "avg"), ("images_subm", "avg")])
def test_pool_full_workloads(name, op):
    wl = synthetic.WORKLOADS[name]
    dtype = TORCH_DT[wl.dtype]
    coords = wl.coords()
    km, ref_nbr = _subm(coords, wl.ksize)
    x, x64 = feats(len(coords), wl.cin, dtype, seed=wl.seed)
    y = scv.sparse_pool(x, km, op)
    _check_pool(y, oracle.pool(x64, ref_nbr, OPS[op]), x64, dtype, op)


@pytest.mark.parametrize("op", ["max", "avg"])
def test_down_pool_full_workload(op):
    wl = synthetic.WORKLOADS["lidar_down_up"]
    coords = wl.coords()
    km, ref_nbr = _strided(coords, 2, 2, 0)
    x, x64 = feats(len(coords), wl.cin, torch.bfloat16, seed=wl.seed)
    y = scv.sparse_pool(x, km, op)
    _check_pool(y, oracle.pool(x64, ref_nbr, OPS[op]), x64, torch.bfloat16, op)


# --------------------------------------------------------------------------- dense materialization
@pytest.mark.parametrize("dtype", DTYPES)
def test_to_dense_small_with_rows_outside(dtype):
    rng = np.random.default_rng(11)
    coords = rand_coords(rng, 900, -7, 9, 3)
    x, x64 = feats(len(coords), 24, dtype, seed=11)
    origin, shape, batch = (-5, -7, -2), (12, 16, 9), 2
    ref, outside = oracle.to_dense(coords, x64, origin, shape, batch)
    assert outside > 0
    st = scv.new_status()
    grid = scv.to_dense(_dev(coords), x, origin, shape, batch, d_status=st,
                        out=torch.full((batch,) + shape + (24,), 5.0, dtype=dtype, device="cuda"))
    assert scv.lat_status_fetch(st) == 2                 # LAT_ERR_COORD_RANGE for the skipped rows
    assert np.array_equal(grid.double().cpu().numpy(), ref)


def test_to_dense_empty_and_errors():
    grid = scv.to_dense(torch.zeros((0, 4), dtype=torch.int32, device="cuda"), torch.zeros((0, 8), device="cuda"),
                        (0, 0, 0), (2, 3, 4), 1)
    assert grid.shape == (1, 2, 3, 4, 8) and torch.count_nonzero(grid).item() == 0
    with pytest.raises(scv.LatticeError):
        scv.to_dense(torch.zeros((1, 4), dtype=torch.int32, device="cuda"), torch.zeros((1, 8), device="cuda"),
                     (0, 0, 0), (0, 3, 4), 1)


def test_to_dense_lidar_sub_box():
    """Full-size lidar coordinates, a 256 x 256 x 41 box: most rows fall outside and are skipped."""
    wl = synthetic.WORKLOADS["lidar_subm"]
    coords = wl.coords()
    x, x64 = feats(len(coords), 16, torch.float16, seed=wl.seed)
    origin, shape, batch = (600, 500, 0), (256, 256, 41), 2
    ref, outside = oracle.to_dense(coords, x64, origin, shape, batch)
    assert 0 < outside < len(coords)
    grid = scv.to_dense(_dev(coords), x, origin, shape, batch)
    assert np.array_equal(grid.double().cpu().numpy(), ref)


def test_to_dense_images_full_grid():
    """The whole image batch as a dense grid (2.1 GB fp32): every row reads back from its
    cell and exactly the active cells are nonzero."""
    wl = synthetic.WORKLOADS["images_subm"]
    coords = wl.coords()
    x, _ = feats(len(coords), wl.cin, torch.float32, seed=wl.seed)
    c = _dev(coords)
    st = scv.new_status()
    grid = scv.to_dense(c, x, (0, 0, 0), (512, 512, 1), 256, d_status=st)
    scv.check_status(st)
    cl = c.long()
    assert torch.equal(grid[cl[:, 0], cl[:, 1], cl[:, 2], cl[:, 3]], x)
    assert int(torch.count_nonzero(grid.abs().amax(-1)).item()) == len(coords)
    del grid
