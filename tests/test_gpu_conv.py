"""Sparse convolution passes on the GPU (through the C ABI) against the fp64 oracle.

Tolerances: fp32 max|err| <= 1e-5 * max|ref|; fp16 / bf16 max|err| <=
2e-2 * max|ref| (both normwise over the whole output).  Cases span several
128-row tiles with a ragged tail, every dtype, the channel counts of the
five workloads, and the full-size workloads themselves.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.util import TORCH_DT, assert_close, check_kmap, feats, rand_coords, weights, with_terms

pytestmark = pytest.mark.gpu

scv = pytest.importorskip("sparse_convolution_voxel_b200")

DTYPES = [torch.float32, torch.float16, torch.bfloat16]


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _subm_map(coords, ks=(3, 3, 3)):
    c = _dev(coords)
    st = scv.new_status()
    km = scv.kernel_map(scv.hash_table(c, 2.0, st), len(coords), c, scv.subm_geom(ks), d_status=st)
    scv.check_status(st)
    return km, oracle.kmap(coords, coords, ks, 1, oracle.subm_pad(ks), oracle.SUBM)


# --------------------------------------------------------------------------- forward
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("cin,cout", [(8, 32), (16, 16), (64, 64), (64, 128), (128, 64), (128, 128)])
def test_subm_fwd_small(dtype, cin, cout):
    rng = np.random.default_rng(cin * 1000 + cout)
    coords = rand_coords(rng, 700, -6, 6, 2)            # 1400 rows: 10 full tiles + a ragged tail
    km, ref_nbr = _subm_map(coords)
    x, x64 = feats(len(coords), cin, dtype, seed=1)
    w, w64 = weights(27, cin, cout, dtype, seed=1)
    st = scv.new_status()
    y = scv.conv_fwd(x, w, km, d_status=st)
    scv.check_status(st)
    assert_close(y.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr), dtype, "fwd")


@pytest.mark.parametrize("dtype", DTYPES)
def test_fwd_rows_without_neighbours_are_zero(dtype):
    coords = np.array([[0, 0, 0, 0], [0, 10, 10, 10], [1, 0, 0, 0]], np.int32)
    km, ref_nbr = _subm_map(coords)
    x, x64 = feats(3, 16, dtype, seed=2)
    w = torch.zeros((27, 16, 16), dtype=dtype, device="cuda")
    y = scv.conv_fwd(x, w, km, out=torch.full((3, 16), 7.0, dtype=dtype, device="cuda"))
    assert torch.count_nonzero(y).item() == 0


def test_fwd_empty_input():
    coords = np.zeros((0, 4), np.int32)
    km, _ = _subm_map(coords)
    x = torch.zeros((0, 16), device="cuda")
    w = torch.zeros((27, 16, 16), device="cuda")
    y = scv.conv_fwd(x, w, km)
    torch.cuda.synchronize()
    assert y.shape == (0, 16)


@pytest.mark.parametrize("name", ["subm_small", "lidar_subm", "images_subm"])
def test_subm_fwd_full_workloads(name):
    wl = synthetic.WORKLOADS[name]
    dtype = TORCH_DT[wl.dtype]
    coords = wl.coords()
    km, ref_nbr = _subm_map(coords, wl.ksize)
    k3 = int(np.prod(wl.ksize))
    x, x64 = feats(len(coords), wl.cin, dtype, seed=wl.seed)
    w, w64 = weights(k3, wl.cin, wl.cout, dtype, seed=wl.seed)
    y = scv.conv_fwd(x, w, km)
    assert_close(y.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr), dtype, name)


def test_down_up_full_workload():
    wl = synthetic.WORKLOADS["lidar_down_up"]
    dtype = TORCH_DT[wl.dtype]
    coords = wl.coords()
    c = _dev(coords)
    g = scv.strided_geom(2, 2, 0)
    coarse = scv.downsample(c, g).contiguous()
    ref_coarse = oracle.downsample(coords, 2, 2, 0)
    down = scv.kernel_map(scv.hash_table(c), len(coords), coarse, g)
    up = scv.kernel_map(scv.hash_table(coarse), len(ref_coarse), c, scv.transposed_geom(2, 2, 0))
    x, x64 = feats(len(coords), 64, dtype, seed=3)
    wd, wd64 = weights(8, 64, 128, dtype, seed=3)
    wu, wu64 = weights(8, 128, 64, dtype, seed=3, stream=1)
    y = scv.conv_fwd(x, wd, down)
    ref_y = with_terms(oracle.conv_fwd, x64, wd64, oracle.kmap(coords, ref_coarse, 2, 2, 0, oracle.STRIDED))
    assert_close(y.double().cpu().numpy(), ref_y, dtype, "down")
    # the up pass consumes the GPU's rounded coarse features, as the layer chain would
    y64 = y.double().cpu().numpy()
    z = scv.conv_fwd(y, wu, up)
    ref_z = with_terms(oracle.conv_fwd, y64, wu64, oracle.kmap(ref_coarse, coords, 2, 2, 0, oracle.TRANSPOSED))
    assert_close(z.double().cpu().numpy(), ref_z, dtype, "up")


# --------------------------------------------------------------------------- backward
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("cin,cout", [(16, 16), (64, 64), (128, 128), (64, 128)])
def test_subm_dgrad_wgrad_small(dtype, cin, cout):
    rng = np.random.default_rng(cin + 7 * cout)
    coords = rand_coords(rng, 600, -6, 6, 2)
    km, ref_nbr = _subm_map(coords)
    x, x64 = feats(len(coords), cin, dtype, seed=5)
    w, w64 = weights(27, cin, cout, dtype, seed=5)
    g, g64 = feats(len(coords), cout, dtype, seed=5, stream=1)
    st = scv.new_status()
    dx = scv.conv_dgrad(g, w, km, flip_offsets=True, d_status=st)
    dw = scv.conv_wgrad(x, g, km, d_status=st)
    scv.check_status(st)
    assert_close(dx.double().cpu().numpy(), with_terms(oracle.conv_dgrad, g64, w64, ref_nbr, len(coords)),
                 dtype, "dgrad")
    assert_close(dw.double().cpu().numpy(), with_terms(oracle.conv_wgrad, x64, g64, ref_nbr), dtype, "wgrad")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_strided_and_transposed_backward(dtype):
    rng = np.random.default_rng(17)
    coords = rand_coords(rng, 1500, -10, 10, 2)
    c = _dev(coords)
    g2 = scv.strided_geom(2, 2, 0)
    coarse = scv.downsample(c, g2).contiguous()
    rc = coarse.cpu().numpy()
    down = scv.kernel_map(scv.hash_table(c), len(coords), coarse, g2)
    up = scv.kernel_map(scv.hash_table(coarse), len(rc), c, scv.transposed_geom(2, 2, 0))
    ref_down = oracle.kmap(coords, rc, 2, 2, 0, oracle.STRIDED)
    ref_up = oracle.kmap(rc, coords, 2, 2, 0, oracle.TRANSPOSED)
    x, x64 = feats(len(coords), 64, dtype, seed=9)
    w, w64 = weights(8, 64, 128, dtype, seed=9)
    gy, gy64 = feats(len(rc), 128, dtype, seed=9, stream=2)
    # strided Conv3d: dgrad walks the transposed map, wgrad uses the forward pairs
    dx = scv.conv_dgrad(gy, w, up, flip_offsets=False)
    assert_close(dx.double().cpu().numpy(), with_terms(oracle.conv_dgrad, gy64, w64, ref_down, len(coords)),
                 dtype, "down dgrad")
    dw = scv.conv_wgrad(x, gy, down)
    assert_close(dw.double().cpu().numpy(), with_terms(oracle.conv_wgrad, x64, gy64, ref_down), dtype, "down wgrad")
    # ConvTranspose3d: dgrad walks the strided map
    wt, wt64 = weights(8, 128, 64, dtype, seed=9, stream=3)
    gz, gz64 = feats(len(coords), 64, dtype, seed=9, stream=4)
    dyc = scv.conv_dgrad(gz, wt, down, flip_offsets=False)
    assert_close(dyc.double().cpu().numpy(), with_terms(oracle.conv_dgrad, gz64, wt64, ref_up, len(rc)),
                 dtype, "up dgrad")
    dwt = scv.conv_wgrad(gy, gz, up)
    assert_close(dwt.double().cpu().numpy(), with_terms(oracle.conv_wgrad, gy64, gz64, ref_up), dtype, "up wgrad")


def test_training_step_full_workload():
    wl = synthetic.WORKLOADS["lidar_train"]
    dtype = TORCH_DT[wl.dtype]
    coords = wl.coords()
    km, ref_nbr = _subm_map(coords)
    x, x64 = feats(len(coords), 128, dtype, seed=5)
    w, w64 = weights(27, 128, 128, dtype, seed=5)
    g, g64 = feats(len(coords), 128, dtype, seed=5, stream=1)
    y = scv.conv_fwd(x, w, km)
    dx = scv.conv_dgrad(g, w, km, flip_offsets=True)
    dw = scv.conv_wgrad(x, g, km)
    assert_close(y.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr), dtype, "fwd")
    assert_close(dx.double().cpu().numpy(), with_terms(oracle.conv_dgrad, g64, w64, ref_nbr, len(coords)),
                 dtype, "dgrad")
    assert_close(dw.double().cpu().numpy(), with_terms(oracle.conv_wgrad, x64, g64, ref_nbr), dtype, "wgrad")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
def test_transposed_fwd_with_rows_without_neighbours(dtype):
    """K < stride on one axis: two thirds of the fine rows have no coarse neighbour, so
    whole 128-row tiles have an empty offset set and must be written as zeros."""
    rng = np.random.default_rng(23)
    coords = rand_coords(rng, 2500, -9, 9, 2)
    ks, st_, pd = (3, 2, 1), (2, 1, 3), (0, 1, 0)
    c = _dev(coords)
    g = scv.strided_geom(ks, st_, pd)
    coarse = scv.downsample(c, g).contiguous()
    rc = coarse.cpu().numpy()
    up = scv.kernel_map(scv.hash_table(coarse), len(rc), c, scv.transposed_geom(ks, st_, pd))
    ref_up = oracle.kmap(rc, coords, ks, st_, pd, oracle.TRANSPOSED)
    assert (ref_up < 0).all(1).sum() >= 256
    x, x64 = feats(len(rc), 64, dtype, seed=29)
    w, w64 = weights(6, 64, 64, dtype, seed=29)
    z = scv.conv_fwd(x, w, up, out=torch.full((len(coords), 64), 3.0, dtype=dtype, device="cuda"))
    assert_close(z.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_up), dtype, "transposed fwd")


@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
def test_target_conv(dtype):
    """TargetConv3d: a stride-1 strided geometry evaluated at caller coordinates."""
    rng = np.random.default_rng(43)
    coords = rand_coords(rng, 1200, -8, 8, 2)
    targets = rand_coords(rng, 1000, -9, 9, 2)
    c, tg = _dev(coords), _dev(targets)
    km = scv.kernel_map(scv.hash_table(c), len(coords), tg, scv.target_geom(3))
    ref_nbr = oracle.kmap(coords, targets, 3, 1, 1, oracle.STRIDED)
    check_kmap(km, ref_nbr)
    x, x64 = feats(len(coords), 64, dtype, seed=47)
    w, w64 = weights(27, 64, 64, dtype, seed=47)
    y = scv.conv_fwd(x, w, km)
    assert_close(y.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr), dtype, "target conv")


# --------------------------------------------------------------------------- generative stride-1 Conv3d
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
@pytest.mark.parametrize("ks", [3, (3, 3, 1)])
def test_generative_stride1_conv(dtype, ks):
    """A stride-1 Conv3d that is not submanifold grows the support by its
    footprint (migration page, "Convolution mapping": generative convs create a
    new support): support = every q whose window holds an input, then the
    strided relation, forward and data gradient against the oracle."""
    rng = np.random.default_rng(23)
    coords = rand_coords(rng, 700, -8, 8, 2)
    if ks != 3:
        coords[:, 3] = 0
        coords = np.unique(coords, axis=0)
        coords = coords[rng.permutation(len(coords))]
    pad = (1, 1, 1) if ks == 3 else (1, 1, 0)
    g = scv.strided_geom(ks, 1, pad)
    c = _dev(coords)
    st = scv.new_status()
    grown = scv.downsample(c, g, d_status=st).contiguous()
    ref_grown = oracle.downsample(coords, ks, 1, pad)
    assert np.array_equal(grown.cpu().numpy(), ref_grown)
    assert len(ref_grown) > len(coords)              # the support grew
    km = scv.kernel_map(scv.hash_table(c, 2.0, st), len(coords), grown, g, d_status=st)
    ref_nbr = oracle.kmap(coords, ref_grown, ks, 1, pad, oracle.STRIDED)
    check_kmap(km, ref_nbr)
    k3 = ref_nbr.shape[1]
    cin, cout = (16, 32) if dtype == torch.float32 else (64, 64)
    x, x64 = feats(len(coords), cin, dtype, seed=9)
    w, w64 = weights(k3, cin, cout, dtype, seed=9)
    y = scv.conv_fwd(x, w, km, d_status=st)
    assert_close(y.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr), dtype, "generative fwd")
    # data gradient through the opposite relation (grown rows -> input rows)
    gy, gy64 = feats(len(ref_grown), cout, dtype, seed=9, stream=1)
    back = scv.kernel_map(scv.hash_table(grown, 2.0, st), len(ref_grown), c, scv.transposed_geom(ks, 1, pad),
                          d_status=st)
    dx = scv.conv_dgrad(gy, w, back, flip_offsets=False, d_status=st)
    scv.check_status(st)
    assert_close(dx.double().cpu().numpy(), with_terms(oracle.conv_dgrad, gy64, w64, ref_nbr, len(coords)), dtype,
                 "generative dgrad")


# --------------------------------------------------------------------------- GenerativeConvTranspose3d
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("ks,st_,pd", [(2, 2, 0), (3, 2, 1)])
def test_generative_transposed_conv(dtype, ks, st_, pd):
    """GenerativeConvTranspose3d: generated fine support, the transposed relation
    from the coarse table to it, forward and data gradient against the oracle."""
    rng = np.random.default_rng(41 + ks)
    coarse = rand_coords(rng, 400, -6, 6, 2)
    c = _dev(coarse)
    g = scv.transposed_geom(ks, st_, pd)
    st = scv.new_status()
    fine = scv.upsample(c, g, d_status=st).contiguous()
    ref_fine = oracle.upsample(coarse, ks, st_, pd)
    assert np.array_equal(fine.cpu().numpy(), ref_fine)
    km = scv.kernel_map(scv.hash_table(c, 2.0, st), len(coarse), fine, g, d_status=st)
    ref_nbr = oracle.kmap(coarse, ref_fine, ks, st_, pd, oracle.TRANSPOSED)
    check_kmap(km, ref_nbr)
    assert np.all((ref_nbr >= 0).any(1))             # every generated row has a source
    k3 = ref_nbr.shape[1]
    cin, cout = (128, 64) if dtype == torch.bfloat16 else (32, 16)
    x, x64 = feats(len(coarse), cin, dtype, seed=13)
    w, w64 = weights(k3, cin, cout, dtype, seed=13)
    y = scv.conv_fwd(x, w, km, d_status=st)
    assert_close(y.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr),
                 dtype, "generative transposed fwd")
    # data gradient back to the coarse rows through the strided relation
    gy, gy64 = feats(len(ref_fine), cout, dtype, seed=13, stream=1)
    back = scv.kernel_map(scv.hash_table(fine, 2.0, st), len(ref_fine), c, scv.strided_geom(ks, st_, pd),
                          d_status=st)
    dx = scv.conv_dgrad(gy, w, back, flip_offsets=False, d_status=st)
    scv.check_status(st)
    assert_close(dx.double().cpu().numpy(), with_terms(oracle.conv_dgrad, gy64, w64, ref_nbr, len(coarse)), dtype,
                 "generative transposed dgrad")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("cout", [64, 128])
def test_tc_fwd_output_16_byte_aligned(dtype, cout):
    """The tensor-core epilogue stores 32-byte slices when the output is 32-byte
    aligned and stages them otherwise: an output view 16 bytes into a buffer
    gives the same bits as an aligned one."""
    rng = np.random.default_rng(61)
    coords = rand_coords(rng, 900, -7, 7, 2)
    km, ref_nbr = _subm_map(coords)
    x, x64 = feats(len(coords), 64, dtype, seed=61)
    w, w64 = weights(27, 64, cout, dtype, seed=61)
    y_al = scv.conv_fwd(x, w, km)
    flat = torch.full((len(coords) * cout + 8,), 7.0, dtype=dtype, device="cuda")
    y_off = flat[8:].view(len(coords), cout)
    assert y_off.data_ptr() % 32 == 16
    scv.conv_fwd(x, w, km, out=y_off)
    torch.cuda.synchronize()
    assert torch.equal(y_al, y_off)
    assert torch.all(flat[:8] == 7.0)
    assert_close(y_al.double().cpu().numpy(), with_terms(oracle.conv_fwd, x64, w64, ref_nbr), dtype, "aligned fwd")
