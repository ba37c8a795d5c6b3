"""Pins the CPU oracle to things other than itself (CPU only).

* the two-voxel worked example printed on the docs page;
* brute-force all-pairs neighbour search (the O(n^2) search SparsePixels'
  abstract describes) against the hashed kernel map;
* dense fp64 ``torch.nn.functional.conv3d`` / ``conv_transpose3d`` on tiny
  grids, read at the active / generated sites, and ``torch.autograd`` for the
  backward passes;
* closed forms and special cases: kernel size 1 equals a dense matmul, an
  isolated voxel sees only the centre weight, adjoint identities, offset
  symmetry of the submanifold map, one parent per input for k = s.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import SUBM, STRIDED, TRANSPOSED


def _rand_coords(rng, n, lo, hi, batch=1):
    """n unique rows per batch sample, coordinates in [lo, hi)."""
    rows = []
    span = hi - lo
    for b in range(batch):
        cells = rng.choice(span ** 3, size=n, replace=False)
        x, r = np.divmod(cells, span * span)
        y, z = np.divmod(r, span)
        rows.append(np.stack([np.full(n, b), x + lo, y + lo, z + lo], 1))
    c = np.concatenate(rows).astype(np.int32)
    return c[rng.permutation(len(c))]


def _brute_kmap(in_c, out_c, ks, st, pd, mode):
    """All-pairs search: for every (output, input) pair decide the offset."""
    ks, st, pd = np.asarray(ks), np.asarray(st), np.asarray(pd)
    k3 = int(np.prod(ks))
    nbr = -np.ones((len(out_c), k3), np.int32)
    for j, q in enumerate(out_c):
        for i, p in enumerate(in_c):
            if p[0] != q[0]:
                continue
            if mode == TRANSPOSED:     # output fine q, input coarse p: s*p + off - pad == q
                off = q[1:] - st * p[1:] + pd
            else:                      # input at s*q + off - pad
                off = p[1:] - st * q[1:] + pd
            if np.all(off >= 0) and np.all(off < ks):
                k = (off[0] * ks[1] + off[1]) * ks[2] + off[2]
                assert nbr[j, k] == -1
                nbr[j, k] = i
    return nbr


def _densify(coords, feats, shape, origin):
    B = int(coords[:, 0].max()) + 1
    C = feats.shape[1]
    g = torch.zeros((B, C) + tuple(shape), dtype=torch.float64)
    c = torch.as_tensor(coords, dtype=torch.long)
    o = torch.as_tensor(origin, dtype=torch.long)
    g[c[:, 0], :, c[:, 1] - o[0], c[:, 2] - o[1], c[:, 3] - o[2]] = torch.as_tensor(feats)
    return g


def _read(grid, coords, origin):
    c = torch.as_tensor(coords, dtype=torch.long)
    o = torch.as_tensor(origin, dtype=torch.long)
    return grid[c[:, 0], :, c[:, 1] - o[0], c[:, 2] - o[1], c[:, 3] - o[2]]


def _dense_weight(w, ks):
    """(K^3, Cin, Cout) -> conv3d weight (Cout, Cin, Kx, Ky, Kz)."""
    k3, cin, cout = w.shape
    return torch.as_tensor(w).reshape(ks[0], ks[1], ks[2], cin, cout).permute(4, 3, 0, 1, 2).contiguous()


# --------------------------------------------------------------------------- worked example
def test_two_voxel_worked_example(golden_dir):
    coords = np.array([[0, 4, 8, 2], [0, 5, 8, 2]], np.int32)
    nbr = oracle.kmap(coords, coords, 3, 1, 1, SUBM)
    off, pin, pout = oracle.pairs(nbr)
    got = set()
    for k in range(27):
        for e in range(off[k], off[k + 1]):
            got.add((k, int(pout[e]), int(pin[e])))
    want = set()
    for line in open(os.path.join(golden_dir, "two_voxel_subm_k3.txt")):
        if line.startswith("#") or not line.strip():
            continue
        k, dx, dy, dz, j, i = map(int, line.split())
        assert k == ((dx + 1) * 3 + dy + 1) * 3 + dz + 1
        want.add((k, j, i))
    assert got == want
    assert len(pin) == 4


# --------------------------------------------------------------------------- key packing + hash fn
def test_packed_key_order_is_lexicographic():
    rng = np.random.default_rng(0)
    rows = np.concatenate([
        rng.integers(-32768, 32768, (400, 4)),
        rng.integers(-3, 3, (200, 4)),
    ])
    rows[:, 0] = np.abs(rows[:, 0]) % 65535
    keys = [oracle.pack_key(*map(int, r)) for r in rows]
    by_key = sorted(range(len(rows)), key=lambda i: keys[i])
    by_lex = sorted(range(len(rows)), key=lambda i: tuple(rows[i]))
    assert [tuple(rows[i]) for i in by_key] == [tuple(rows[i]) for i in by_lex]
    assert oracle.pack_key(65535, 0, 0, 0) == 2 ** 64 - 1       # out of range
    assert oracle.pack_key(0, 32768, 0, 0) == 2 ** 64 - 1
    assert oracle.pack_key(0, -32768, -32768, -32768) == 0


# --------------------------------------------------------------------------- kernel maps
@pytest.mark.parametrize("seed", range(4))
def test_subm_kmap_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    c = _rand_coords(rng, 60, -4, 5, batch=2)
    ks = (3, 3, 3) if seed % 2 == 0 else (5, 3, 1)
    pd = oracle.subm_pad(ks)
    got = oracle.kmap(c, c, ks, 1, pd, SUBM)
    assert np.array_equal(got, _brute_kmap(c, c, ks, (1, 1, 1), pd, SUBM))


@pytest.mark.parametrize("ks,st,pd", [((2, 2, 2), (2, 2, 2), (0, 0, 0)),
                                      ((3, 3, 3), (2, 2, 2), (1, 1, 1)),
                                      ((3, 2, 1), (2, 1, 3), (0, 1, 0))])
def test_strided_and_transposed_kmap_match_brute_force(ks, st, pd):
    rng = np.random.default_rng(7)
    c = _rand_coords(rng, 70, -5, 6, batch=2)
    coarse = oracle.downsample(c, ks, st, pd)
    got = oracle.kmap(c, coarse, ks, st, pd, STRIDED)
    assert np.array_equal(got, _brute_kmap(c, coarse, ks, st, pd, STRIDED))
    gotT = oracle.kmap(coarse, c, ks, st, pd, TRANSPOSED)
    assert np.array_equal(gotT, _brute_kmap(coarse, c, ks, st, pd, TRANSPOSED))
    # every coarse row has at least one input in its window; when the kernel
    # covers the stride on every axis, every input also reaches a coarse row
    assert np.all((got >= 0).any(1))
    if all(k >= s for k, s in zip(ks, st)):
        assert np.all((gotT >= 0).any(1))


def test_downsample_support_equals_nonempty_dense_windows():
    rng = np.random.default_rng(3)
    c = _rand_coords(rng, 150, 0, 12, batch=2)
    for ks, st in [((2, 2, 2), (2, 2, 2)), ((3, 3, 3), (2, 2, 2))]:
        coarse = oracle.downsample(c, ks, st, 0)
        # pad by 2 (a multiple of the stride) so windows hanging off either edge are seen:
        # dense output o then covers the window of coarse q = o - 1
        occ = _densify(c, np.ones((len(c), 1)), (16, 16, 16), (-2, -2, -2))
        win = torch.nn.functional.conv3d(occ, torch.ones((1, 1) + ks, dtype=torch.float64), stride=st)
        nz = torch.nonzero(win[:, 0] > 0).numpy().astype(np.int32)
        nz[:, 1:] -= 1
        nz = nz[np.lexsort(nz.T[::-1])]
        assert np.array_equal(coarse, nz)


def test_subm_kmap_invariants():
    rng = np.random.default_rng(11)
    c = _rand_coords(rng, 300, 0, 10, batch=3)
    nbr = oracle.kmap(c, c, 3, 1, 1, SUBM)
    n = len(c)
    assert np.array_equal(nbr[:, 13], np.arange(n))             # centre: every row, itself
    for k in range(27):                                          # M_-d is M_d with in/out swapped
        j = np.nonzero(nbr[:, k] >= 0)[0]
        i = nbr[j, k]
        assert np.array_equal(nbr[i, 26 - k], j)
        assert (nbr[:, k] >= 0).sum() == (nbr[:, 26 - k] >= 0).sum()


def test_downsample_k_equals_s_gives_one_parent_per_input():
    rng = np.random.default_rng(5)
    c = _rand_coords(rng, 400, -6, 7, batch=2)
    coarse = oracle.downsample(c, 2, 2, 0)
    nbrT = oracle.kmap(coarse, c, 2, 2, 0, TRANSPOSED)
    assert np.all((nbrT >= 0).sum(1) == 1)
    nbr = oracle.kmap(c, coarse, 2, 2, 0, STRIDED)
    assert (nbr >= 0).sum() == len(c)
    got = np.sort(nbr[nbr >= 0])
    assert np.array_equal(got, np.arange(len(c)))
    # parent is floor(p / 2) per axis
    parent = coarse[nbrT.max(1)]
    assert np.array_equal(parent[:, 1:], np.floor_divide(c[:, 1:], 2))


def test_kmap_errors():
    c = np.array([[0, 1, 1, 1], [0, 1, 1, 1]], np.int32)
    with pytest.raises(oracle.OracleError):
        oracle.kmap(c, c, 3, 1, 1, SUBM)
    c = np.array([[0, 40000, 1, 1]], np.int32)
    with pytest.raises(oracle.OracleError):
        oracle.kmap(c, c, 3, 1, 1, SUBM)


def test_edge_of_key_range_queries_are_absent():
    c = np.array([[0, 32767, 0, 0], [0, -32768, 0, 0], [1, 32766, 0, 0]], np.int32)
    nbr = oracle.kmap(c, c, 3, 1, 1, SUBM)
    assert np.array_equal(nbr[:, 13], [0, 1, 2])
    assert nbr[0, 22] == -1 and nbr[1, 4] == -1                  # x+1 / x-1 leave the range
    assert (nbr >= 0).sum() == 3                                 # no wrap-around, no batch mixing


# --------------------------------------------------------------------------- features
@pytest.mark.parametrize("seed", range(3))
def test_subm_fwd_matches_dense_conv3d(seed):
    rng = np.random.default_rng(100 + seed)
    c = _rand_coords(rng, 120, 0, 8, batch=2)
    cin, cout = 5, 7
    x = rng.standard_normal((len(c), cin))
    w = rng.standard_normal((27, cin, cout))
    y = oracle.conv_fwd(x, w, oracle.kmap(c, c, 3, 1, 1, SUBM))
    dense = torch.nn.functional.conv3d(_densify(c, x, (8, 8, 8), (0, 0, 0)), _dense_weight(w, (3, 3, 3)),
                                       padding=1)
    np.testing.assert_allclose(y, _read(dense, c, (0, 0, 0)).numpy(), rtol=1e-12, atol=1e-12)


def test_subm_fwd_2d_kernel_matches_dense_conv():
    rng = np.random.default_rng(4)
    c = _rand_coords(rng, 90, 0, 9, batch=2)
    c[:, 3] = 0
    c = np.unique(c, axis=0)
    c = c[rng.permutation(len(c))]
    x = rng.standard_normal((len(c), 3))
    w = rng.standard_normal((9, 3, 4))
    y = oracle.conv_fwd(x, w, oracle.kmap(c, c, (3, 3, 1), 1, (1, 1, 0), SUBM))
    dense = torch.nn.functional.conv3d(_densify(c, x, (9, 9, 1), (0, 0, 0)), _dense_weight(w, (3, 3, 1)),
                                       padding=(1, 1, 0))
    np.testing.assert_allclose(y, _read(dense, c, (0, 0, 0)).numpy(), rtol=1e-12, atol=1e-12)


def test_strided_fwd_and_transposed_match_dense():
    rng = np.random.default_rng(9)
    c = _rand_coords(rng, 200, 0, 10, batch=2)
    cin, cmid = 4, 6
    x = rng.standard_normal((len(c), cin))
    w = rng.standard_normal((8, cin, cmid))
    coarse = oracle.downsample(c, 2, 2, 0)
    y = oracle.conv_fwd(x, w, oracle.kmap(c, coarse, 2, 2, 0, STRIDED))
    dense = torch.nn.functional.conv3d(_densify(c, x, (10, 10, 10), (0, 0, 0)), _dense_weight(w, (2, 2, 2)),
                                       stride=2)
    np.testing.assert_allclose(y, _read(dense, coarse, (0, 0, 0)).numpy(), rtol=1e-12, atol=1e-12)
    # transposed conv back onto the fine support: dense weight (Cin, Cout, Kx, Ky, Kz)
    wt = rng.standard_normal((8, cmid, cin))
    z = oracle.conv_fwd(y, wt, oracle.kmap(coarse, c, 2, 2, 0, TRANSPOSED))
    wtd = torch.as_tensor(wt).reshape(2, 2, 2, cmid, cin).permute(3, 4, 0, 1, 2)
    dz = torch.nn.functional.conv_transpose3d(_densify(coarse, y, (5, 5, 5), (0, 0, 0)), wtd, stride=2)
    np.testing.assert_allclose(z, _read(dz, c, (0, 0, 0)).numpy(), rtol=1e-12, atol=1e-12)


def test_k1_conv_is_dense_matmul():
    rng = np.random.default_rng(2)
    c = _rand_coords(rng, 500, -20, 20, batch=2)
    x = rng.standard_normal((len(c), 9))
    w = rng.standard_normal((1, 9, 11))
    y = oracle.conv_fwd(x, w, oracle.kmap(c, c, 1, 1, 0, SUBM))
    np.testing.assert_allclose(y, x @ w[0], rtol=1e-13, atol=1e-13)


def test_isolated_voxel_sees_centre_weight_only():
    c = np.array([[0, 0, 0, 0], [0, 10, 0, 0], [1, 0, 0, 0]], np.int32)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 4))
    w = rng.standard_normal((27, 4, 3))
    y = oracle.conv_fwd(x, w, oracle.kmap(c, c, 3, 1, 1, SUBM))
    np.testing.assert_allclose(y, x @ w[13], rtol=1e-14)


# --------------------------------------------------------------------------- backward
def _inner(a, b):
    return float(np.sum(np.asarray(a, np.float64) * np.asarray(b, np.float64)))


@pytest.mark.parametrize("mode", ["subm", "down", "up"])
def test_adjoint_identities(mode):
    rng = np.random.default_rng(21)
    c = _rand_coords(rng, 250, -6, 6, batch=2)
    if mode == "subm":
        inc, outc, nbr = c, c, oracle.kmap(c, c, 3, 1, 1, SUBM)
    elif mode == "down":
        outc = oracle.downsample(c, 2, 2, 0)
        inc, nbr = c, oracle.kmap(c, outc, 2, 2, 0, STRIDED)
    else:
        inc = oracle.downsample(c, 2, 2, 0)
        outc, nbr = c, oracle.kmap(inc, c, 2, 2, 0, TRANSPOSED)
    k3 = nbr.shape[1]
    x = rng.standard_normal((len(inc), 6))
    w = rng.standard_normal((k3, 6, 5))
    g = rng.standard_normal((len(outc), 5))
    y = oracle.conv_fwd(x, w, nbr)
    dx = oracle.conv_dgrad(g, w, nbr, len(inc))
    dw = oracle.conv_wgrad(x, g, nbr)
    a, b, d = _inner(y, g), _inner(x, dx), _inner(w, dw)
    assert abs(a - b) <= 1e-11 * max(1.0, abs(a))
    assert abs(a - d) <= 1e-11 * max(1.0, abs(a))


def test_transposed_conv_with_transposed_weights_is_dgrad_of_down_conv():
    rng = np.random.default_rng(8)
    c = _rand_coords(rng, 300, -8, 8, batch=2)
    coarse = oracle.downsample(c, 2, 2, 0)
    down = oracle.kmap(c, coarse, 2, 2, 0, STRIDED)
    up = oracle.kmap(coarse, c, 2, 2, 0, TRANSPOSED)
    w = rng.standard_normal((8, 5, 7))
    g = rng.standard_normal((len(coarse), 7))
    dx = oracle.conv_dgrad(g, w, down, len(c))
    z = oracle.conv_fwd(g, np.transpose(w, (0, 2, 1)), up)
    np.testing.assert_allclose(z, dx, rtol=1e-13, atol=1e-13)


def test_backward_matches_dense_autograd():
    rng = np.random.default_rng(31)
    c = _rand_coords(rng, 100, 0, 7, batch=2)
    cin, cout = 4, 3
    x = rng.standard_normal((len(c), cin))
    w = rng.standard_normal((27, cin, cout))
    g = rng.standard_normal((len(c), cout))
    nbr = oracle.kmap(c, c, 3, 1, 1, SUBM)
    xt = torch.tensor(x, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    B = 2
    grid = torch.zeros((B, cin, 7, 7, 7), dtype=torch.float64)
    ci = torch.as_tensor(c, dtype=torch.long)
    grid[ci[:, 0], :, ci[:, 1], ci[:, 2], ci[:, 3]] = xt
    wd = wt.reshape(3, 3, 3, cin, cout).permute(4, 3, 0, 1, 2)
    out = torch.nn.functional.conv3d(grid, wd, padding=1)[ci[:, 0], :, ci[:, 1], ci[:, 2], ci[:, 3]]
    (out * torch.as_tensor(g)).sum().backward()
    np.testing.assert_allclose(oracle.conv_dgrad(g, w, nbr, len(c)), xt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.conv_wgrad(x, g, nbr), wt.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_support_preserving_counts():
    """SubmConv3d keeps the coordinate count exactly; Conv3d k=2 s=2 never grows it."""
    rng = np.random.default_rng(12)
    c = _rand_coords(rng, 400, 0, 16, batch=2)
    nbr = oracle.kmap(c, c, 3, 1, 1, SUBM)
    assert nbr.shape[0] == len(c)
    assert len(oracle.downsample(c, 2, 2, 0)) <= len(c)


def test_target_conv_matches_dense_conv_at_target_sites():
    """TargetConv3d ("Convolution mapping": convolution at known output
    coordinates) = the stride-1 strided relation evaluated at caller targets."""
    rng = np.random.default_rng(41)
    c = _rand_coords(rng, 150, 0, 8, batch=2)
    targets = _rand_coords(rng, 90, 0, 8, batch=2)       # mixes active and inactive sites
    x = rng.standard_normal((len(c), 3))
    w = rng.standard_normal((27, 3, 5))
    y = oracle.conv_fwd(x, w, oracle.kmap(c, targets, 3, 1, 1, STRIDED))
    dense = torch.nn.functional.conv3d(_densify(c, x, (8, 8, 8), (0, 0, 0)), _dense_weight(w, (3, 3, 3)), padding=1)
    np.testing.assert_allclose(y, _read(dense, targets, (0, 0, 0)).numpy(), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- generative transposed conv
_UP_GEOMS = [((2, 2, 2), (2, 2, 2), (0, 0, 0)), ((3, 3, 3), (2, 2, 2), (1, 1, 1)),
             ((3, 2, 1), (2, 1, 3), (1, 0, 0))]


@pytest.mark.parametrize("ks,st,pd", _UP_GEOMS)
def test_upsample_support_equals_nonzero_dense_transposed_conv(ks, st, pd):
    """Generated support = where a dense conv_transpose3d of the occupancy grid
    with an all-ones kernel is nonzero (input index i <-> coordinate i + origin,
    output index o <-> coordinate o + s*origin - pad)."""
    rng = np.random.default_rng(sum(ks) + 7 * sum(st))
    c = _rand_coords(rng, 60, -3, 5, batch=2)
    origin = np.array([-3, -3, -3])
    occ = _densify(c, np.ones((len(c), 1)), (8, 8, 8), tuple(origin))
    out = torch.nn.functional.conv_transpose3d(occ, torch.ones((1, 1) + ks, dtype=torch.float64), stride=st)
    nz = torch.nonzero(out[:, 0] > 0).numpy().astype(np.int64)
    nz[:, 1:] += np.array(st) * origin - np.array(pd)
    nz = nz[np.lexsort(nz.T[::-1])].astype(np.int32)
    assert np.array_equal(oracle.upsample(c, ks, st, pd), nz)


@pytest.mark.parametrize("ks,st,pd", _UP_GEOMS)
def test_generative_transposed_conv_matches_dense_conv_transpose3d(ks, st, pd):
    """GenerativeConvTranspose3d forward on the generated support (transposed
    relation from the input table) = dense conv_transpose3d read at every
    generated site."""
    rng = np.random.default_rng(5 + sum(pd))
    c = _rand_coords(rng, 40, -3, 5, batch=2)
    gen = oracle.upsample(c, ks, st, pd)
    k3, cin, cout = int(np.prod(ks)), 3, 4
    x = rng.standard_normal((len(c), cin))
    w = rng.standard_normal((k3, cin, cout))
    y = oracle.conv_fwd(x, w, oracle.kmap(c, gen, ks, st, pd, TRANSPOSED))
    wd = torch.as_tensor(w).reshape(ks[0], ks[1], ks[2], cin, cout).permute(3, 4, 0, 1, 2)
    origin = np.array([-3, -3, -3])
    dense = torch.nn.functional.conv_transpose3d(_densify(c, x, (8, 8, 8), tuple(origin)), wd, stride=st)
    read_origin = tuple(np.array(st) * origin - np.array(pd))
    np.testing.assert_allclose(y, _read(dense, gen, read_origin).numpy(), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- pooling / dense grids
_POOL_GEOMS = [(3, 1, 1, SUBM), (2, 2, 0, STRIDED), (3, 2, 1, STRIDED), ((3, 3, 1), 1, (1, 1, 0), SUBM)]


def _pool_case(rng, ks, st, pd, mode):
    c = _rand_coords(rng, 150, 0, 8, batch=2)
    out = c if mode == SUBM else oracle.downsample(c, ks, st, pd)
    x = rng.standard_normal((len(c), 5)) - 2.0          # mostly negative: a stray 0 would win a max
    return c, out, x, oracle.kmap(c, out, ks, st, pd, mode)


@pytest.mark.parametrize("ks,st,pd,mode", _POOL_GEOMS)
def test_max_pool_matches_dense_max_pool3d(ks, st, pd, mode):
    """Max over active neighbours = dense max_pool3d of a grid that holds -inf
    at every inactive cell (torch pads with -inf too), read at the outputs."""
    rng = np.random.default_rng(31 + st)
    c, out, x, nbr = _pool_case(rng, ks, st, pd, mode)
    grid = _densify(c, x, (10, 10, 10), (0, 0, 0))
    occ = _densify(c, np.ones((len(c), 1)), (10, 10, 10), (0, 0, 0))
    grid = torch.where(occ > 0, grid, torch.tensor(-np.inf, dtype=torch.float64))
    ksz = (ks,) * 3 if np.isscalar(ks) else ks
    pad = (pd,) * 3 if np.isscalar(pd) else pd
    dense = torch.nn.functional.max_pool3d(grid, ksz, stride=st, padding=pad)
    np.testing.assert_array_equal(oracle.pool(x, nbr, oracle.POOL_MAX), _read(dense, out, (0, 0, 0)).numpy())


@pytest.mark.parametrize("ks,st,pd,mode", _POOL_GEOMS)
def test_avg_pool_is_dense_window_sum_over_active_count(ks, st, pd, mode):
    """Mean over active neighbours = (window sum of the zero-filled grid) /
    (window sum of the occupancy grid): two dense avg_pool3d with divisor 1."""
    rng = np.random.default_rng(47 + st)
    c, out, x, nbr = _pool_case(rng, ks, st, pd, mode)
    ksz = (ks,) * 3 if np.isscalar(ks) else ks
    pad = (pd,) * 3 if np.isscalar(pd) else pd
    sums = [torch.nn.functional.avg_pool3d(_densify(c, v, (10, 10, 10), (0, 0, 0)), ksz, stride=st, padding=pad,
                                           count_include_pad=True, divisor_override=1)
            for v in (x, np.ones((len(c), 1)))]
    ref = (_read(sums[0], out, (0, 0, 0)) / _read(sums[1], out, (0, 0, 0))).numpy()
    np.testing.assert_allclose(oracle.pool(x, nbr, oracle.POOL_AVG), ref, rtol=1e-13, atol=1e-13)


def test_pool_of_row_without_neighbours_is_zero_and_k1_is_identity():
    c = np.array([[0, 0, 0, 0], [0, 1, 0, 0]], np.int32)
    far = np.array([[0, 9, 9, 9], [1, 0, 0, 0], [0, 0, 0, 0]], np.int32)
    x = np.array([[-3.0, 4.0], [-1.0, 2.0]])
    nbr = oracle.kmap(c, far, 3, 1, 1, STRIDED)
    for op in (oracle.POOL_MAX, oracle.POOL_AVG):
        y = oracle.pool(x, nbr, op)
        assert np.all(y[:2] == 0.0)
    np.testing.assert_array_equal(oracle.pool(x, nbr, oracle.POOL_MAX)[2], [-1.0, 4.0])
    np.testing.assert_array_equal(oracle.pool(x, nbr, oracle.POOL_AVG)[2], [-2.0, 3.0])
    rng = np.random.default_rng(3)
    cc = _rand_coords(rng, 40, -5, 5, batch=2)
    xx = rng.standard_normal((len(cc), 3))
    for op in (oracle.POOL_MAX, oracle.POOL_AVG):
        np.testing.assert_array_equal(oracle.pool(xx, oracle.kmap(cc, cc, 1, 1, 0, SUBM), op), xx)


def test_to_dense_matches_sparse_coo_to_dense():
    """Scatter into the box = torch's sparse COO tensor densified, shifted by the origin;
    rows outside the box are dropped and counted."""
    rng = np.random.default_rng(11)
    c = _rand_coords(rng, 80, -4, 6, batch=3)
    x = rng.standard_normal((len(c), 4))
    origin, shape, batch = (-2, -4, -3), (7, 8, 9), 2
    grid, outside = oracle.to_dense(c, x, origin, shape, batch)
    rel = c.astype(np.int64) - np.array((0,) + origin)
    inside = (rel[:, 0] < batch) & np.all(rel[:, 1:] >= 0, 1) & np.all(rel[:, 1:] < np.array(shape), 1)
    assert outside == int((~inside).sum()) > 0
    with torch.sparse.check_sparse_tensor_invariants():
        ref = torch.sparse_coo_tensor(torch.as_tensor(rel[inside].T), torch.as_tensor(x[inside]),
                                      (batch,) + shape + (4,)).to_dense()
    np.testing.assert_array_equal(grid, ref.numpy())
    assert np.count_nonzero(np.any(grid != 0, axis=-1)) == int(inside.sum())
