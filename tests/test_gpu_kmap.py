"""Hash table, kernel-map query and support generation on the GPU against the oracle.

Integer results are compared bit-exactly: neighbour tables, masks, pair
lists (canonical order: offset, then output row), the stable mask sort, tile
masks and generated coordinates.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.util import check_kmap, rand_coords, u32

pytestmark = pytest.mark.gpu

scv = pytest.importorskip("sparse_convolution_voxel_b200")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _slot_hash(key: int) -> int:
    """The table's placement function (fold of the halves of the key's z-brick, the
    key with the two low bits of its z field cleared, then MurmurHash3 fmix32),
    restated here to check where the GPU put every key."""
    M = 0xFFFFFFFF
    key &= ~3
    h = (key & M) ^ (((key >> 32) * 0x9E3779B1) & M)
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & M
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & M
    h ^= h >> 16
    return h


def _table_slots(table):
    """(key, row) of every slot of a table of 64-byte groups {key[4], row[4], unused[4]}."""
    g = table.cpu().numpy().view(np.uint8).reshape(-1, 64)
    keys = np.ascontiguousarray(g[:, :32]).view(np.uint64).reshape(-1)
    rows = np.ascontiguousarray(g[:, 32:48]).view(np.uint32).reshape(-1).astype(np.int64)
    return keys, rows


def _subm(coords, ks=(3, 3, 3), d_status=None):
    c = _dev(coords)
    table = scv.hash_table(c, 2.0, d_status)
    g = scv.subm_geom(ks)
    return scv.kernel_map(table, len(coords), c, g, d_status=d_status), table


# --------------------------------------------------------------------------- hash table
def test_hash_table_places_every_key_reachably():
    rng = np.random.default_rng(0)
    coords = rand_coords(rng, 3000, -40, 40, batch=3)
    st = scv.new_status()
    table = scv.hash_table(_dev(coords), 2.0, st)
    scv.check_status(st)
    keys, rows = _table_slots(table)
    cap = len(keys)
    empty = np.uint64(0xFFFFFFFFFFFFFFFF)
    occupied = np.nonzero(keys != empty)[0]
    assert len(occupied) == len(coords)
    want = {oracle.pack_key(*map(int, r)): i for i, r in enumerate(coords)}
    for s in occupied:
        k = int(keys[s])
        assert want[k] == rows[s]
        start = _slot_hash(k) & (cap - 1) & ~3     # probing starts at the home slot's 4-slot group
        d = (s - start) % cap                      # linear probing: no empty slot between start and s
        assert all(keys[(start + e) % cap] != empty for e in range(d))


def test_hash_flags_duplicates_and_keeps_lowest_row():
    coords = np.array([[0, 1, 2, 3], [0, 5, 5, 5], [0, 1, 2, 3], [0, 1, 2, 3]], np.int32)
    st = scv.new_status()
    table = scv.hash_table(_dev(coords), 2.0, st)
    assert scv.lat_status_fetch(st) & 4
    keys, rows = _table_slots(table)
    k = np.uint64(oracle.pack_key(0, 1, 2, 3))
    assert int(rows[keys == k][0]) == 0


def test_hash_flags_out_of_range_coordinates():
    coords = np.array([[0, 40000, 0, 0], [0, 1, 1, 1], [70000, 0, 0, 0]], np.int32)
    st = scv.new_status()
    scv.hash_table(_dev(coords), 2.0, st)
    assert scv.lat_status_fetch(st) & 2


def test_hash_flags_full_table():
    rng = np.random.default_rng(1)
    coords = rand_coords(rng, 100, 0, 10)
    table = torch.empty(2 * 64, dtype=torch.int64, device="cuda")   # 64 slots < 100 rows
    st = scv.new_status()
    scv.lat_hash_build(_dev(coords), table, st)
    assert scv.lat_status_fetch(st) & 8


# --------------------------------------------------------------------------- submanifold maps
@pytest.mark.parametrize("n,batch,lo,hi", [(1, 1, 0, 4), (127, 1, 0, 8), (129, 2, -5, 5), (1000, 3, -12, 12)])
def test_subm_kmap_small_ragged(n, batch, lo, hi):
    rng = np.random.default_rng(n)
    coords = rand_coords(rng, n, lo, hi, batch)
    st = scv.new_status()
    km, _ = _subm(coords, d_status=st)
    scv.check_status(st)
    check_kmap(km, oracle.kmap(coords, coords, 3, 1, 1, oracle.SUBM))


@pytest.mark.parametrize("ratio", [1.0, 2.0, 4.0])
def test_subm_kmap_dense_cube(ratio):
    """Every cell of an 11^3 cube in two batches: each z-brick holds 4 keys, so
    home groups fill up and probes run on into the following groups (at ratio 1
    the table is 65% full)."""
    ax = np.arange(-5, 6)
    g = np.stack(np.meshgrid(ax, ax, ax, indexing="ij"), -1).reshape(-1, 3)
    coords = np.concatenate([np.c_[np.full(len(g), b), g] for b in range(2)]).astype(np.int32)
    coords = np.ascontiguousarray(coords[np.random.default_rng(1).permutation(len(coords))])
    c = _dev(coords)
    st = scv.new_status()
    table = scv.hash_table(c, ratio, st)
    km = scv.kernel_map(table, len(coords), c, scv.subm_geom(3), d_status=st)
    scv.check_status(st)
    check_kmap(km, oracle.kmap(coords, coords, 3, 1, 1, oracle.SUBM))
    keys, rows = _table_slots(table)
    cap = len(keys)
    empty = np.uint64(0xFFFFFFFFFFFFFFFF)
    for s in np.nonzero(keys != empty)[0]:
        start = _slot_hash(int(keys[s])) & (cap - 1) & ~3
        d = (s - start) % cap
        assert all(keys[(start + e) % cap] != empty for e in range(d))


def test_subm_kmap_at_the_edges_of_the_key_range():
    """Rows packed against the key range (x, y, z at -32768 / 32767, batch 0 and
    65534): neighbours outside the range are absent, never wrapped around."""
    rows = []
    for b in (0, 65534):
        for xs in ((-32768, -32767, -32766), (32765, 32766, 32767)):
            for zs in ((-32768, -32767, -32766, -32765), (32764, 32765, 32766, 32767)):
                for x in xs:
                    for y in (-32768, -32767, 32766, 32767):
                        for z in zs:
                            rows.append((b, x, y, z))
    coords = np.array(rows, np.int32)
    coords = np.ascontiguousarray(coords[np.random.default_rng(2).permutation(len(coords))])
    for ks in ((3, 3, 3), (3, 3, 1), (1, 1, 5)):
        km, _ = _subm(coords, ks)
        check_kmap(km, oracle.kmap(coords, coords, ks, 1, oracle.subm_pad(ks), oracle.SUBM))


def test_subm_kmap_empty():
    coords = np.zeros((0, 4), np.int32)
    km, _ = _subm(coords)
    torch.cuda.synchronize()
    assert km.pair_off.cpu().numpy().tolist() == [0] * 28


@pytest.mark.parametrize("ks", [(5, 3, 1), (1, 1, 1), (3, 3, 1), (5, 5, 1), (1, 1, 5), (3, 1, 5), (1, 3, 7),
                                (1, 5, 3), (1, 1, 11), (1, 1, 13)])
def test_subm_kmap_other_kernels(ks):
    """(1, 1, 11): a column of five z cells below the centre, the longest the
    brick lookups take; (1, 1, 13): six, which takes the per-offset probe."""
    rng = np.random.default_rng(3)
    coords = rand_coords(rng, 700, -9, 9, 2)
    km, _ = _subm(coords, ks)
    check_kmap(km, oracle.kmap(coords, coords, ks, 1, oracle.subm_pad(ks), oracle.SUBM))


@pytest.mark.parametrize("name", ["subm_small", "lidar_subm", "images_subm", "lidar_train"])
def test_subm_kmap_full_workloads(name):
    w = synthetic.WORKLOADS[name]
    coords = w.coords()
    st = scv.new_status()
    km, _ = _subm(coords, w.ksize, st)
    scv.check_status(st)
    check_kmap(km, oracle.kmap(coords, coords, w.ksize, 1, oracle.subm_pad(w.ksize), oracle.SUBM))


def test_kmap_runs_are_deterministic():
    coords = synthetic.WORKLOADS["lidar_subm"].coords()
    a, _ = _subm(coords)
    b, _ = _subm(coords)
    P = int(a.pair_off[-1].item())
    n, k3 = a.n_out, a.k3
    for f, m in (("nbr", n * k3), ("mask", n), ("perm", n), ("tile_mask", a.ntiles), ("pair_off", k3 + 1),
                 ("pair_in", P), ("pair_out", P)):
        assert torch.equal(getattr(a, f)[:m], getattr(b, f)[:m]), f


def test_kmap_flags_small_pair_capacity():
    rng = np.random.default_rng(5)
    coords = rand_coords(rng, 500, 0, 9)
    c = _dev(coords)
    st = scv.new_status()
    table = scv.hash_table(c, 2.0, st)
    km = scv.kernel_map(table, len(coords), c, scv.subm_geom(3), d_status=st, pair_capacity=100)
    assert scv.lat_status_fetch(st) & 16
    ref = oracle.kmap(coords, coords, 3, 1, 1, oracle.SUBM)
    assert np.array_equal(km.pair_off.cpu().numpy(), oracle.pairs(ref)[0])


# --------------------------------------------------------------------------- strided / transposed
@pytest.mark.parametrize("ks,st_,pd", [((2, 2, 2), (2, 2, 2), (0, 0, 0)), ((3, 3, 3), (2, 2, 2), (1, 1, 1)),
                                       ((3, 2, 1), (2, 1, 3), (0, 1, 0))])
def test_downsample_and_strided_maps_small(ks, st_, pd):
    rng = np.random.default_rng(11)
    coords = rand_coords(rng, 900, -10, 10, 2)
    c = _dev(coords)
    st = scv.new_status()
    g = scv.strided_geom(ks, st_, pd)
    coarse = scv.downsample(c, g, d_status=st)
    ref_coarse = oracle.downsample(coords, ks, st_, pd)
    assert np.array_equal(coarse.cpu().numpy(), ref_coarse)
    table = scv.hash_table(c, 2.0, st)
    down = scv.kernel_map(table, len(coords), coarse.contiguous(), g, d_status=st)
    check_kmap(down, oracle.kmap(coords, ref_coarse, ks, st_, pd, oracle.STRIDED))
    ctable = scv.hash_table(coarse.contiguous(), 2.0, st)
    up = scv.kernel_map(ctable, len(ref_coarse), c, scv.transposed_geom(ks, st_, pd), d_status=st)
    check_kmap(up, oracle.kmap(ref_coarse, coords, ks, st_, pd, oracle.TRANSPOSED))
    scv.check_status(st)


def test_downsample_full_workload():
    coords = synthetic.WORKLOADS["lidar_down_up"].coords()
    c = _dev(coords)
    g = scv.strided_geom(2, 2, 0)
    coarse = scv.downsample(c, g)
    ref = oracle.downsample(coords, 2, 2, 0)
    assert np.array_equal(coarse.cpu().numpy(), ref)
    table = scv.hash_table(c)
    check_kmap(scv.kernel_map(table, len(coords), coarse.contiguous(), g),
               oracle.kmap(coords, ref, 2, 2, 0, oracle.STRIDED))
    ctable = scv.hash_table(coarse.contiguous())
    check_kmap(scv.kernel_map(ctable, len(ref), c, scv.transposed_geom(2, 2, 0)),
               oracle.kmap(ref, coords, 2, 2, 0, oracle.TRANSPOSED))


def test_downsample_capacity_error():
    rng = np.random.default_rng(2)
    coords = rand_coords(rng, 300, 0, 20)
    with pytest.raises(scv.LatticeError):
        scv.downsample(_dev(coords), scv.strided_geom(2, 2, 0), capacity=10)


# --------------------------------------------------------------------------- parents and maps from parents
@pytest.mark.parametrize("lo,hi", [(-10, 10), (-30000, 30000)])   # bitmap counting sort / radix sort path
def test_downsample_parent_and_maps_from_parent(lo, hi):
    rng = np.random.default_rng(abs(lo))
    if hi - lo > 100:
        coords = np.unique(rng.integers(lo, hi, (3000, 4)).astype(np.int32), axis=0)
        coords[:, 0] = rng.integers(0, 3, len(coords))
        coords = np.unique(coords, axis=0)
        coords = coords[rng.permutation(len(coords))]
    else:
        coords = rand_coords(rng, 1500, lo, hi, 3)
    c = _dev(coords)
    g = scv.strided_geom(2, 2, 0)
    st = scv.new_status()
    coarse, parent = scv.downsample(c, g, d_status=st, with_parent=True)
    ref = oracle.downsample(coords, 2, 2, 0)
    assert np.array_equal(coarse.cpu().numpy(), ref)
    par = parent.cpu().numpy()
    assert np.array_equal(ref[par][:, 1:], np.floor_divide(coords[:, 1:], 2))
    assert np.array_equal(ref[par][:, 0], coords[:, 0])
    down, up = scv.maps_from_parent(c, parent, len(ref), g, d_status=st)
    scv.check_status(st)
    check_kmap(down, oracle.kmap(coords, ref, 2, 2, 0, oracle.STRIDED))
    check_kmap(up, oracle.kmap(ref, coords, 2, 2, 0, oracle.TRANSPOSED))


@pytest.mark.parametrize("lo,hi", [(-10, 10), (-30000, 30000)])   # bitmap path / blocking radix-sort fallback
def test_downsample_async_matches_blocking(lo, hi):
    rng = np.random.default_rng(7 + abs(lo))
    if hi - lo > 100:
        coords = np.unique(rng.integers(lo, hi, (2000, 4)).astype(np.int32), axis=0)
        coords[:, 0] = rng.integers(0, 2, len(coords))
        coords = np.unique(coords, axis=0)
        coords = coords[rng.permutation(len(coords))]
    else:
        coords = rand_coords(rng, 1200, lo, hi, 2)
    c = _dev(coords)
    g = scv.strided_geom(2, 2, 0)
    st = scv.new_status()
    pending = scv.downsample_async(c, g, d_status=st, with_parent=True)
    raw = int(pending._host[0]) if pending._event.query() else None
    coarse, parent = pending.result()
    ref = oracle.downsample(coords, 2, 2, 0)
    assert np.array_equal(coarse.cpu().numpy(), ref)
    par = parent.cpu().numpy()
    assert np.array_equal(ref[par][:, 1:], np.floor_divide(coords[:, 1:], 2))
    scv.check_status(st)
    if raw is not None:   # the enqueued count is the row count on the bitmap path, -1 when the fallback ran
        assert raw == (len(ref) if hi - lo <= 100 else -1)
    # a count above the capacity is reported (on either path), not written past the buffer
    small = scv.downsample_async(c, g, capacity=max(1, len(ref) // 2))
    with pytest.raises(scv.LatticeError):
        small.count()


def test_maps_from_parent_full_workload():
    coords = synthetic.WORKLOADS["lidar_down_up"].coords()
    c = _dev(coords)
    g = scv.strided_geom(2, 2, 0)
    coarse, parent = scv.downsample(c, g, with_parent=True)
    ref = oracle.downsample(coords, 2, 2, 0)
    assert np.array_equal(coarse.cpu().numpy(), ref)
    down, up = scv.maps_from_parent(c, parent, len(ref), g)
    check_kmap(down, oracle.kmap(coords, ref, 2, 2, 0, oracle.STRIDED))
    check_kmap(up, oracle.kmap(ref, coords, 2, 2, 0, oracle.TRANSPOSED))


def test_downsample_parent_needs_kernel_equal_stride():
    coords = rand_coords(np.random.default_rng(0), 100, 0, 8)
    with pytest.raises(scv.LatticeError):
        scv.downsample(_dev(coords), scv.strided_geom(3, 2, 1), with_parent=True)


# --------------------------------------------------------------------------- generative transposed support
@pytest.mark.parametrize("ks,st_,pd,lo,hi", [((2, 2, 2), (2, 2, 2), (0, 0, 0), -10, 10),
                                             ((3, 3, 3), (2, 2, 2), (1, 1, 1), -10, 10),
                                             ((3, 2, 1), (2, 1, 3), (1, 0, 0), -10, 10),
                                             ((2, 2, 2), (2, 2, 2), (0, 0, 0), -10000, 10000)])  # radix-sort path
def test_upsample_matches_oracle(ks, st_, pd, lo, hi):
    rng = np.random.default_rng(31 + abs(lo))
    if hi - lo > 100:
        coords = np.unique(rng.integers(lo, hi, (800, 4)).astype(np.int32), axis=0)
        coords[:, 0] = rng.integers(0, 2, len(coords))
        coords = np.unique(coords, axis=0)
        coords = coords[rng.permutation(len(coords))]
    else:
        coords = rand_coords(rng, 500, lo, hi, 2)
    st = scv.new_status()
    g = scv.transposed_geom(ks, st_, pd)
    fine = scv.upsample(_dev(coords), g, d_status=st)
    scv.check_status(st)
    assert np.array_equal(fine.cpu().numpy(), oracle.upsample(coords, ks, st_, pd))


def test_upsample_errors():
    coords = rand_coords(np.random.default_rng(4), 200, 0, 10)
    with pytest.raises(scv.LatticeError):            # needs the transposed geometry
        scv.upsample(_dev(coords), scv.strided_geom(2, 2, 0))
    with pytest.raises(scv.LatticeError):            # undersized output buffer
        scv.upsample(_dev(coords), scv.transposed_geom(2, 2, 0), capacity=100)
