"""The hash table's probe window is never reached on the benchmark workloads.

An insert flags LAT_ERR_TABLE_FULL when it finds no free slot within 4096
slots of the start of its key's home group (include/lattice.h, hashing).
With linear probing the set of occupied slots does not depend on the order
of the inserts, and a key always sits before the first slot that is empty
in the finished table, counting from its home group.  So the largest
distance from a home group to the next empty slot bounds the displacement
of every key under every insertion order, and the GPU's concurrent inserts
cannot reach the window if that bound stays below 4096.  The placement
function (the z-brick of the key, folded and mixed) is restated from the
header; this runs on the CPU at the default ratio 4 and at ratio 2, on the
five workloads and on a fully dense cube, where every z-brick holds four keys.
"""
import numpy as np
import pytest

import synthetic

WINDOW = 4096
M = np.uint64(0xFFFFFFFF)


def pack(c: np.ndarray) -> np.ndarray:
    c = c.astype(np.int64)
    return ((c[:, 0].astype(np.uint64) << np.uint64(48)) | ((c[:, 1] + 32768).astype(np.uint64) << np.uint64(32))
            | ((c[:, 2] + 32768).astype(np.uint64) << np.uint64(16)) | (c[:, 3] + 32768).astype(np.uint64))


def home_groups(keys: np.ndarray, cap: int) -> np.ndarray:
    k = keys & ~np.uint64(3)
    h = (k & M) ^ (((k >> np.uint64(32)) * np.uint64(0x9E3779B1)) & M)
    h ^= h >> np.uint64(16)
    h = (h * np.uint64(0x85EBCA6B)) & M
    h ^= h >> np.uint64(13)
    h = (h * np.uint64(0xC2B2AE35)) & M
    h ^= h >> np.uint64(16)
    return (h & np.uint64(cap - 1) & ~np.uint64(3)).astype(np.int64)


def table_slots(n: int, ratio: float) -> int:
    cap = 64
    while cap < ratio * n:
        cap <<= 1
    return cap


def worst_probe_distance(keys: np.ndarray, ratio: float) -> int:
    """Largest distance from a key's home group start to the first empty slot
    at or after it in the finished table (linear probing, any insert order)."""
    cap = table_slots(len(keys), ratio)
    homes = home_groups(keys, cap)
    occ = bytearray(cap)
    mask = cap - 1
    for h in np.sort(homes).tolist():
        s = h
        while occ[s]:
            s = (s + 1) & mask
        occ[s] = 1
    empty = np.flatnonzero(np.frombuffer(bytes(occ), np.uint8) == 0)
    idx = np.searchsorted(empty, homes)
    nxt = np.where(idx < len(empty), empty[np.minimum(idx, len(empty) - 1)], empty[0] + cap)
    return int((nxt - homes).max())


def dense_cube(side: int, batch: int) -> np.ndarray:
    ax = np.arange(side)
    g = np.stack(np.meshgrid(ax, ax, ax, indexing="ij"), -1).reshape(-1, 3)
    return np.concatenate([np.c_[np.full(len(g), b), g] for b in range(batch)]).astype(np.int32)


def test_distance_bound_matches_a_direct_simulation():
    """The bound is an upper bound of the displacement of a real insertion order."""
    rng = np.random.default_rng(0)
    c = dense_cube(12, 2)[rng.permutation(2 * 12 ** 3)]
    keys = pack(c)
    cap = table_slots(len(keys), 1.0)
    occ = bytearray(cap)
    worst = 0
    for h in home_groups(keys, cap).tolist():
        s, d = h, 0
        while occ[s]:
            s, d = (s + 1) & (cap - 1), d + 1
        occ[s] = 1
        worst = max(worst, d)
    assert worst < worst_probe_distance(keys, 1.0)


@pytest.mark.parametrize("ratio", [2.0, 4.0])
@pytest.mark.parametrize("name", sorted(synthetic.WORKLOADS))
def test_workloads_stay_inside_the_probe_window(name, ratio):
    keys = pack(synthetic.WORKLOADS[name].coords())
    assert worst_probe_distance(keys, ratio) < WINDOW


@pytest.mark.parametrize("ratio", [2.0, 4.0])
def test_dense_cube_stays_inside_the_probe_window(ratio):
    keys = pack(dense_cube(80, 1))   # 512,000 cells, every z-brick full
    assert worst_probe_distance(keys, ratio) < WINDOW
