"""The seeded input generators produce what the input recipe states (CPU only).

Every workload: int32 (N, 4) rows, unique, inside its grid, the stated count
per batch sample, identical on every call (seeded), and shuffled (not in key
order).  LiDAR scans: about two thirds of the cells on the two ground layers;
sparse images: z = 0 and floor(1% of 512^2) pixels per image.  Features are
N(0, 1) and weights N(0, 1 / (K^3 Cin)).
"""
import numpy as np
import pytest

import synthetic

GRIDS = {"uniform": (32, 32, 32), "lidar": (1440, 1440, 41), "images": (512, 512, 1)}


def _check_rows(c: np.ndarray, grid, batch: int, per_sample: int):
    assert c.dtype == np.int32 and c.ndim == 2 and c.shape[1] == 4
    assert c.shape[0] == batch * per_sample
    assert len(np.unique(c, axis=0)) == len(c), "duplicate coordinate rows"
    assert c[:, 0].min() == 0 and c[:, 0].max() == batch - 1
    assert np.array_equal(np.bincount(c[:, 0], minlength=batch), np.full(batch, per_sample))
    for a in range(3):
        assert c[:, a + 1].min() >= 0 and c[:, a + 1].max() < grid[a]


@pytest.mark.parametrize("name", sorted(synthetic.WORKLOADS))
def test_workload_rows(name):
    wl = synthetic.WORKLOADS[name]
    c = wl.coords()
    args = wl.gen_args
    if wl.kind == "uniform":
        batch, per = 1, args["n"]
    elif wl.kind == "lidar":
        batch, per = args["batch"], args["per_sample"]
    else:
        batch, per = args["batch"], int(args["active_frac"] * args["height"] * args["width"])
    _check_rows(c, GRIDS[wl.kind], batch, per)
    assert np.array_equal(c, wl.coords()), "not reproducible"
    order = np.lexsort(c.T[::-1])
    assert not np.array_equal(order, np.arange(len(c))), "rows come sorted"


def test_lidar_ground_share_and_images_plane():
    c = synthetic.WORKLOADS["lidar_subm"].coords()
    ground = np.isin(c[:, 3], (2, 3)).mean()
    assert 0.60 <= ground <= 0.70, ground            # 60% of the draws, ~65% of the final cells
    img = synthetic.WORKLOADS["images_subm"].coords()
    assert np.all(img[:, 3] == 0)


def test_lidar_workloads_differ_by_seed():
    a = synthetic.WORKLOADS["lidar_subm"].coords()
    b = synthetic.WORKLOADS["lidar_down_up"].coords()
    assert a.shape == b.shape and not np.array_equal(a, b)


def test_feature_and_weight_distributions():
    f = synthetic.features(200_000, 8, seed=7)
    assert f.dtype == np.float32 and f.shape == (200_000, 8)
    assert abs(float(f.mean())) < 0.01 and abs(float(f.std()) - 1.0) < 0.01
    assert np.array_equal(f, synthetic.features(200_000, 8, seed=7))
    assert not np.array_equal(f, synthetic.features(200_000, 8, seed=7, stream=1))
    w = synthetic.weights(27, 64, 64, seed=7)
    assert w.dtype == np.float32 and w.shape == (27, 64, 64)
    assert abs(float(w.std()) * np.sqrt(27 * 64) - 1.0) < 0.02
