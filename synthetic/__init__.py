"""Seeded synthetic inputs for the sparse-convolution workloads.

This module only draws random numbers and arranges them into coordinate
rows, feature rows and weights.  It holds none of the method's arithmetic
(no key packing, no neighbour search, no convolution): both the CPU oracle
and the CUDA path consume what it produces, and neither is imported here.

The pages' own workloads (nuScenes / Waymo LiDAR scans for TorchSparse++,
LArTPC neutrino images for SparsePixels) are not available, so these
generators stand in for them with the same shapes and structure:

* ``uniform_cube``  -- N unique voxels drawn uniformly in a cube.
* ``lidar``         -- a LiDAR-shaped scan: a ground plane (two z layers)
                       plus Gaussian clusters, per batch sample.
* ``sparse_images`` -- 2D images with ~1% active pixels in Gaussian
                       clusters (z fixed to 0).

Every generator draws candidates, rejects duplicates and out-of-grid
draws (never clamps), keeps the order of first appearance, and finally
shuffles the rows with the seed so that no consumer sees pre-sorted input.
Random streams come from ``numpy.random.SeedSequence(seed).spawn``.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = [
    "uniform_cube", "lidar", "sparse_images", "features", "weights",
    "Workload", "WORKLOADS", "make_workload",
]


def _rng(seed_seq: np.random.SeedSequence) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed_seq))


def _take_unique(cells: np.ndarray, seen: set | None, need: int):
    """Return the first ``need`` cell ids not seen before, in draw order."""
    _, first = np.unique(cells, return_index=True)
    first.sort()
    ordered = cells[first]
    if seen:
        keep = np.fromiter((c not in seen for c in ordered.tolist()), bool, len(ordered))
        ordered = ordered[keep]
    return ordered[:need]


def _draw_unique(draw, need: int, rng: np.random.Generator, chunk: int) -> np.ndarray:
    """Draw candidate cell ids with ``draw(rng, m)`` (-1 = rejected) until ``need``
    unique ids exist; the order of first appearance is kept."""
    out: list[np.ndarray] = []
    seen: set[int] = set()
    have = 0
    while have < need:
        cand = draw(rng, chunk)
        cand = cand[cand >= 0]
        new = _take_unique(cand, seen, need - have)
        seen.update(new.tolist())
        out.append(new)
        have += len(new)
    return np.concatenate(out)[:need]


def uniform_cube(n: int, grid: int, seed: int, batch: int = 1) -> np.ndarray:
    """``batch`` samples of ``n`` unique voxels each, uniform in ``grid``^3.

    Returns int32 (batch*n, 4) rows (b, x, y, z), shuffled."""
    ss = np.random.SeedSequence(seed)
    kids = ss.spawn(batch + 1)
    rows = []
    for b in range(batch):
        rng = _rng(kids[b])
        if n > grid ** 3:
            raise ValueError("more voxels than cells")
        cells = rng.choice(grid ** 3, size=n, replace=False)
        x, rem = np.divmod(cells, grid * grid)
        y, z = np.divmod(rem, grid)
        rows.append(np.stack([np.full(n, b), x, y, z], 1))
    coords = np.concatenate(rows).astype(np.int32)
    perm = _rng(kids[batch]).permutation(len(coords))
    return np.ascontiguousarray(coords[perm])


def lidar(batch: int, per_sample: int, seed: int, dims=(1440, 1440, 41),
          ground_frac: float = 0.6, ground_z=(2, 3), n_clusters: int = 200,
          sigma: float = 8.0) -> np.ndarray:
    """LiDAR-shaped scan: per sample ``per_sample`` unique voxels.

    Each candidate is a ground point with probability ``ground_frac``
    (x, y uniform integers, z uniform over ``ground_z``) or else a cluster
    point: one of ``n_clusters`` centres drawn uniformly in the continuous
    grid, plus an N(0, sigma^2) offset per axis, rounded half up.
    Out-of-grid candidates and repeats are rejected.  Returns int32
    (batch*per_sample, 4), shuffled."""
    X, Y, Z = dims
    ss = np.random.SeedSequence(seed)
    kids = ss.spawn(batch + 1)
    gz = np.asarray(ground_z)
    rows = []
    for b in range(batch):
        rng = _rng(kids[b])
        centres = rng.random((n_clusters, 3)) * np.array([X, Y, Z], dtype=np.float64)

        def draw(r: np.random.Generator, m: int) -> np.ndarray:
            is_ground = r.random(m) < ground_frac
            gx = r.integers(0, X, m)
            gy = r.integers(0, Y, m)
            gzz = gz[r.integers(0, len(gz), m)]
            ci = r.integers(0, n_clusters, m)
            p = centres[ci] + r.normal(0.0, sigma, (m, 3))
            p = np.floor(p + 0.5).astype(np.int64)
            x = np.where(is_ground, gx, p[:, 0])
            y = np.where(is_ground, gy, p[:, 1])
            z = np.where(is_ground, gzz, p[:, 2])
            ok = (x >= 0) & (x < X) & (y >= 0) & (y < Y) & (z >= 0) & (z < Z)
            cell = (x * Y + y) * Z + z
            return np.where(ok, cell, -1)

        cells = _draw_unique(draw, per_sample, rng, chunk=max(1024, per_sample // 2))
        x, rem = np.divmod(cells, Y * Z)
        y, z = np.divmod(rem, Z)
        rows.append(np.stack([np.full(per_sample, b), x, y, z], 1))
    coords = np.concatenate(rows).astype(np.int32)
    perm = _rng(kids[batch]).permutation(len(coords))
    return np.ascontiguousarray(coords[perm])


def sparse_images(batch: int, height: int, width: int, active_frac: float, seed: int,
                  n_clusters: int = 16, sigma: float = 6.0) -> np.ndarray:
    """2D sparse images with z = 0: per image floor(active_frac*H*W) unique
    active pixels drawn around ``n_clusters`` uniformly placed centres with
    an N(0, sigma^2) offset per axis (rounded half up).  Returns int32
    (batch*n, 4) rows (b, x, y, 0), shuffled."""
    n = int(np.floor(active_frac * height * width))
    ss = np.random.SeedSequence(seed)
    kids = ss.spawn(batch + 1)
    rows = []
    for b in range(batch):
        rng = _rng(kids[b])
        centres = rng.random((n_clusters, 2)) * np.array([height, width], dtype=np.float64)

        def draw(r: np.random.Generator, m: int) -> np.ndarray:
            ci = r.integers(0, n_clusters, m)
            p = np.floor(centres[ci] + r.normal(0.0, sigma, (m, 2)) + 0.5).astype(np.int64)
            ok = (p[:, 0] >= 0) & (p[:, 0] < height) & (p[:, 1] >= 0) & (p[:, 1] < width)
            return np.where(ok, p[:, 0] * width + p[:, 1], -1)

        cells = _draw_unique(draw, n, rng, chunk=max(1024, n))
        x, y = np.divmod(cells, width)
        rows.append(np.stack([np.full(n, b), x, y, np.zeros(n, np.int64)], 1))
    coords = np.concatenate(rows).astype(np.int32)
    perm = _rng(kids[batch]).permutation(len(coords))
    return np.ascontiguousarray(coords[perm])


def features(n: int, c: int, seed: int, stream: int = 0) -> np.ndarray:
    """N(0,1) float32 (n, c).  Callers cast to fp16/bf16 (round to nearest even)."""
    ss = np.random.SeedSequence([seed, 1000 + stream])
    return _rng(ss).standard_normal((n, c), dtype=np.float32)


def weights(k3: int, cin: int, cout: int, seed: int, stream: int = 0) -> np.ndarray:
    """Per-offset weights (k3, cin, cout) drawn N(0, 1/(k3*cin)) in float32
    (the second argument of N(.,.) read as the variance, fan-in k3*cin)."""
    ss = np.random.SeedSequence([seed, 2000 + stream])
    std = np.float32(1.0 / np.sqrt(k3 * cin))
    return (_rng(ss).standard_normal((k3, cin, cout), dtype=np.float32) * std).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One of the five seeded workloads (coordinates are generated lazily)."""
    name: str
    seed: int
    kind: str            # "uniform" | "lidar" | "images"
    gen_args: dict
    ksize: tuple
    dtype: str           # "f32" | "f16" | "bf16"
    cin: int
    cout: int
    description: str

    def coords(self) -> np.ndarray:
        if self.kind == "uniform":
            return uniform_cube(seed=self.seed, **self.gen_args)
        if self.kind == "lidar":
            return lidar(seed=self.seed, **self.gen_args)
        if self.kind == "images":
            return sparse_images(seed=self.seed, **self.gen_args)
        raise ValueError(self.kind)


WORKLOADS = {
    "subm_small": Workload(
        "subm_small", 1, "uniform", dict(n=2000, grid=32), (3, 3, 3), "f32", 16, 16,
        "SubmConv3d k=3, batch 1, 2,000 unique voxels uniform in 32^3, 16->16, fp32"),
    "lidar_subm": Workload(
        "lidar_subm", 2, "lidar", dict(batch=2, per_sample=100_000), (3, 3, 3), "f16", 64, 64,
        "LiDAR-shaped SubmConv3d k=3, batch 2 x 100k voxels in 1440x1440x41, 64->64, fp16"),
    "lidar_down_up": Workload(
        "lidar_down_up", 3, "lidar", dict(batch=2, per_sample=100_000), (2, 2, 2), "bf16", 64, 128,
        "strided Conv3d k=2 s=2 64->128 then ConvTranspose3d k=2 s=2 128->64, 200k LiDAR voxels, bf16"),
    "images_subm": Workload(
        "images_subm", 4, "images", dict(batch=256, height=512, width=512, active_frac=0.01),
        (3, 3, 1), "f32", 8, 32,
        "2D submanifold 3x3 over 256 images 512x512 with 1% active pixels, 8->32, fp32"),
    "lidar_train": Workload(
        "lidar_train", 5, "lidar", dict(batch=4, per_sample=125_000), (3, 3, 3), "bf16", 128, 128,
        "SubmConv3d k=3 training step (fwd + dgrad + wgrad), 4 x 125k LiDAR voxels, 128->128, bf16"),
}


def make_workload(name: str) -> Workload:
    return WORKLOADS[name]
