"""Shared helpers for the parity tests: seeded inputs, layout conversion, tolerances,
and the per-element error statistics reported beside every feature check."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import synthetic

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}

# Tolerances: fp32 normwise 1e-5 relative; fp16 / bf16 max|err| <= 2e-2 * max|ref|.
REL_TOL = {torch.float32: 1e-5, torch.float16: 2e-2, torch.bfloat16: 2e-2}


def feats(n: int, c: int, dtype: torch.dtype, seed: int, stream: int = 0, device="cuda"):
    """N(0,1) features rounded to `dtype`; returns (device tensor, fp64 numpy of the rounded values)."""
    t = torch.from_numpy(synthetic.features(n, c, seed, stream)).to(dtype)
    return t.to(device), t.double().numpy()


def weights(k3: int, cin: int, cout: int, dtype: torch.dtype, seed: int, stream: int = 0, device="cuda"):
    t = torch.from_numpy(synthetic.weights(k3, cin, cout, seed, stream)).to(dtype)
    return t.to(device), t.double().numpy()


# Error statistics of every check made with a reference that carries its terms
# (see with_terms): kept for the session summary, and appended as JSON lines to
# the file named by LAT_ERR_REPORT when that variable is set.
ERROR_LOG: list[dict] = []


class _Ref(np.ndarray):
    """An oracle result that also carries, per element, the sum of the absolute
    values of the terms summed into it (``terms``)."""
    terms = None


def with_terms(fn, *args, **kw) -> np.ndarray:
    """fn(*args) (an oracle routine that sums products of its float inputs) with
    ``.terms`` = the same routine on the absolute values of those inputs, which
    is, element by element, the sum of |term| over the terms of that element."""
    ref = np.asarray(fn(*args, **kw), np.float64).view(_Ref)
    absargs = [np.abs(a) if isinstance(a, np.ndarray) and a.dtype.kind == "f" else a for a in args]
    ref.terms = np.asarray(fn(*absargs, **kw), np.float64)
    return ref


def error_stats(got: np.ndarray, ref: np.ndarray, terms: np.ndarray) -> dict:
    """Per-element |got - ref| / sum|terms| over the elements that have a term:
    median, 99th percentile and maximum (the validation of CUDA results against
    another backend by percentile error statistics)."""
    err = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    sel = terms > 0
    rel = err[sel] / terms[sel]
    if rel.size == 0:
        return {"rel_terms_p50": 0.0, "rel_terms_p99": 0.0, "rel_terms_max": 0.0, "elements": 0}
    p50, p99 = np.percentile(rel, [50, 99])
    return {"rel_terms_p50": float(p50), "rel_terms_p99": float(p99), "rel_terms_max": float(rel.max()),
            "elements": int(rel.size)}


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: torch.dtype, what: str = ""):
    """Normwise check max|got - ref| <= tol(dtype) * max|ref|; when ``ref`` carries
    its terms (with_terms), the per-element error statistics are recorded too."""
    terms = getattr(ref, "terms", None)
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    scale = max(np.abs(ref).max(initial=0.0), 1e-30)
    err = np.abs(got - ref).max(initial=0.0)
    tol = REL_TOL[dtype]
    if terms is not None:
        rec = {"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "what": what,
               "dtype": str(dtype).replace("torch.", ""), "max_err_over_max_ref": float(err / scale), "tol": tol,
               **error_stats(got, ref, terms)}
        ERROR_LOG.append(rec)
        path = os.environ.get("LAT_ERR_REPORT")
        if path:
            with open(path, "a") as f:
                f.write(json.dumps(rec) + "\n")
    assert err <= tol * scale, f"{what}: max|err| {err:.3e} > {tol:g} * max|ref| {scale:.3e}"
    return err / scale


def rand_coords(rng: np.random.Generator, n: int, lo: int, hi: int, batch: int = 1) -> np.ndarray:
    rows = []
    span = hi - lo
    for b in range(batch):
        cells = rng.choice(span ** 3, size=n, replace=False)
        x, r = np.divmod(cells, span * span)
        y, z = np.divmod(r, span)
        rows.append(np.stack([np.full(n, b), x + lo, y + lo, z + lo], 1))
    c = np.concatenate(rows).astype(np.int32) if rows else np.zeros((0, 4), np.int32)
    return np.ascontiguousarray(c[rng.permutation(len(c))])


def u32(a: np.ndarray) -> np.ndarray:
    return np.asarray(a).astype(np.int64) & 0xFFFFFFFF


def group_key(mask: np.ndarray, k3: int) -> np.ndarray:
    """The documented row-grouping key of a neighbour mask (include/lattice.h, lat_kmap.perm)."""
    m = np.asarray(mask, np.int64) & 0xFFFFFFFF
    if k3 <= 8:
        return m
    pc = np.minimum(np.array([bin(int(v)).count("1") for v in m], np.int64), 31)
    return (pc << 11) | (((m * 0x9E3779B1) & 0xFFFFFFFF) >> 21)


def check_kmap(km, ref_nbr: np.ndarray):
    """Bit-exact comparison of a device KernelMap against the oracle's (n_out, k3) table."""
    import oracle
    n_out, k3 = ref_nbr.shape
    got = km.nbr_table().cpu().numpy() if n_out else np.zeros((0, k3), np.int32)
    assert np.array_equal(got, ref_nbr), "neighbour table differs"
    ref_mask = ((ref_nbr >= 0).astype(np.int64) << np.arange(k3)).sum(1) if n_out else np.zeros(0, np.int64)
    mask = u32(km.mask[:n_out].cpu().numpy())
    assert np.array_equal(mask, ref_mask), "mask differs"
    off, pin, pout = oracle.pairs(ref_nbr)
    assert np.array_equal(km.pair_off.cpu().numpy(), off), "pair offsets differ"
    P = int(off[-1])
    assert np.array_equal(km.pair_in[:P].cpu().numpy(), pin), "pair inputs differ"
    assert np.array_equal(km.pair_out[:P].cpu().numpy(), pout), "pair outputs differ"
    perm = km.perm[:n_out].cpu().numpy()
    assert np.array_equal(perm, np.argsort(group_key(ref_mask, k3), kind="stable")), "perm is not the stable key sort"
    ntiles = (n_out + 127) // 128
    tm = u32(km.tile_mask[:ntiles].cpu().numpy())
    sm = ref_mask[perm] if n_out else ref_mask
    for t in range(ntiles):
        assert tm[t] == np.bitwise_or.reduce(sm[t * 128:(t + 1) * 128]), f"tile mask {t}"
