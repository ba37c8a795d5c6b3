"""The error statistics reported beside every feature check (tests/util.py):
the per-element sum of |terms| that with_terms attaches to an oracle result is
checked against a brute-force sum over the pairs, and error_stats against
hand-computed percentiles.  CPU only."""
import numpy as np

import oracle
from tests.util import error_stats, rand_coords, with_terms


def test_terms_of_forward_equal_brute_force_sum_of_absolute_products():
    rng = np.random.default_rng(5)
    coords = rand_coords(rng, 60, 0, 5)
    nbr = oracle.kmap(coords, coords, 3, 1, 1, oracle.SUBM)
    x = rng.standard_normal((len(coords), 3))
    w = rng.standard_normal((27, 3, 2))
    ref = with_terms(oracle.conv_fwd, x, w, nbr)
    want = np.zeros((len(coords), 2))
    for j in range(len(coords)):
        for k in range(27):
            i = nbr[j, k]
            if i >= 0:
                for ci in range(3):
                    for co in range(2):
                        want[j, co] += abs(x[i, ci] * w[k, ci, co])
    np.testing.assert_allclose(ref.terms, want, rtol=1e-12, atol=0)
    np.testing.assert_allclose(np.asarray(ref), oracle.conv_fwd(x, w, nbr), rtol=0, atol=0)


def test_terms_of_weight_gradient_equal_brute_force():
    rng = np.random.default_rng(6)
    coords = rand_coords(rng, 40, 0, 4)
    nbr = oracle.kmap(coords, coords, 3, 1, 1, oracle.SUBM)
    x = rng.standard_normal((len(coords), 2))
    g = rng.standard_normal((len(coords), 3))
    ref = with_terms(oracle.conv_wgrad, x, g, nbr)
    want = np.zeros((27, 2, 3))
    for j in range(len(coords)):
        for k in range(27):
            i = nbr[j, k]
            if i >= 0:
                want[k] += np.abs(np.outer(x[i], g[j]))
    np.testing.assert_allclose(ref.terms, want, rtol=1e-12, atol=0)


def test_error_stats_percentiles_and_elements_without_terms():
    ref = np.zeros(101)
    got = np.arange(101, dtype=np.float64)        # |err| = 0 .. 100
    terms = np.full(101, 100.0)
    terms[0] = 0.0                                # an element with no term is left out
    s = error_stats(got, ref, terms)
    assert s["elements"] == 100
    assert s["rel_terms_max"] == 1.0
    assert np.isclose(s["rel_terms_p50"], np.percentile(np.arange(1, 101) / 100.0, 50))
    assert np.isclose(s["rel_terms_p99"], np.percentile(np.arange(1, 101) / 100.0, 99))
