"""Identities the GPU kernels use in place of the oracle's literal formulas.

Each is exact in real arithmetic; these tests check them on exact rationals
(or exactly representable floats) so that a kernel that relies on one is
computing the oracle's quantity up to rounding.

- Page scores (Quest bound, summed over the G query heads of a KV head):
  sum_g max(q_g a, q_g b) = A max(a, b) + B min(a, b) per channel, with
  A = sum_g max(q_g, 0) and B = sum_g min(q_g, 0), for any a, b (the
  selector folds the G rows into A and B once).
- Inverse-CDF draws are invariant under a common positive scale of the
  weights, so the sampler may shift each chunk by its own maximum and merge
  the chunk sums by exact powers of two.
- The online normaliser: a running maximum with the partial sum rescaled when
  it grows gives sum_i exp(x_i - max) (the sampler's statistics pass).
"""
from fractions import Fraction

import numpy as np

from oracle import s3r_oracle as O


def test_selector_fold_of_the_query_heads_is_exact():
    rng = np.random.default_rng(3)
    for _ in range(400):
        G = int(rng.integers(1, 9))
        q = [Fraction(int(v), int(rng.integers(1, 64))) for v in rng.integers(-50, 51, G)]
        a = Fraction(int(rng.integers(-80, 81)), int(rng.integers(1, 32)))
        b = Fraction(int(rng.integers(-80, 81)), int(rng.integers(1, 32)))   # a > b allowed too
        direct = sum(max(qg * a, qg * b) for qg in q)
        A = sum(max(qg, 0) for qg in q)
        B = sum(min(qg, 0) for qg in q)
        assert direct == A * max(a, b) + B * min(a, b)


def test_selector_fold_matches_the_oracle_page_scores():
    rng = np.random.default_rng(4)
    G, D, n = 4, 128, 37
    q = rng.normal(size=(G, D)).astype(np.float32).astype(np.float64)
    lo = rng.normal(size=(n, D)).astype(np.float32).astype(np.float64)
    hi = lo + np.abs(rng.normal(size=(n, D))).astype(np.float32).astype(np.float64)
    ref = O.page_scores(q, lo[:, None, :], hi[:, None, :], G)[0]
    A = np.maximum(q, 0).sum(axis=0)
    B = np.minimum(q, 0).sum(axis=0)
    fold = (A * np.maximum(lo, hi) + B * np.minimum(lo, hi)).sum(axis=1)
    assert np.allclose(fold, ref, rtol=1e-13, atol=0)


def test_inverse_cdf_is_invariant_under_power_of_two_scales():
    rng = np.random.default_rng(5)
    for _ in range(50):
        V = int(rng.integers(2, 300))
        w = rng.random(V) * (rng.random(V) > 0.3)
        if w.sum() == 0:
            continue
        u = rng.random(7)
        k0, _ = O.inverse_cdf(np.tile(w, (7, 1)), u)
        for e in (-600, -37, 0, 11, 700):
            k1, _ = O.inverse_cdf(np.tile(np.ldexp(w, e), (7, 1)), u)        # exact scaling
            assert np.array_equal(k0, k1)


def test_online_normaliser_equals_the_direct_sum():
    rng = np.random.default_rng(6)
    for _ in range(50):
        x = rng.normal(0.0, 3.0, int(rng.integers(1, 500)))
        m, s = -np.inf, 0.0
        for v in x:                        # one element at a time, maximum first seen late
            if v > m:
                s = s * np.exp(m - v) if np.isfinite(m) else 0.0
                m = v
            s += np.exp(v - m)
        direct = np.exp(x - x.max()).sum()
        assert m == x.max()
        assert abs(s - direct) <= 1e-12 * direct
