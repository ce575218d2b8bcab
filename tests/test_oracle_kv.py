"""Pins of the oracle's KV-cache upkeep (kv_append, kv_rollback) against an
independent model: one dense array of rows per sequence, indexed by
position, with no pages and no block table. After every operation the paged
cache read through its block table must equal the dense rows, the lengths
must agree, and every page a sequence uses must carry the min / max of its
valid tokens (checked against the dense rows, not the oracle's page loop).
None of these calls the CUDA path."""
import numpy as np
import pytest

import oracle as O


def _paged(rng, S, H, P, D, lens, cap_pages):
    total = S * cap_pages + 3
    perm = rng.permutation(total)
    bt = perm[:S * cap_pages].reshape(S, cap_pages).astype(np.int64)
    K = rng.standard_normal((total, H, P, D))
    V = rng.standard_normal((total, H, P, D))
    return K, V, bt


def _dense_rows(cache, bt, b, L, P):
    return np.stack([cache[bt[b, t // P], :, t % P, :] for t in range(L)])      # [L, H, D]


def _check(K, V, bt, lens, kmin, kmax, dense_k, dense_v, P):
    for b, L in enumerate(lens):
        L = int(L)
        assert L == len(dense_k[b])
        np.testing.assert_array_equal(_dense_rows(K, bt, b, L, P), np.stack(dense_k[b]))
        np.testing.assert_array_equal(_dense_rows(V, bt, b, L, P), np.stack(dense_v[b]))
        rows = np.stack(dense_k[b])
        for i in range(-(-L // P)):
            seg = rows[i * P:min(L, (i + 1) * P)]                 # this page's valid tokens, from the dense model
            np.testing.assert_array_equal(kmin[bt[b, i]], seg.min(axis=0))
            np.testing.assert_array_equal(kmax[bt[b, i]], seg.max(axis=0))


@pytest.mark.parametrize("P,seed", [(16, 0), (16, 1), (64, 2), (4, 3)])
def test_append_overwrite_rollback_match_dense_model(P, seed):
    rng = np.random.default_rng(seed)
    S, H, D, cap = 3, 2, 8, 12
    lens = rng.integers(1, 3 * P, size=S)
    K, V, bt = _paged(rng, S, H, P, D, lens, cap)
    dense_k = [[K[bt[b, t // P], :, t % P, :].copy() for t in range(int(lens[b]))] for b in range(S)]
    dense_v = [[V[bt[b, t // P], :, t % P, :].copy() for t in range(int(lens[b]))] for b in range(S)]
    kmin, kmax = O.page_summaries(K, bt, lens, P)
    _check(K, V, bt, lens, kmin, kmax, dense_k, dense_v, P)
    for rnd in range(6):
        gamma = int(rng.integers(1, 6))
        R = gamma + 1
        # gamma draft steps, one row each, appended at the end
        for i in range(gamma):
            kn = rng.standard_normal((S, 1, H, D))
            vn = rng.standard_normal((S, 1, H, D))
            K, V, lens, kmin, kmax = O.kv_append(K, V, bt, lens, kn, vn, 0, P, kmin, kmax)
            for b in range(S):
                dense_k[b].append(kn[b, 0])
                dense_v[b].append(vn[b, 0])
            _check(K, V, bt, lens, kmin, kmax, dense_k, dense_v, P)
        # verification: R rows over the round's positions (the gamma drafts and one more)
        kn = rng.standard_normal((S, R, H, D))
        vn = rng.standard_normal((S, R, H, D))
        K, V, lens, kmin, kmax = O.kv_append(K, V, bt, lens, kn, vn, gamma, P, kmin, kmax)
        for b in range(S):
            del dense_k[b][-gamma:]
            del dense_v[b][-gamma:]
            dense_k[b].extend(kn[b])
            dense_v[b].extend(vn[b])
        _check(K, V, bt, lens, kmin, kmax, dense_k, dense_v, P)
        # commit: the round's first position plus the accepted drafts stay
        n_acc = rng.integers(0, gamma + 1, size=S)
        lens, kmin, kmax = O.kv_rollback(K, bt, lens, n_acc, R, P, kmin, kmax)
        for b in range(S):
            keep = len(dense_k[b]) - R + int(n_acc[b]) + 1
            del dense_k[b][keep:]
            del dense_v[b][keep:]
        _check(K, V, bt, lens, kmin, kmax, dense_k, dense_v, P)


def test_rollback_extremes():
    """All drafts accepted keeps every position; none accepted keeps only the
    round's first position; the refreshed tail forgets the dropped tokens."""
    rng = np.random.default_rng(9)
    P, H, D = 8, 1, 4
    K = rng.standard_normal((6, H, P, D))
    bt = np.array([[0, 1, 2], [3, 4, 5]])
    lens = np.array([20, 9])
    kmin, kmax = O.page_summaries(K, bt, lens, P)
    R = 5
    l2, _, _ = O.kv_rollback(K, bt, lens, np.array([4, 4]), R, P, kmin, kmax)
    assert l2.tolist() == [20, 9]
    l3, mn, mx = O.kv_rollback(K, bt, lens, np.array([0, 0]), R, P, kmin, kmax)
    assert l3.tolist() == [16, 5]
    # sequence 0 now ends exactly at a page boundary: page 1 (tokens 8..15) full
    np.testing.assert_array_equal(mn[1], K[1, :, :8, :].min(axis=1))
    # sequence 1's tail page 0 now holds tokens 0..4 only
    np.testing.assert_array_equal(mx[3], K[3, :, :5, :].max(axis=1))


def test_append_nothing_changes_nothing():
    rng = np.random.default_rng(4)
    P, H, D = 16, 2, 8
    K = rng.standard_normal((4, H, P, D))
    V = rng.standard_normal((4, H, P, D))
    bt = np.array([[0, 1], [2, 3]])
    lens = np.array([17, 5])
    kmin, kmax = O.page_summaries(K, bt, lens, P)
    K2, V2, l2, mn, mx = O.kv_append(K, V, bt, lens, np.zeros((2, 0, H, D)), np.zeros((2, 0, H, D)), 0, P, kmin, kmax)
    np.testing.assert_array_equal(K2, K)
    assert l2.tolist() == [17, 5]
    np.testing.assert_array_equal(mn, kmin)
