"""Pins of the float64 oracle against what the pages and mathematics fix.

None of these calls the CUDA path. Each check is chosen so that a plausible
slip in the oracle (a dropped term, a wrong sign or index, a transposed
operand, an off-by-one in a mask or a running sum) fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy import stats

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------ hand-derived fixtures
def test_golden_attention_hand_example():
    g = _golden("attention_hand.json")
    q = np.array([g["q"]])
    out, lse = O.attend(q, np.array(g["keys"]), np.array(g["values"]),
                        np.ones((1, 3), bool), g["scale"])
    np.testing.assert_allclose(out[0], g["out"], rtol=0, atol=1e-12)
    assert abs(lse[0] - g["lse"]) < 1e-12


def test_golden_inverse_cdf_hand_cases():
    for c in _golden("inverse_cdf_hand.json")["cases"]:
        k, _ = O.inverse_cdf(np.array([c["weights"]], float), np.array([c["u"]]))
        assert int(k[0]) == c["k"], c


def test_golden_spec_sample_hand_cases():
    g = _golden("spec_sample_hand.json")
    tl = np.array([g["target_logits"]])
    dl = np.array([g["draft_logits"]])
    for c in g["cases"]:
        out, n_acc, _, _ = O.spec_sample(tl, dl, np.array([[c["draft_token"]]]),
                                         np.array([[c["u_accept"]]]), np.array([c["u_sample"]]),
                                         g["temperature"])
        assert out[0].tolist() == c["out"], c
        assert int(n_acc[0]) == c["n_acc"]


# ------------------------------------------------------------ paged cache helpers
def _random_paged(rng, S, Hkv, P, D, lens, extra_pages=3):
    n_pages = [-(-L // P) for L in lens]
    total = sum(n_pages) + extra_pages
    perm = rng.permutation(total)
    bt = np.full((S, max(n_pages)), -1, dtype=np.int64)
    off = 0
    for b, n in enumerate(n_pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    k = rng.standard_normal((total, Hkv, P, D))
    v = rng.standard_normal((total, Hkv, P, D))
    return k, v, bt, np.array(lens)


def _sdpa_reference(q, k, v, bt, lens, scale):
    """torch.nn.functional.scaled_dot_product_attention in float64 on the
    gathered contiguous history, causal with the rows at the last R positions."""
    S, R, Hq, D = q.shape
    Hkv, P = k.shape[1], k.shape[2]
    G = Hq // Hkv
    out = np.zeros_like(q)
    for b in range(S):
        L = int(lens[b])
        n = -(-L // P)
        idx = torch.as_tensor(bt[b, :n])
        kk = torch.as_tensor(k).index_select(0, idx).permute(1, 0, 2, 3).reshape(Hkv, n * P, D)[:, :L]
        vv = torch.as_tensor(v).index_select(0, idx).permute(1, 0, 2, 3).reshape(Hkv, n * P, D)[:, :L]
        kk = kk.repeat_interleave(G, dim=0)
        vv = vv.repeat_interleave(G, dim=0)
        qq = torch.as_tensor(q[b]).permute(1, 0, 2)                      # [Hq, R, D]
        pos_q = torch.arange(L - R, L)[:, None]
        mask = torch.arange(L)[None, :] <= pos_q                          # [R, L]
        o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale)
        out[b] = o.permute(1, 0, 2).numpy()
    return out


@pytest.mark.parametrize("P,D,G,R", [(16, 64, 4, 4), (64, 128, 4, 5), (16, 32, 2, 1), (64, 16, 5, 9)])
def test_paged_attention_matches_sdpa(P, D, G, R):
    rng = np.random.default_rng(P * 1000 + D + G + R)
    Hkv, S = 2, 3
    lens = [R, P * 3 + 5, P * 2]
    k, v, bt, lens = _random_paged(rng, S, Hkv, P, D, lens)
    q = rng.standard_normal((S, R, G * Hkv, D))
    scale = 1 / math.sqrt(D)
    out, lse = O.verify_attn(q, k, v, bt, lens, scale)
    ref = _sdpa_reference(q, k, v, bt, lens, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_verify_rows_equal_decode_at_shorter_lengths():
    rng = np.random.default_rng(7)
    P, D, Hkv, G, R = 16, 32, 2, 3, 5
    k, v, bt, lens = _random_paged(rng, 2, Hkv, P, D, [70, 41])
    q = rng.standard_normal((2, R, G * Hkv, D))
    out, lse = O.verify_attn(q, k, v, bt, lens, 0.3)
    for r in range(R):
        lens_r = lens - R + r + 1
        o1, l1 = O.dense_decode(q[:, r], k, v, bt, lens_r, 0.3)
        np.testing.assert_allclose(out[:, r], o1, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[:, r], l1, rtol=1e-12, atol=1e-13)


def test_attention_closed_forms():
    rng = np.random.default_rng(3)
    P, D, Hkv, G = 16, 8, 1, 2
    k, v, bt, lens = _random_paged(rng, 2, Hkv, P, D, [37, 1])
    q = np.zeros((2, G * Hkv, D))
    out, lse = O.dense_decode(q, k, v, bt, lens, 1.0)
    # q = 0: uniform weights -> mean of the valid values; lse = log(n_valid)
    for b, L in enumerate(lens):
        vals = np.concatenate([v[bt[b, i], 0, :min(P, L - i * P)] for i in range(-(-L // P))])
        np.testing.assert_allclose(out[b], np.broadcast_to(vals.mean(0), (G, D)), atol=1e-12)
        np.testing.assert_allclose(lse[b], math.log(L), atol=1e-12)
    # a single valid key returns its value whatever the query
    q = rng.standard_normal((2, G, D))
    out, _ = O.dense_decode(q, k, v, bt, lens, 1.0)
    np.testing.assert_allclose(out[1], np.broadcast_to(v[bt[1, 0], 0, 0], (G, D)), atol=1e-12)
    # a dominant key takes (almost) all the weight
    k2 = k.copy()
    k2[bt[0, 1], 0, 3] = q[0, 0] * 50
    out, _ = O.dense_decode(q, k2, v, bt, lens, 1.0)
    np.testing.assert_allclose(out[0, 0], v[bt[0, 1], 0, 3], atol=1e-9)


def test_sparse_equals_dense_at_full_budget():
    rng = np.random.default_rng(11)
    P, D, Hkv, G = 16, 16, 2, 4
    k, v, bt, lens = _random_paged(rng, 3, Hkv, P, D, [100, 16, 33])
    q = rng.standard_normal((3, G * Hkv, D))
    kmin, kmax = O.page_summaries(k, bt, lens, P)
    n_max = max(-(-int(L) // P) for L in lens)
    sel, _ = O.sparse_draft_select(q, kmin, kmax, bt, lens, P, n_max, G)
    o_s, l_s = O.sparse_draft_attn(q, k, v, bt, lens, sel, 0.25)
    o_d, l_d = O.dense_decode(q, k, v, bt, lens, 0.25)
    np.testing.assert_allclose(o_s, o_d, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l_s, l_d, rtol=1e-13, atol=1e-14)
    # with a smaller budget the sparse output differs (the pin is not vacuous)
    sel2, _ = O.sparse_draft_select(q, kmin, kmax, bt, lens, P, 2, G)
    o2, _ = O.sparse_draft_attn(q, k, v, bt, lens, sel2, 0.25)
    assert np.abs(o2[0] - o_d[0]).max() > 1e-3


# ------------------------------------------------------------ summaries and scores
def test_summaries_bound_and_attain():
    rng = np.random.default_rng(5)
    P, D, Hkv = 16, 8, 2
    k, v, bt, lens = _random_paged(rng, 2, Hkv, P, D, [45, 16])
    # garbage beyond the context must not leak into the tail summary
    k[bt[0, 2], :, 45 - 32:, :] = 1e30
    kmin, kmax = O.page_summaries(k, bt, lens, P)
    for b, L in enumerate(lens):
        for i in range(-(-int(L) // P)):
            ph = bt[b, i]
            valid = min(P, int(L) - i * P)
            tile = k[ph, :, :valid, :]
            assert np.all(kmin[ph][:, None, :] <= tile) and np.all(tile <= kmax[ph][:, None, :])
            assert np.all(np.any(tile == kmin[ph][:, None, :], axis=1))
            assert np.all(np.any(tile == kmax[ph][:, None, :], axis=1))
    assert np.all(kmax[bt[0, 2]] < 1e29)
    # tail-only mode rewrites only each sequence's last page
    k3 = k.copy()
    k3[bt[0, 0]] += 5.0
    k3[bt[0, 2], :, 0, :] -= 7.0
    tmin, tmax = O.page_summaries(k3, bt, lens, P, tail_only=True, kmin=kmin, kmax=kmax)
    np.testing.assert_array_equal(tmin[bt[0, 0]], kmin[bt[0, 0]])
    np.testing.assert_array_equal(tmin[bt[0, 2]], k3[bt[0, 2], :, :13, :].min(axis=1))


def test_quest_score_bounds_every_token():
    rng = np.random.default_rng(9)
    P, D, Hkv, G = 16, 16, 2, 3
    k, v, bt, lens = _random_paged(rng, 1, Hkv, P, D, [75])
    q = rng.standard_normal((G * Hkv, D))
    kmin, kmax = O.page_summaries(k, bt, lens, P)
    n = 5
    sc = O.page_scores(q, kmin[bt[0, :n]], kmax[bt[0, :n]], G)
    for h in range(Hkv):
        for i in range(n):
            valid = min(P, 75 - i * P)
            toks = k[bt[0, i], h, :valid]
            group_dot = (q[h * G:(h + 1) * G] @ toks.T).sum(axis=0)   # sum over group
            assert np.all(group_dot <= sc[h, i] + 1e-12)
    # the bound is tight for a page holding a single token
    k1, _, bt1, lens1 = _random_paged(rng, 1, 1, P, D, [1])
    kmn, kmx = O.page_summaries(k1, bt1, lens1, P)
    q1 = rng.standard_normal((2, D))
    s = O.page_scores(q1, kmn[bt1[0, :1]], kmx[bt1[0, :1]], 2)
    assert abs(s[0, 0] - (q1 @ k1[bt1[0, 0], 0, 0]).sum()) < 1e-12


def test_top_pages_equal_exhaustive_subset_search():
    for seed in range(20):
        rng = np.random.default_rng(seed)
        s = rng.standard_normal(16)
        chosen, gap = O.select_top_pages(s, 4)
        best = max(itertools.combinations(range(16), 4), key=lambda c: sum(s[list(c)]))
        assert chosen.tolist() == sorted(best)
        assert gap > 0


def test_top_pages_ties_and_small_n():
    chosen, gap = O.select_top_pages(np.array([1.0, 3.0, 3.0, 2.0, 3.0]), 2)
    assert chosen.tolist() == [1, 2] and gap == 0.0
    chosen, _ = O.select_top_pages(np.array([5.0, 5.0, 5.0]), 1)
    assert chosen.tolist() == [0]
    chosen, gap = O.select_top_pages(np.array([0.5, -1.0]), 4)
    assert chosen.tolist() == [0, 1] and gap == np.inf


# ------------------------------------------------------------ sampling
def test_q_equals_p_accepts_every_draft():
    for seed in range(8):
        rng = np.random.default_rng(seed)
        S, gamma, V = 6, 5, 300
        t = 2 * rng.standard_normal((S, gamma + 1, V))
        d = t[:, :gamma].copy()
        x, _ = O.sample_rows(d.reshape(-1, V), rng.random(S * gamma), 0.8)
        out, n_acc, _, _ = O.spec_sample(t, d, x.reshape(S, gamma), rng.random((S, gamma)),
                                         rng.random((S, gamma + 1)), 0.8)
        assert np.all(n_acc == gamma)
        assert np.array_equal(out[:, :gamma], x.reshape(S, gamma))


def _fixed_dists(V, gamma, seed):
    rng = np.random.default_rng(seed)
    t = 1.5 * rng.standard_normal((gamma + 1, V))
    d = t[:gamma] + 1.0 * rng.standard_normal((gamma, V))
    return t, d


def _run_trials(t, d, n, seed, chunk=200_000):
    """n independent rounds with the same logits; returns out_tokens, n_acc."""
    rng = np.random.default_rng(seed)
    R, V = t.shape
    gamma = R - 1
    outs, accs = [], []
    for start in range(0, n, chunk):
        m = min(chunk, n - start)
        tl = np.broadcast_to(t, (m, R, V))
        dl = np.broadcast_to(d, (m, gamma, V))
        x, _ = O.sample_rows(dl.reshape(-1, V), rng.random(m * gamma), 1.0)
        out, n_acc, _, _ = O.spec_sample(tl, dl, x.reshape(m, gamma), rng.random((m, gamma)),
                                         rng.random((m, R)), 1.0)
        outs.append(out)
        accs.append(n_acc)
    return np.concatenate(outs), np.concatenate(accs)


@pytest.fixture(scope="module")
def chi_trials():
    t, d = _fixed_dists(16, 3, 123)
    out, n_acc = _run_trials(t, d, 1_000_000, 321)
    return t, d, out, n_acc


def test_committed_tokens_follow_p_chi_square(chi_trials):
    t, d, out, n_acc = chi_trials
    p = O.softmax_t(t, 1.0)
    crit = stats.chi2.ppf(0.999, 15)            # 37.70
    for j in range(t.shape[0]):
        reached = n_acc >= j
        toks = out[reached, j]
        counts = np.bincount(toks, minlength=16)
        exp = p[j] * reached.sum()
        chi = ((counts - exp) ** 2 / exp).sum()
        assert chi < crit, (j, chi)


def test_committed_tokens_chi_square_detects_a_wrong_rule(chi_trials):
    """The same statistic rejects the sparse policy q itself (the test has power)."""
    t, d, out, n_acc = chi_trials
    q = O.softmax_t(d, 1.0)
    toks = out[:, 0]
    exp = q[0] * len(toks)
    chi = ((np.bincount(toks, minlength=16) - exp) ** 2 / exp).sum()
    assert chi > stats.chi2.ppf(0.999, 15)


def test_acceptance_rate_closed_form(chi_trials):
    t, d, out, n_acc = chi_trials
    p = O.softmax_t(t, 1.0)
    q = O.softmax_t(d, 1.0)
    alpha = np.minimum(p[0], q[0]).sum()
    n = len(n_acc)
    rate = (n_acc >= 1).mean()
    sigma = math.sqrt(alpha * (1 - alpha) / n)
    assert abs(rate - alpha) < 4 * sigma
    # second position, conditional on reaching it
    alpha1 = np.minimum(p[1], q[1]).sum()
    reached = n_acc >= 1
    rate1 = (n_acc[reached] >= 2).mean()
    assert abs(rate1 - alpha1) < 4 * math.sqrt(alpha1 * (1 - alpha1) / reached.sum())


def _exact_outcomes(p, q):
    """Exact distribution of committed sequences, with rational arithmetic:
    at each draft position the draft x ~ q_i is kept with probability
    min(1, p_i(x)/q_i(x)); otherwise a token from the normalised residual ends
    the round; after gamma kept drafts the bonus token comes from p_gamma."""
    gamma = len(q)
    V = len(p[0])
    dist = {}

    def walk(i, prefix, prob):
        if i == gamma:
            for y in range(V):
                dist[prefix + (y,)] = dist.get(prefix + (y,), 0) + prob * p[gamma][y]
            return
        resid = [max(p[i][y] - q[i][y], Fraction(0)) for y in range(V)]
        rs = sum(resid)
        reject = Fraction(0)
        for x in range(V):
            a = min(Fraction(1), p[i][x] / q[i][x])
            walk(i + 1, prefix + (x,), prob * q[i][x] * a)
            reject += q[i][x] * (1 - a)
        for y in range(V):
            if rs > 0:
                dist[prefix + (y,)] = dist.get(prefix + (y,), 0) + prob * reject * resid[y] / rs

    walk(0, (), Fraction(1))
    return dist


def test_exact_enumeration_rational():
    # p and q with integer weights, so that the logits ln(w) give these exact rationals
    pw = [[1, 2, 3], [4, 1, 1], [2, 2, 1]]
    qw = [[3, 2, 1], [1, 1, 4]]
    p = [[Fraction(w, sum(r)) for w in r] for r in pw]
    q = [[Fraction(w, sum(r)) for w in r] for r in qw]
    dist = _exact_outcomes(p, q)
    assert sum(dist.values()) == 1
    # every committed position follows p exactly, conditional on being reached
    for j in range(3):
        reach = sum(pr for seq, pr in dist.items() if len(seq) > j)
        for y in range(3):
            mass = sum(pr for seq, pr in dist.items() if len(seq) > j and seq[j] == y)
            assert mass == reach * p[j][y]
    # the oracle's empirical outcome histogram matches the exact distribution
    t = np.log(np.array(pw, float))
    d = np.log(np.array(qw, float))
    out, n_acc = _run_trials(t, d, 1_000_000, 77)
    keys = sorted(dist)
    index = {k: i for i, k in enumerate(keys)}
    counts = np.zeros(len(keys))
    lens = n_acc + 1
    codes = {}
    for L in (1, 2, 3):
        sel = lens == L
        sub = out[sel, :L]
        uniq, cnt = np.unique(sub, axis=0, return_counts=True)
        for row, c in zip(uniq, cnt):
            counts[index[tuple(int(v) for v in row)]] += c
            codes[tuple(int(v) for v in row)] = c
    exp = np.array([float(dist[k]) for k in keys]) * len(n_acc)
    keep = exp > 0
    assert counts[~keep].sum() == 0
    chi = ((counts[keep] - exp[keep]) ** 2 / exp[keep]).sum()
    assert chi < stats.chi2.ppf(0.999, keep.sum() - 1), chi
