"""Pins of the oracle's tree verification (the ai.info SpecRoll page:
concurrency-aware node budget, exact rejection sampling with the residual
fallback at every visited node): a chain tree reduces to ordinary
speculative sampling and to causal verification; the tree mask attention
equals SDPA with an explicit ancestor mask; the committed tokens follow the
target policy exactly (rational enumeration) and empirically (chi-square
over a two-level tree whose siblings repeat tokens). None of these calls the
CUDA path."""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy import stats

import oracle as O


def test_node_budget_formula():
    assert O.node_budget(600, 16, 2, 16) == 16          # floor(600 / 16) = 37, clipped to 16
    assert O.node_budget(600, 100, 2, 16) == 6
    assert O.node_budget(600, 1000, 2, 16) == 2         # clipped up to N_min
    assert O.node_budget(64, 8, 1, 64) == 8


def test_tree_shapes_and_masks():
    par = O.build_tree(9, [2, 2, 1])
    assert par.tolist() == [-1, 0, 0, 1, 1, 2, 2, 3, 4]
    m = O.tree_ancestor_masks(par)
    assert m[0] == 0b1 and m[3] == 0b1011 and m[8] == (1 | 2 | 16 | 256)
    assert O.tree_ancestor_masks(O.chain_parents(5)) == [1, 3, 7, 15, 31]


def test_chain_tree_is_ordinary_speculative_sampling():
    rng = np.random.default_rng(0)
    for _ in range(200):
        S, g, V = 3, int(rng.integers(1, 7)), 50
        R = g + 1
        t = 2 * rng.standard_normal((S, R, V))
        d = t + rng.standard_normal((S, R, V))
        x, _ = O.sample_rows(d[:, :g].reshape(-1, V), rng.random(S * g), 0.9)
        x = x.reshape(S, g)
        ua, us = rng.random((S, g)), rng.random((S, R))
        out, n_acc, _, _ = O.spec_sample(t, d[:, :g], x, ua, us, 0.9)
        tokens = np.concatenate([np.zeros((S, 1), np.int64), x], axis=1)       # node i + 1 carries draft x_i
        ua_t = np.concatenate([np.zeros((S, 1)), ua], axis=1)                  # node c is tested with u_accept[c]
        par = np.broadcast_to(O.chain_parents(R), (S, R))
        out_t, n_t, path, _, _ = O.tree_spec_sample(t, d, tokens, par, ua_t, us, 0.9)
        assert np.array_equal(out_t, out) and np.array_equal(n_t, n_acc)
        for b in range(S):
            assert path[b, :n_t[b]].tolist() == list(range(1, n_t[b] + 1))


def _paged(rng, S, H, P, D, lens):
    n_pages = [-(-L // P) for L in lens]
    total = sum(n_pages) + 2
    perm = rng.permutation(total)
    bt = np.full((S, max(n_pages)), -1, dtype=np.int64)
    off = 0
    for b, n in enumerate(n_pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    return rng.standard_normal((total, H, P, D)), rng.standard_normal((total, H, P, D)), bt, np.array(lens)


@pytest.mark.parametrize("R,lens", [(7, [50, 23]), (64, [64, 90])])
def test_tree_attention_equals_masked_sdpa_and_chain_equals_verify(R, lens):
    """R = 64: the widest tree, every bit of a 64-bit ancestor mask in use."""
    rng = np.random.default_rng(1)
    P, D, H, G = 16, 32, 2, 3
    S = 2
    k, v, bt, lens = _paged(rng, S, H, P, D, lens)
    q = rng.standard_normal((S, R, G * H, D))
    if R == 7:
        par = np.stack([O.build_tree(R, [3, 1]), O.build_tree(R, [1, 2])])
    else:
        par = np.stack([O.build_tree(R, [2]), np.array([-1] + [int(rng.integers(0, c)) for c in range(1, R)])])
    out, _ = O.tree_verify_attn(q, k, v, bt, lens, par, 0.2)
    for b in range(S):
        L = int(lens[b])
        masks = O.tree_ancestor_masks(par[b])
        n = -(-L // P)
        kk = torch.as_tensor(k).index_select(0, torch.as_tensor(bt[b, :n])).permute(1, 0, 2, 3).reshape(H, n * P, D)[:, :L]
        vv = torch.as_tensor(v).index_select(0, torch.as_tensor(bt[b, :n])).permute(1, 0, 2, 3).reshape(H, n * P, D)[:, :L]
        allow = torch.zeros((R, L), dtype=torch.bool)
        allow[:, :L - R] = True
        for i in range(R):
            for j in range(R):
                allow[i, L - R + j] = bool((masks[i] >> j) & 1)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.as_tensor(q[b]).permute(1, 0, 2), kk.repeat_interleave(G, 0), vv.repeat_interleave(G, 0),
            attn_mask=allow, scale=0.2)
        np.testing.assert_allclose(out[b], ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    chain = np.broadcast_to(O.chain_parents(R), (S, R))
    o1, l1 = O.tree_verify_attn(q, k, v, bt, lens, chain, 0.2)
    o2, l2 = O.verify_attn(q, k, v, bt, lens, 0.2)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-14)


def _first_token_distribution(p, q, k):
    """Exact distribution of the first committed token of a root with k
    children drawn i.i.d. from q (rational arithmetic), the multi-draft rule:
    child j accepted with probability min(1, p'(x_j)/q(x_j)), p' replaced by
    its normalised residual after every rejection, a draw from p' at the end."""
    V = len(p)
    dist = [Fraction(0)] * V
    for xs in itertools.product(range(V), repeat=k):
        w = Fraction(1)
        for x in xs:
            w *= q[x]
        pr = list(p)
        reach = w
        for x in xs:
            a = min(Fraction(1), pr[x] / q[x])
            dist[x] += reach * a
            reach *= 1 - a
            res = [max(pr[y] - q[y], Fraction(0)) for y in range(V)]
            s = sum(res)
            if s > 0:
                pr = [r / s for r in res]
        for y in range(V):
            dist[y] += reach * pr[y]
    return dist


def test_multi_draft_rule_is_exact_by_enumeration():
    p = [Fraction(1, 6), Fraction(2, 6), Fraction(3, 6)]
    q = [Fraction(3, 6), Fraction(2, 6), Fraction(1, 6)]
    for k in (1, 2, 3):
        assert _first_token_distribution(p, q, k) == p


def _two_level(rng, V):
    t_root = 1.2 * rng.standard_normal(V)
    d_root = t_root + rng.standard_normal(V)
    t_child = 1.2 * rng.standard_normal((V, V))          # the target after token a: row a
    d_child = t_child + rng.standard_normal((V, V))
    return t_root, d_root, t_child, d_child


def test_committed_tokens_follow_p_over_a_two_level_tree():
    """Root with 3 children drawn i.i.d. from q_root (tokens may repeat), each
    child with 2 children drawn from its own q: the first committed token
    follows p_root, the second (when reached) follows the target after the
    first. Chi-square over 200K rounds, V = 8."""
    V, n = 8, 200_000
    rng = np.random.default_rng(5)
    t_root, d_root, t_child, d_child = _two_level(rng, V)
    par = O.build_tree(10, [3, 2])                                   # 1 + 3 + 6 nodes
    R = len(par)
    T = 1.0
    qr = O.softmax_t(d_root, T)
    first, second = [], []
    chunk = 20_000
    for s0 in range(0, n, chunk):
        m = chunk
        tokens = np.zeros((m, R), dtype=np.int64)
        # children of the root from q_root, grandchildren from q after their parent's token
        tokens[:, 1:4] = np.searchsorted(np.cumsum(qr), rng.random((m, 3)) * qr.sum(), side="right").clip(0, V - 1)
        for c in range(4, R):
            a = tokens[:, par[c]]
            qa = O.softmax_t(d_child[a], T)
            tokens[:, c] = (np.cumsum(qa, axis=1) <= (rng.random(m) * qa.sum(axis=1))[:, None]).sum(axis=1).clip(0, V - 1)
        tl = np.empty((m, R, V))
        dl = np.empty((m, R, V))
        tl[:, 0], dl[:, 0] = t_root, d_root
        for c in range(1, R):
            tl[:, c] = t_child[tokens[:, c]]
            dl[:, c] = d_child[tokens[:, c]]
        out, n_acc, _, _, _ = O.tree_spec_sample(tl, dl, tokens, np.broadcast_to(par, (m, R)), rng.random((m, R)),
                                                 rng.random((m, R)), T)
        first.append(out[:, 0])
        second.append(np.where(n_acc >= 1, out[:, 1], -1))
    first = np.concatenate(first)
    second = np.concatenate(second)
    crit = stats.chi2.ppf(0.999, V - 1)
    p_root = O.softmax_t(t_root, T)
    chi = ((np.bincount(first, minlength=V) - p_root * n) ** 2 / (p_root * n)).sum()
    assert chi < crit, chi
    # power: the same statistic rejects q_root
    chi_q = ((np.bincount(first, minlength=V) - qr * n) ** 2 / (qr * n)).sum()
    assert chi_q > crit
    for a in range(V):
        sel = (first == a) & (second >= 0)
        if sel.sum() < 2000:
            continue
        pa = O.softmax_t(t_child[a], T)
        c2 = ((np.bincount(second[sel], minlength=V) - pa * sel.sum()) ** 2 / (pa * sel.sum())).sum()
        assert c2 < crit, (a, c2)
