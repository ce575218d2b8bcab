"""Pins of the draft-length policy oracle (oracle/gamma_policy.py): the
expected committed tokens against a Monte Carlo of the oracle's speculative
sampling with a known per-position acceptance, the weighted acceptance
estimate, the choice against brute force, and the roofline cost model's
regimes. None of these calls the CUDA path."""
import math

import numpy as np
import pytest

import oracle as O
from oracle import gamma_policy as GP


def _dists(alpha, V=4):
    """Target p = [alpha, 1 - alpha, 0, ...] and draft q = the first token
    only: sum_x min(p, q) = alpha, so every position accepts with
    probability alpha."""
    with np.errstate(divide="ignore"):
        t = np.log(np.array([alpha, 1 - alpha] + [0.0] * (V - 2)))
        d = np.log(np.array([1.0] + [0.0] * (V - 1)))
    return t, d


@pytest.mark.parametrize("alpha,gamma", [(0.3, 3), (0.7, 5), (0.9, 8), (0.5, 1)])
def test_expected_tokens_matches_simulated_rounds(alpha, gamma):
    t, d = _dists(alpha)
    n = 100_000
    rng = np.random.default_rng(int(alpha * 100) + gamma)
    R, V = gamma + 1, len(t)
    tl = np.broadcast_to(t, (n, R, V))
    dl = np.broadcast_to(d, (n, gamma, V))
    x, _ = O.sample_rows(dl.reshape(-1, V), rng.random(n * gamma), 1.0)
    _, n_acc, _, _ = O.spec_sample(tl, dl, x.reshape(n, gamma), rng.random((n, gamma)), rng.random((n, R)), 1.0)
    committed = n_acc + 1
    e = GP.expected_tokens(alpha, gamma)
    sd = committed.std() / math.sqrt(n)
    assert abs(committed.mean() - e) < 4 * sd + 1e-12
    # the accepted / tested ratio estimates alpha
    tested = np.minimum(n_acc + 1, gamma)
    assert abs(n_acc.sum() / tested.sum() - alpha) < 4 * math.sqrt(alpha * (1 - alpha) / tested.sum())


def test_expected_tokens_special_cases():
    assert GP.expected_tokens(0.0, 7) == 1.0
    assert GP.expected_tokens(1.0, 7) == 8.0
    assert GP.expected_tokens(0.5, 1) == 1.5
    assert abs(GP.expected_tokens(0.6, 4) - (1 - 0.6 ** 5) / 0.4) < 1e-14
    assert [GP.tests_made(k, 4) for k in range(5)] == [1, 2, 3, 4, 4]


def test_weighted_acceptance_estimate():
    p = GP.Policy(8, 0.9, 0.5, 4.0, [1.0] * 9)
    assert p.alpha() == 0.5                                   # the prior alone
    for _ in range(400):                                      # rounds of 4 sequences, 3 of 4 drafts accepted
        p.update([3, 3, 3, 3], 4)
    assert abs(p.alpha() - 0.75) < 1e-12
    q = GP.Policy(8, 0.0, 0.5, 4.0, [1.0] * 9)                # no memory: the last round only
    q.update([4, 4], 4)
    q.update([0, 1], 4)
    assert q.alpha() == 1 / 3


def test_choice_is_the_best_rate_and_toggles_drafting_off():
    rng = np.random.default_rng(3)
    for _ in range(200):
        gmax = int(rng.integers(1, 12))
        cost = list(rng.uniform(1.0, 5.0, gmax + 1))
        p = GP.Policy(gmax, 0.8, rng.uniform(0, 1), 10.0, cost)
        g, r = p.choose()
        rates = [p.rate(k) for k in range(gmax + 1)]
        assert r == max(rates) and g == rates.index(max(rates))
    # a plain decode step far cheaper than a round: drafting off
    p = GP.Policy(8, 0.8, 0.6, 10.0, [0.1] + [1.0] * 8)
    assert p.choose()[0] == 0
    # free drafts and near-certain acceptance: the longest round
    p = GP.Policy(8, 0.8, 0.99, 1e6, [1.0] * 9)
    assert p.choose()[0] == 8


def test_round_cost_regimes():
    args = dict(q_heads=32, kv_heads=8, head_dim=128, page_size=64, kv_bytes=2, mean_context=16384,
                budget_pages=32, vocab=151936, logit_bytes=2, hbm_gbs=6500.0, tensor_tflops=1500.0)
    att = dict(q_heads=32, kv_heads=8, head_dim=128, kv_bytes=2, mean_context=16384)
    # memory-bound (16 sequences): dense attention costs the same for 2 or 9 rows, the
    # bytes of every key and value over the bandwidth
    a2 = GP.attend_cost_us(16, rows=2, hbm_gbs=6500.0, tensor_tflops=1500.0, **att)
    a9 = GP.attend_cost_us(16, rows=9, hbm_gbs=6500.0, tensor_tflops=1500.0, **att)
    assert a2 == a9 == pytest.approx(16 * 2 * 8 * 128 * 2 * 16384 / 6500e9 * 1e6)
    # with a low tensor peak it turns compute-bound and grows with the rows
    s2 = GP.attend_cost_us(16, rows=2, hbm_gbs=6500.0, tensor_tflops=5.0, **att)
    s9 = GP.attend_cost_us(16, rows=9, hbm_gbs=6500.0, tensor_tflops=5.0, **att)
    assert s9 / s2 == pytest.approx(9 / 2, rel=1e-12)
    assert GP.round_cost_us(16, gamma=8, **args) > GP.round_cost_us(16, gamma=1, **args)
    # the toggle follows: at 0.7 acceptance drafting pays while memory-bound, not when compute-bound
    for tf, want_on in ((1500.0, True), (0.5, False)):
        a = dict(args, tensor_tflops=tf)
        cost = [GP.round_cost_us(16, gamma=g, **a) for g in range(9)]
        p = GP.Policy(8, 0.9, 0.7, 1e3, cost)
        assert (p.choose()[0] > 0) == want_on, (tf, p.choose())
