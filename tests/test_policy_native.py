"""The library's draft-length policy and roofline cost model (host code in
libs3r) against the float64 oracle (oracle/gamma_policy.py) on random
rounds, and its argument checks. Runs without a GPU."""
import math

import numpy as np
import pytest

from self_sparse_speculative_b200 import s3r
from oracle import gamma_policy as GP


def test_policy_follows_the_oracle_over_random_rounds():
    rng = np.random.default_rng(0)
    for trial in range(60):
        gmax = int(rng.integers(1, 17))
        decay = float(rng.uniform(0, 1))
        prior = float(rng.uniform(0, 1))
        weight = float(rng.uniform(0, 50))
        cost = list(rng.uniform(10.0, 500.0, gmax + 1))
        lib = s3r.GammaPolicyHandle(gmax, decay, prior, weight, cost)
        ora = GP.Policy(gmax, decay, prior, weight, cost)
        for rnd in range(int(rng.integers(1, 30))):
            g_used = int(rng.integers(1, gmax + 1))
            n_acc = rng.integers(0, g_used + 1, size=int(rng.integers(1, 40)))
            lib.update(n_acc, g_used)
            ora.update(n_acc, g_used)
            g, a, r = lib.choose()
            go, ro = ora.choose()
            assert a == pytest.approx(ora.alpha(), rel=1e-14, abs=1e-15)
            rates = sorted((ora.rate(k) for k in range(gmax + 1)), reverse=True)
            if rates[0] - rates[1] > 1e-12 * rates[0]:          # not a near-tie between two lengths
                assert g == go, (trial, rnd, g, go)
            assert r == pytest.approx(ro, rel=1e-12)


def test_cost_model_follows_the_oracle():
    rng = np.random.default_rng(1)
    for _ in range(200):
        S, G, H = int(rng.integers(1, 300)), int(rng.integers(1, 9)), int(rng.integers(1, 9))
        D, P = int(rng.choice([64, 128])), int(rng.choice([16, 64]))
        kvb, lb = int(rng.choice([2, 4])), int(rng.choice([2, 4]))
        L, B, V = float(rng.uniform(64, 70000)), int(rng.integers(1, 129)), int(rng.integers(1000, 200000))
        g = int(rng.integers(0, 17))
        bw, tf = float(rng.uniform(1000, 8000)), float(rng.uniform(1, 2500))
        got = s3r.s3r_round_cost_us(S, G * H, H, D, P, kvb, L, B, V, lb, g, bw, tf)
        want = GP.round_cost_us(S, G * H, H, D, P, kvb, L, B, V, lb, g, bw, tf)
        assert got == pytest.approx(want, rel=1e-12)
        rows = int(rng.integers(1, 20))
        assert s3r.s3r_attend_cost_us(S, G * H, H, D, kvb, L, rows, bw, tf) == pytest.approx(
            GP.attend_cost_us(S, G * H, H, D, kvb, L, rows, bw, tf), rel=1e-12)


def test_policy_argument_checks():
    with pytest.raises(s3r.S3RError):
        s3r.GammaPolicyHandle(0, 0.9, 0.5, 1.0, [1.0])                       # gamma_max < 1
    with pytest.raises(s3r.S3RError):
        s3r.GammaPolicyHandle(4, 1.5, 0.5, 1.0, [1.0] * 5)                   # decay outside [0, 1]
    with pytest.raises(s3r.S3RError):
        s3r.GammaPolicyHandle(4, 0.9, 0.5, 1.0, [1.0, 2.0, 0.0, 1.0, 1.0])   # a cost that is not positive
    p = s3r.GammaPolicyHandle(4, 0.9, 0.5, 1.0, [1.0] * 5)
    with pytest.raises(s3r.S3RError):
        p.update([5], 4)                                                    # more accepted than drafted
    assert math.isnan(s3r.s3r_round_cost_us(1, 8, 2, 128, 64, 2, 100.0, 4, 1000, 2, 17, 6500.0, 1500.0))


def test_workload_regimes_with_the_native_policy():
    """At the 16 x 16K layer's shapes and 0.6 acceptance drafting pays; with
    4096 sequences of the 256-sequence layer's shapes and a tensor peak of a
    few TFLOP/s the verification is compute-bound and drafting switches off."""
    def choose(S, tf, alpha):
        cost = [s3r.s3r_round_cost_us(S, 32, 8, 128, 64, 2, 16384.0, 32, 151936, 2, g, 6500.0, tf)
                for g in range(9)]
        p = s3r.GammaPolicyHandle(8, 0.9, alpha, 1e4, cost)
        return p.choose()[0]
    assert choose(16, 1500.0, 0.6) > 0
    assert choose(4096, 2.0, 0.6) == 0


def test_tree_node_budget_follows_the_oracle():
    """N_t = clip(floor(C_hw / B_t), N_min, N_max) in libs3r against the
    oracle's node_budget over random capacities and concurrencies."""
    import oracle as O
    rng = np.random.default_rng(7)
    for _ in range(2000):
        n_min = int(rng.integers(1, 8))
        n_max = int(rng.integers(n_min, 65))
        active = int(rng.integers(1, 513))
        cap = int(rng.integers(0, 1 << 40)) if rng.random() < 0.1 else int(rng.integers(0, 20000))
        assert s3r.s3r_tree_node_budget(cap, active, n_min, n_max) == O.node_budget(cap, active, n_min, n_max)
    # as responses finish (B_t falls) the budget grows up to N_max
    seq = [s3r.s3r_tree_node_budget(600, b, 2, 32) for b in (256, 64, 32, 16, 8, 1)]
    assert seq == sorted(seq) and seq[0] == 2 and seq[-1] == 32
    for bad in ((600, 0, 2, 16), (600, 4, 0, 16), (600, 4, 8, 4), (-1, 4, 2, 16)):
        assert s3r.s3r_tree_node_budget(*bad) == -1
