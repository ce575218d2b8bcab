"""The parity tests' comparison rules (oracle/reference_run.py) on
hand-made "GPU" outputs: exact equality away from near-ties, and at a
near-tie a validity check that still rejects a wrong choice. CPU only."""
import numpy as np
import pytest

import oracle.reference_run as RR


def test_valid_top_set_within_band():
    s = np.array([3.0, 1.0, 3.0 + 1e-14, 2.0])
    assert RR.valid_top_set([0, 2], s, 2)
    assert not RR.valid_top_set([0, 3], s, 2)         # drops a score above a kept one
    assert not RR.valid_top_set([2, 0], s, 2)         # not ascending
    assert not RR.valid_top_set([0], s, 2)            # wrong size
    assert not RR.valid_top_set([0, 4], s, 2)         # out of range
    assert RR.valid_top_set([0, 1], np.array([5.0, 4.0]), 4)   # n <= budget: all pages


def test_compare_selection_near_tie_checks_the_choice():
    s = np.array([[3.0, 1.0, 3.0 + 1e-14, 2.0]])
    gaps = np.array([1e-14 / 3.0])
    ref = [np.array([0, 2])]
    tally = RR.Tally()
    # three pages tie for two places: another tied pair than the oracle's is
    # a valid choice (counted as a near-tie, outputs not comparable) ...
    s2 = np.array([[3.0, 1.0, 3.0, 2.0, 3.0]])
    ok = RR.compare_selection("t", np.array([[0, 4]]), [np.array([0, 2])], np.array([0.0]), tally, scores=s2)
    assert ok == [False] and tally.near_ties == 1
    # ... a set that drops a clearly larger score is rejected even at a near-tie
    with pytest.raises(AssertionError):
        RR.compare_selection("t", np.array([[0, 3]]), ref, gaps, RR.Tally(), scores=s)
    # away from a near-tie the sets must be equal
    with pytest.raises(AssertionError):
        RR.compare_selection("t", np.array([[0, 3]]), ref, np.array([0.5]), RR.Tally(), scores=s)
    # a near-tie without scores cannot be checked
    with pytest.raises(AssertionError):
        RR.compare_selection("t", np.array([[0, 2]]), ref, gaps, RR.Tally())


def test_valid_draw():
    w = np.array([1.0, 0.0, 3.0])               # CDF 0.25, 0.25, 1
    assert RR.valid_draw(w, 0.1, 0)
    assert RR.valid_draw(w, 0.25, 2)
    assert RR.valid_draw(w, 0.25, 0)            # on the boundary: within the band
    assert not RR.valid_draw(w, 0.25, 1)        # zero weight never wins
    assert not RR.valid_draw(w, 0.5, 0)
    assert not RR.valid_draw(w, 0.1, 3)


def _ref(seed=0, V=12, gamma=3):
    rng = np.random.default_rng(seed)
    t = 2 * rng.standard_normal((gamma + 1, V))
    d = t[:gamma] + rng.standard_normal((gamma, V))
    return RR.sampling_ref_from_logits(t, d, rng.random(gamma), rng.random(gamma), rng.random(gamma + 1), 0.9)


def test_validity_walk_accepts_the_oracles_own_outputs():
    for seed in range(20):
        r = _ref(seed)
        RR.validity_walk("t", r["x"], r["out_tokens"], r["n_acc"], r)
        tally = RR.Tally()
        RR.compare_sampling("t", r["x"], r["out_tokens"], r["n_acc"], r, tally)


def test_validity_walk_rejects_wrong_choices():
    r = _ref(3)
    n, x, out = r["n_acc"], r["x"].copy(), r["out_tokens"].copy()
    # a draft token that is not the draw at u_draft
    bad_x = x.copy()
    bad_x[0] = (bad_x[0] + 1) % len(r["q"][0])
    with pytest.raises(AssertionError):
        RR.validity_walk("t", bad_x, out, n, r)
    # a drawn token of zero residual weight (or simply the wrong one)
    bad_out = out.copy()
    w = r["p"][n] if n == len(x) else RR.O.residual_weights(r["p"][n], r["q"][n])
    zero = np.nonzero(w == 0)[0]
    bad_out[n] = int(zero[0]) if len(zero) else (int(out[n]) + 1) % len(w)
    with pytest.raises(AssertionError):
        RR.validity_walk("t", x, bad_out, n, r)
    # an extra accept the uniform does not allow
    if n < len(x):
        acc = out.copy()
        acc[:n + 1] = x[:n + 1]
        with pytest.raises(AssertionError):
            RR.validity_walk("t", x, acc, n + 1, r)
    # trailing tokens after the drawn one
    trail = out.copy()
    if n + 1 < len(trail):
        trail[n + 1] = 0
        with pytest.raises(AssertionError):
            RR.validity_walk("t", x, trail, n, r)


def test_compare_sampling_runs_the_walk_at_a_near_tie():
    r = _ref(4)
    # declare the first accept test a near-tie: the GPU's outputs are then
    # checked for validity, so a wrong drawn token still fails
    r2 = dict(r, accept_margin=np.where(np.isnan(r["accept_margin"]), np.nan, 0.0))
    tally = RR.Tally()
    RR.compare_sampling("t", r["x"], r["out_tokens"], r["n_acc"], r2, tally)
    assert tally.near_ties == 1
    bad = r["out_tokens"].copy()
    n = r["n_acc"]
    bad[n] = (bad[n] + 1) % r["p"].shape[1]
    w = r["p"][n] if n == len(r["x"]) else RR.O.residual_weights(r["p"][n], r["q"][n])
    if not RR.valid_draw(w, r["u_sample"][n], bad[n]):
        with pytest.raises(AssertionError):
            RR.compare_sampling("t", r["x"], bad, n, r2, RR.Tally())
