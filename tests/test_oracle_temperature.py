"""Pins of the oracle's sampling temperature (p = softmax(target / T),
q = softmax(draft / T)) against hand-derived values and a chi-square run at
T != 1, with planted slips that the pins must catch.

Every expected value here comes from weights w chosen so that the logits
T ln w make softmax(logits / T) = w / sum(w); nothing is recomputed with the
oracle's own softmax. None of these calls the CUDA path.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy import stats

import oracle as O
import oracle.s3r_oracle as OM

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "temperature_hand.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _mismatches():
    """Cases of the temperature fixture that the oracle (as currently bound
    in the module) gets wrong."""
    g = _golden()
    bad = []
    for c in g["softmax_cases"]:
        T = c["temperature"]
        logits = np.log(np.array([c["logits_weights"]], float))
        p = O.softmax_t(logits, T)[0]
        if not np.allclose(p, np.array(c["p_num"], float) / c["p_den"], rtol=0, atol=1e-12):
            bad.append(("softmax", T))
        for d in c["draws"]:
            k, _ = O.sample_rows(logits, np.array([d["u"]]), T)
            if int(k[0]) != d["k"]:
                bad.append(("draw", T, d["u"]))
    T = g["spec_temperature"]
    tl = T * np.log(np.array([g["target_weights"]], float))
    dl = T * np.log(np.array([g["draft_weights"]], float))
    for c in g["spec_cases"]:
        out, n_acc, _, _ = O.spec_sample(tl, dl, np.array([[c["draft_token"]]]), np.array([[c["u_accept"]]]),
                                         np.array([c["u_sample"]]), T)
        if out[0].tolist() != c["out"] or int(n_acc[0]) != c["n_acc"]:
            bad.append(("spec", c["draft_token"], c["u_accept"], c["u_sample"]))
    return bad


def test_temperature_hand_cases():
    assert _mismatches() == []


def _softmax_with(x):
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def _plant_times_t(logits, temperature):
    return _softmax_with(np.asarray(logits, dtype=np.float64) * temperature)


def _plant_ignore_t(logits, temperature):
    return _softmax_with(logits)


def _alternating(first_gets_t):
    """spec_sample calls softmax_t twice per call, target rows first: apply T
    to only one of the two."""
    state = {"n": 0}

    def f(logits, temperature):
        state["n"] += 1
        use_t = (state["n"] % 2 == 1) == first_gets_t
        return _softmax_with(np.asarray(logits, dtype=np.float64) / (temperature if use_t else 1.0))
    return f


@pytest.mark.parametrize("plant", ["times_t", "ignore_t", "target_only", "draft_only"])
def test_temperature_pins_catch_planted_slips(monkeypatch, plant):
    """A softmax that multiplies by T, ignores it, or applies it to only the
    target or only the draft rows fails the hand cases."""
    fn = {"times_t": _plant_times_t, "ignore_t": _plant_ignore_t,
          "target_only": _alternating(True), "draft_only": _alternating(False)}[plant]
    monkeypatch.setattr(OM, "softmax_t", fn)
    monkeypatch.setattr(O, "softmax_t", fn)
    assert len(_mismatches()) > 0


def _weights_dists(V, gamma, seed):
    """Target and draft weights (the distributions at temperature T are
    w / sum(w) when the logits are T ln w)."""
    rng = np.random.default_rng(seed)
    wt = np.exp(1.2 * rng.standard_normal((gamma + 1, V)))
    wd = wt[:gamma] * np.exp(0.8 * rng.standard_normal((gamma, V)))
    return wt, wd


@pytest.mark.parametrize("T", [0.7])
def test_committed_tokens_follow_p_at_temperature(T):
    """Chi-square of committed tokens against p_j = w_j / sum(w_j) at T = 0.7
    (logits T ln w), 300K rounds, V = 16, gamma = 3; and the same statistic
    rejects the distribution a T-slip would give (w^T normalised)."""
    V, gamma, n = 16, 3, 300_000
    wt, wd = _weights_dists(V, gamma, 2024)
    t = T * np.log(wt)
    d = T * np.log(wd)
    rng = np.random.default_rng(99)
    x, _ = O.sample_rows(np.broadcast_to(d, (n, gamma, V)).reshape(-1, V), rng.random(n * gamma), T)
    out, n_acc, _, _ = O.spec_sample(np.broadcast_to(t, (n, gamma + 1, V)), np.broadcast_to(d, (n, gamma, V)),
                                     x.reshape(n, gamma), rng.random((n, gamma)), rng.random((n, gamma + 1)), T)
    crit = stats.chi2.ppf(0.999, V - 1)
    p = wt / wt.sum(axis=1, keepdims=True)
    for j in range(gamma + 1):
        reached = n_acc >= j
        counts = np.bincount(out[reached, j], minlength=V)
        exp = p[j] * reached.sum()
        chi = ((counts - exp) ** 2 / exp).sum()
        assert chi < crit, (j, chi)
    # power: the distribution softmax(logits) (temperature ignored) is rejected
    wrong = wt ** T / (wt ** T).sum(axis=1, keepdims=True)
    counts = np.bincount(out[:, 0], minlength=V)
    exp = wrong[0] * n
    assert ((counts - exp) ** 2 / exp).sum() > crit
    # and the draft tokens follow q = wd / sum(wd)
    q = wd / wd.sum(axis=1, keepdims=True)
    xs = x.reshape(n, gamma)
    for i in range(gamma):
        counts = np.bincount(xs[:, i], minlength=V)
        exp = q[i] * n
        assert ((counts - exp) ** 2 / exp).sum() < crit


def test_acceptance_rate_closed_form_at_temperature():
    """Acceptance at position 0 equals sum_x min(p, q) with p, q the
    temperature-T distributions (w / sum w), within 4 sigma."""
    T, V, n = 0.7, 16, 200_000
    wt, wd = _weights_dists(V, 1, 7)
    p = wt[0] / wt[0].sum()
    q = wd[0] / wd[0].sum()
    rng = np.random.default_rng(5)
    d = T * np.log(wd)
    x, _ = O.sample_rows(np.broadcast_to(d, (n, V)), rng.random(n), T)
    _, n_acc, _, _ = O.spec_sample(np.broadcast_to(T * np.log(wt), (n, 2, V)), np.broadcast_to(d, (n, 1, V)),
                                   x.reshape(n, 1), rng.random((n, 1)), rng.random((n, 2)), T)
    alpha = np.minimum(p, q).sum()
    assert abs((n_acc >= 1).mean() - alpha) < 4 * math.sqrt(alpha * (1 - alpha) / n)
