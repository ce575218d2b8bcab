"""Float64 oracle of the draft-length policy: acceptance-aware choice of
gamma with a regime toggle (gamma = 0: plain decoding).

TEST INFRASTRUCTURE ONLY (tests; nothing in the product path imports it).
It shares no code with libs3r's policy (src: csrc/s3r_policy.cu).

Source: the researchpod.app page on EfficientRollout (another self-drafting
method for RL rollouts) describes two controls: a regime-aware toggle that
drafts only when drafting speeds the step up (it depends on whether the step
is limited by compute or by memory bandwidth), and a draft length adapted to
how often drafts are accepted. The expected committed tokens per round come
from the speculative-decoding papers on the mlsanity.com reference list.

Readings (the pages give no formulas):
* acceptance estimate: accepted / tested draft positions over the rounds, each
  round's counts weighted by decay^age (an exponentially weighted ratio) and
  started from a prior (prior_accept, prior_weight);
* a round with gamma drafts and per-position acceptance alpha commits
  E(gamma) = sum_{i=0}^{gamma} alpha^i tokens per sequence;
* rate(gamma) = E(gamma) / cost(gamma), rate(0) = 1 / cost(0) (one token per
  plain decode step); the chosen gamma maximises the rate over 0..gamma_max
  (the smaller gamma on exact ties), so gamma = 0 switches drafting off;
* cost model (when the caller has no measured costs): every call is bounded
  by HBM bytes / bandwidth, verification by max(bytes / bandwidth,
  flops / tensor peak), so it turns compute-bound as batch x rows grows.
"""
from __future__ import annotations

import numpy as np


def expected_tokens(alpha, gamma):
    """E(gamma) = sum_{i=0}^{gamma} alpha^i: committed tokens per sequence and
    round with per-position acceptance alpha (0 <= alpha <= 1)."""
    return float(sum(float(alpha) ** i for i in range(int(gamma) + 1)))


def tests_made(n_acc, gamma):
    """Accept tests a round makes for one sequence: every accepted draft and
    the first rejected one (none after the last draft)."""
    return min(int(n_acc) + 1, int(gamma))


class Policy:
    def __init__(self, gamma_max, decay, prior_accept, prior_weight, cost):
        self.gamma_max = int(gamma_max)
        self.decay = float(decay)
        self.accepted = float(prior_accept) * float(prior_weight)
        self.tested = float(prior_weight)
        self.cost = [float(c) for c in cost]                   # cost[g], g = 0..gamma_max

    def update(self, num_accepted, gamma):
        """One round's acceptance counts (gamma drafts per sequence)."""
        a = float(sum(int(x) for x in num_accepted))
        t = float(sum(tests_made(x, gamma) for x in num_accepted))
        self.accepted = self.decay * self.accepted + a
        self.tested = self.decay * self.tested + t

    def alpha(self):
        return self.accepted / self.tested if self.tested > 0 else 0.0

    def rate(self, gamma):
        if gamma == 0:
            return 1.0 / self.cost[0]
        return expected_tokens(self.alpha(), gamma) / self.cost[gamma]

    def choose(self):
        """(gamma, rate): the largest rate over 0..gamma_max, the smaller gamma on ties."""
        best, best_rate = 0, self.rate(0)
        for g in range(1, self.gamma_max + 1):
            r = self.rate(g)
            if r > best_rate:
                best, best_rate = g, r
        return best, best_rate


def attend_cost_us(num_seqs, q_heads, kv_heads, head_dim, kv_bytes, mean_context, rows, hbm_gbs, tensor_tflops):
    """Roofline time of dense attention of `rows` query rows per sequence over
    the whole cache: max(bytes / bandwidth, flops / tensor peak), in us."""
    kv = num_seqs * 2.0 * kv_heads * head_dim * kv_bytes * float(mean_context)
    flops = 4.0 * num_seqs * q_heads * rows * float(mean_context) * head_dim
    return max(kv / (float(hbm_gbs) * 1e9), flops / (float(tensor_tflops) * 1e12)) * 1e6


def round_cost_us(num_seqs, q_heads, kv_heads, head_dim, page_size, kv_bytes, mean_context, budget_pages, vocab,
                  logit_bytes, gamma, hbm_gbs, tensor_tflops):
    """Roofline time of one round in microseconds (the reading above).

    gamma >= 1: gamma sparse draft calls (every page's summary, the kept
    pages' keys and values), one verification of R = gamma + 1 rows over the
    whole cache, the drafter's draws (gamma rows) and speculative sampling
    (2 gamma + 1 rows and a re-read of two). gamma = 0: one dense decode row
    and one draw.
    """
    bw = float(hbm_gbs) * 1e9
    S, H, D, P = num_seqs, kv_heads, head_dim, page_size
    L = float(mean_context)
    pages = np.ceil(L / P)

    def attend(rows):                                           # seconds
        return attend_cost_us(S, q_heads, H, D, kv_bytes, L, rows, hbm_gbs, tensor_tflops) * 1e-6

    if gamma == 0:
        t = attend(1) + S * vocab * logit_bytes / bw
        return t * 1e6
    draft = S * H * (pages * 2.0 * D * kv_bytes + min(budget_pages, pages) * P * 2.0 * D * kv_bytes) / bw
    sample = S * ((2 * gamma + 1) + 2) * vocab * logit_bytes / bw
    draws = S * gamma * vocab * logit_bytes / bw
    return (gamma * draft + attend(gamma + 1) + sample + draws) * 1e6
