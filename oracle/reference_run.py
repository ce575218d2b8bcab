"""Oracle run of a whole decode step on (a sample of) a workload, and the
comparison rules of the parity tests.

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline). The
oracle computes only from the seeded inputs of the workload generator; no
value here comes from the CUDA path. The comparison helpers take the GPU's
outputs as plain arrays.

Comparison rules:
* page summaries, page selection and token indices are compared exactly;
* attention outputs within |gpu - oracle| <= atol + rtol * |oracle|,
  2e-2 / 1e-2 for bf16 inputs and 1e-5 / 1e-5 for fp32;
* an accept test with |u - p/q| < 1e-6, a draw with |u - C(k)/C(V-1)|
  < 1e-10 at the drawn token's boundary (both sides decide draws in float64;
  only the order of the float64 sums differs), or a page boundary whose
  scores differ by at most 1e-12 of the largest score is a near-tie: it is
  counted, and it and every later decision of that sequence are left out of
  the exact comparison. The GPU's choices there are still checked for
  validity: a selection must be a top-B set up to the score band (every kept
  score at least every dropped one minus the band); after a near-tie in the
  sampling, the GPU's own draft tokens, accept decisions and drawn token are
  walked in order, and each must be what the oracle decides for those same
  tokens, or within the near-tie band of it (an accept needs u < p/q + band,
  a reject u >= p/q - band, a draw a token of positive weight whose CDF
  interval holds u up to the band).
"""
from __future__ import annotations

import numpy as np

from self_sparse_speculative_b200.workloads import to_float64

from . import s3r_oracle as O

NEAR_TIE_DECISION = 1e-6     # accept tests |u - p/q|
NEAR_TIE_DRAW = 1e-10        # inverse-CDF draws |u - C(k)/C(V-1)|
NEAR_TIE_SCORE = 1e-12
TOL = {"bf16": (2e-2, 1e-2), "f32": (1e-5, 1e-5)}


def f32(x: float) -> float:
    """The float32 value the GPU receives for a Python float argument."""
    return float(np.float32(x))


def sequence_cache(wl, b):
    """float64 K, V of sequence b's pages, with a local block table."""
    dt = wl.spec.kv_dtype
    n = int(wl.pages_per_seq[b])
    phys = wl.block_table[b, :n]
    K = to_float64(wl.kv_pages("K", phys), dt)
    V = to_float64(wl.kv_pages("V", phys), dt)
    bt = np.arange(n, dtype=np.int64)[None, :]
    return K, V, bt, phys


def sequence_inputs(wl, b, draft_steps=None, attention=True, sampling=True):
    """Every float64 input of sequence b's round, generated from the seeded
    workload (no arithmetic of the method): the cache of its pages, its draft
    and verify queries, its logits and uniforms."""
    ws = wl.spec
    inp = {"b": b, "spec": ws, "scale": f32(wl.scale), "T": f32(ws.temperature),
           "lens": wl.context_lens[b:b + 1].astype(np.int64)}
    if attention:
        inp["K"], inp["V"], inp["bt"], inp["phys"] = sequence_cache(wl, b)
        steps = range(ws.gamma) if draft_steps is None else draft_steps
        inp["q_draft"] = {i: to_float64(wl.q_draft[i, b], ws.kv_dtype)[None] for i in steps}   # [1, Hq, D]
        inp["q_verify"] = to_float64(wl.q_verify[b], ws.kv_dtype)[None]                         # [1, R, Hq, D]
    if sampling:
        t, d = wl.logits_for_seq(b)
        inp["tl"] = to_float64(t, ws.logit_dtype)
        inp["dl"] = to_float64(d, ws.logit_dtype)
        inp["u_draft"] = wl.u_draft[b].astype(np.float64)
        inp["u_accept"] = wl.u_accept[b].astype(np.float64)
        inp["u_sample"] = wl.u_sample[b].astype(np.float64)
    return inp


def oracle_attention(inp):
    """Oracle summaries, page selection, sparse draft and verify attention of
    one sequence's inputs (sequence_inputs)."""
    ws = inp["spec"]
    P, B, G = ws.page_size, ws.budget_pages, ws.group
    K, V, bt, lens, scale = inp["K"], inp["V"], inp["bt"], inp["lens"], inp["scale"]
    kmin, kmax = O.page_summaries(K, bt, lens, P)
    draft = {}
    for i, q in inp["q_draft"].items():
        sel, gaps, scores = O.sparse_draft_select(q, kmin, kmax, bt, lens, P, B, G, return_scores=True)
        out, lse = O.sparse_draft_attn(q, K, V, bt, lens, sel, scale)
        draft[i] = {"selected": sel[0], "gaps": gaps[0], "scores": scores[0], "out": out[0], "lse": lse[0],
                    "q": q}
    vout, vlse = O.verify_attn(inp["q_verify"], K, V, bt, lens, scale)
    return {"phys": inp["phys"], "kmin": kmin, "kmax": kmax, "draft": draft,
            "verify_out": vout[0], "verify_lse": vlse[0], "K": K, "V": V, "bt": bt, "lens": lens}


def oracle_attention_seq(wl, b, draft_steps=None):
    """Oracle summaries, page selection, sparse draft and verify attention of
    sequence b. draft_steps: which draft queries to run (default: all)."""
    return oracle_attention(sequence_inputs(wl, b, draft_steps=draft_steps, sampling=False))


def oracle_kv_round_seq(wl, b):
    """Oracle of sequence b's round with the cache upkept: from committed
    length C = L - R, each draft step writes its rows at the end of the cache
    and attends sparsely from that position; verification writes its R rows
    over the round's positions and attends densely; sampling commits; the
    cache is rolled back to the committed prefix. Returns the selections,
    outputs, tokens and the cache state after the round."""
    ws = wl.spec
    P, B, G, R, g = ws.page_size, ws.budget_pages, ws.group, ws.rows, ws.gamma
    dt = ws.kv_dtype
    scale = f32(wl.scale)
    K, V, bt, phys = sequence_cache(wl, b)
    L = int(wl.context_lens[b])
    lens = np.array([L - R], dtype=np.int64)
    kmin, kmax = O.page_summaries(K, bt, lens, P)
    kd, vd, kv_, vv = (to_float64(x, dt) for x in wl.round_kv(b))
    draft = {}
    for i in range(g):
        K, V, lens, kmin, kmax = O.kv_append(K, V, bt, lens, kd[i][None, None], vd[i][None, None], 0, P, kmin, kmax)
        q = to_float64(wl.q_draft[i, b], dt)[None]
        sel, gaps, scores = O.sparse_draft_select(q, kmin, kmax, bt, lens, P, B, G, return_scores=True)
        out, lse = O.sparse_draft_attn(q, K, V, bt, lens, sel, scale)
        draft[i] = {"selected": sel[0], "gaps": gaps[0], "scores": scores[0], "out": out[0], "lse": lse[0]}
    K, V, lens, kmin, kmax = O.kv_append(K, V, bt, lens, kv_[None], vv[None], g, P, kmin, kmax)
    qv = to_float64(wl.q_verify[b], dt)[None]
    vout, vlse = O.verify_attn(qv, K, V, bt, lens, scale)
    smp = oracle_sampling_seq(wl, b)
    lens_c, kmin_c, kmax_c = O.kv_rollback(K, bt, lens, np.array([smp["n_acc"]]), R, P, kmin, kmax)
    return {"phys": phys, "draft": draft, "verify_out": vout[0], "verify_lse": vlse[0], "sampling": smp,
            "K": K, "V": V, "len_after": int(lens_c[0]), "kmin": kmin_c, "kmax": kmax_c, "start": L - R}


def oracle_sampling(inp):
    """Oracle draft-token draws and speculative sampling of one sequence's
    inputs (sequence_inputs)."""
    return sampling_ref_from_logits(inp["tl"], inp["dl"], inp["u_draft"], inp["u_accept"], inp["u_sample"],
                                    inp["T"])


def oracle_sampling_seq(wl, b):
    """Oracle draft-token draws and speculative sampling of sequence b."""
    return oracle_sampling(sequence_inputs(wl, b, attention=False))


def sampling_ref_from_logits(target_logits, draft_logits, u_draft, u_accept, u_sample, temperature):
    """The same record as oracle_sampling_seq for one sequence's float64
    logits and uniforms given directly (the draft tokens drawn from q with
    u_draft)."""
    T = f32(temperature)
    tl = np.asarray(target_logits, dtype=np.float64)
    dl = np.asarray(draft_logits, dtype=np.float64)
    ud = np.asarray(u_draft, dtype=np.float64)
    x, xm = O.sample_rows(dl, ud, T)
    out, n_acc, am, sm = O.spec_sample(tl[None], dl[None], x[None], np.asarray(u_accept)[None],
                                       np.asarray(u_sample)[None], T)
    return {"x": x, "x_margin": xm, "out_tokens": out[0], "n_acc": int(n_acc[0]),
            "accept_margin": am[0], "sample_margin": float(sm[0]),
            "p": O.softmax_t(tl, T), "q": O.softmax_t(dl, T), "u_draft": ud,
            "u_accept": np.asarray(u_accept, dtype=np.float64), "u_sample": np.asarray(u_sample, dtype=np.float64)}


# ------------------------------------------------------------------ comparisons
class Tally:
    """Counts of exact decisions compared and near-ties left out."""

    def __init__(self):
        self.decisions = 0
        self.near_ties = 0
        self.notes = []

    def near_tie_fraction(self):
        return self.near_ties / max(1, self.decisions)


def assert_close(name, gpu, ref, dtype):
    atol, rtol = TOL[dtype]
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    both_inf = np.isinf(gpu) & np.isinf(ref) & (np.sign(gpu) == np.sign(ref))
    err = np.abs(gpu - ref)
    bad = ~(both_inf | (err <= atol + rtol * np.abs(ref)))
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(f"{name}: {int(bad.sum())} of {bad.size} outside tolerance "
                             f"(atol {atol}, rtol {rtol}); first at {tuple(idx)}: gpu {gpu[tuple(idx)]} "
                             f"oracle {ref[tuple(idx)]}; max err {np.nanmax(np.where(both_inf, 0, err)):.3e}")


def valid_top_set(gpu_set, scores, budget):
    """Whether gpu_set (ascending logical pages) is a top-`budget` set of
    `scores` up to the near-tie band: the right size, distinct in-range pages
    in ascending order, and every kept score >= every dropped score minus
    NEAR_TIE_SCORE times the largest |score|."""
    s = np.asarray(scores, dtype=np.float64)
    n = len(s)
    g = np.asarray(gpu_set, dtype=np.int64)
    if len(g) != min(n, budget) or np.any(g < 0) or np.any(g >= n) or np.any(np.diff(g) <= 0):
        return False
    if len(g) == n:
        return True
    dropped = np.setdiff1d(np.arange(n), g)
    band = NEAR_TIE_SCORE * float(np.abs(s).max())
    return float(s[g].min()) >= float(s[dropped].max()) - band


def compare_selection(name, gpu_sel, ref_sel, gaps, tally: Tally, scores=None):
    """gpu_sel [Hkv, B] (-1 padded), ref_sel list of arrays, gaps [Hkv],
    scores [Hkv, n_b] (the oracle's page scores). Exact set equality, except
    at a near-tie boundary, where the GPU's set must be a valid top-B set up
    to the band (scores are required there). Returns per head whether the
    sets are equal (attention outputs are comparable)."""
    ok_heads = []
    for h, rs in enumerate(ref_sel):
        tally.decisions += 1
        g = np.asarray(gpu_sel[h])
        g = g[g >= 0]
        if gaps[h] <= NEAR_TIE_SCORE:
            tally.near_ties += 1
            tally.notes.append(f"{name} head {h}: near-tie page boundary")
            if scores is None:
                raise AssertionError(f"{name} head {h}: near-tie boundary but no scores to check the choice")
            if not valid_top_set(g, scores[h], len(rs)):
                raise AssertionError(f"{name} head {h}: gpu selection {g.tolist()} is not a top-B set "
                                     f"within the near-tie band")
            eq = np.array_equal(g, np.asarray(rs))
            ok_heads.append(eq)
            continue
        if not np.array_equal(g, np.asarray(rs)):
            raise AssertionError(f"{name} head {h}: selected pages differ: gpu {g.tolist()} oracle {list(rs)}")
        ok_heads.append(True)
    return ok_heads


def valid_draw(weights, u, k, band=NEAR_TIE_DRAW):
    """Whether token k is a valid inverse-CDF draw from the unnormalised
    weights at uniform u, up to the band: positive weight, and
    C(k-1)/C(V-1) - band <= u < C(k)/C(V-1) + band."""
    w = np.asarray(weights, dtype=np.float64)
    k = int(k)
    if k < 0 or k >= len(w) or not w[k] > 0:
        return False
    C = np.cumsum(w)
    lo = (C[k - 1] if k > 0 else 0.0) / C[-1]
    hi = C[k] / C[-1]
    return lo - band <= float(u) < hi + band


def validity_walk(name, gpu_x, gpu_out, gpu_nacc, ref):
    """Check the GPU's sampling of one sequence decision by decision against
    the oracle's distributions, following the GPU's own choices (used after a
    near-tie, where the two may legitimately part ways)."""
    p, q = ref["p"], ref["q"]
    gamma = q.shape[0]
    x = np.asarray(gpu_x, dtype=np.int64)
    out = np.asarray(gpu_out, dtype=np.int64)
    n = int(gpu_nacc)
    for i in range(gamma):
        if not valid_draw(q[i], ref["u_draft"][i], x[i]):
            raise AssertionError(f"{name}: draft token {i} = {int(x[i])} is not a valid draw from q_{i}")
    if not 0 <= n <= gamma:
        raise AssertionError(f"{name}: n_acc {n} outside [0, {gamma}]")
    for i in range(min(n + 1, gamma)):
        qx = q[i, x[i]]
        ratio = p[i, x[i]] / qx if qx > 0 else 0.0
        u = ref["u_accept"][i]
        if i < n and not u < ratio + NEAR_TIE_DECISION:
            raise AssertionError(f"{name}: accept {i} taken with u {u} >= p/q {ratio}")
        if i == n and not u >= ratio - NEAR_TIE_DECISION:
            raise AssertionError(f"{name}: reject {i} taken with u {u} < p/q {ratio}")
    if not np.array_equal(out[:n], x[:n]):
        raise AssertionError(f"{name}: committed drafts {out[:n].tolist()} differ from the drafts {x[:n].tolist()}")
    w = p[gamma] if n == gamma else O.residual_weights(p[n], q[n])
    if not valid_draw(w, ref["u_sample"][n], out[n]):
        raise AssertionError(f"{name}: drawn token {int(out[n])} at position {n} is not a valid draw")
    if np.any(out[n + 1:] != -1):
        raise AssertionError(f"{name}: tokens after the drawn one are not -1: {out.tolist()}")


def compare_sampling(name, gpu_x, gpu_out, gpu_nacc, ref, tally: Tally):
    """Exact comparison of one sequence's draft draws, accept decisions and
    drawn token. At the first near-tie the exact comparison stops (the
    decision and everything after it may differ) and the GPU's choices are
    checked for validity instead (validity_walk)."""
    gamma = len(ref["x"])
    for i in range(gamma):
        tally.decisions += 1
        if ref["x_margin"][i] < NEAR_TIE_DRAW:
            tally.near_ties += 1
            tally.notes.append(f"{name}: near-tie draft draw {i}")
            if not np.array_equal(np.asarray(gpu_x[:i]), ref["x"][:i]):
                raise AssertionError(f"{name}: draft tokens before the near-tie differ")
            validity_walk(name, gpu_x, gpu_out, gpu_nacc, ref)
            return
        if int(gpu_x[i]) != int(ref["x"][i]):
            raise AssertionError(f"{name}: draft token {i} gpu {int(gpu_x[i])} oracle {int(ref['x'][i])}")
    n_ref = ref["n_acc"]
    for i in range(min(gamma, n_ref + 1)):
        tally.decisions += 1
        if ref["accept_margin"][i] < NEAR_TIE_DECISION:
            tally.near_ties += 1
            tally.notes.append(f"{name}: near-tie accept test {i}")
            if int(gpu_nacc) < i:
                raise AssertionError(f"{name}: n_acc {int(gpu_nacc)} stops before the near-tie test {i}")
            validity_walk(name, gpu_x, gpu_out, gpu_nacc, ref)
            return
    if int(gpu_nacc) != n_ref:
        raise AssertionError(f"{name}: n_acc gpu {int(gpu_nacc)} oracle {n_ref}")
    tally.decisions += 1
    if ref["sample_margin"] < NEAR_TIE_DRAW:
        tally.near_ties += 1
        tally.notes.append(f"{name}: near-tie draw")
        validity_walk(name, gpu_x, gpu_out, gpu_nacc, ref)
        return
    if not np.array_equal(np.asarray(gpu_out), ref["out_tokens"]):
        raise AssertionError(f"{name}: out_tokens gpu {np.asarray(gpu_out).tolist()} "
                             f"oracle {ref['out_tokens'].tolist()}")
