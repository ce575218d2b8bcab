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
  the exact comparison (the GPU's choice there is checked for validity).
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


def oracle_attention_seq(wl, b, draft_steps=None):
    """Oracle summaries, page selection, sparse draft and verify attention of
    sequence b. draft_steps: which draft queries to run (default: all)."""
    ws = wl.spec
    P, B, G = ws.page_size, ws.budget_pages, ws.group
    scale = f32(wl.scale)
    K, V, bt, phys = sequence_cache(wl, b)
    lens = wl.context_lens[b:b + 1].astype(np.int64)
    kmin, kmax = O.page_summaries(K, bt, lens, P)
    steps = range(ws.gamma) if draft_steps is None else draft_steps
    draft = {}
    for i in steps:
        q = to_float64(wl.q_draft[i, b], ws.kv_dtype)[None]            # [1, Hq, D]
        sel, gaps = O.sparse_draft_select(q, kmin, kmax, bt, lens, P, B, G)
        out, lse = O.sparse_draft_attn(q, K, V, bt, lens, sel, scale)
        draft[i] = {"selected": sel[0], "gaps": gaps[0], "out": out[0], "lse": lse[0], "q": q}
    qv = to_float64(wl.q_verify[b], ws.kv_dtype)[None]                  # [1, R, Hq, D]
    vout, vlse = O.verify_attn(qv, K, V, bt, lens, scale)
    return {"phys": phys, "kmin": kmin, "kmax": kmax, "draft": draft,
            "verify_out": vout[0], "verify_lse": vlse[0], "K": K, "V": V, "bt": bt, "lens": lens}


def oracle_sampling_seq(wl, b):
    """Oracle draft-token draws and speculative sampling of sequence b."""
    ws = wl.spec
    T = f32(ws.temperature)
    t, d = wl.logits_for_seq(b)
    tl = to_float64(t, ws.logit_dtype)
    dl = to_float64(d, ws.logit_dtype)
    x, xm = O.sample_rows(dl, wl.u_draft[b].astype(np.float64), T)
    out, n_acc, am, sm = O.spec_sample(tl[None], dl[None], x[None], wl.u_accept[b][None],
                                       wl.u_sample[b][None], T)
    return {"x": x, "x_margin": xm, "out_tokens": out[0], "n_acc": int(n_acc[0]),
            "accept_margin": am[0], "sample_margin": float(sm[0])}


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


def compare_selection(name, gpu_sel, ref_sel, gaps, tally: Tally, scores=None):
    """gpu_sel [Hkv, B] (-1 padded), ref_sel list of arrays, gaps [Hkv]."""
    ok_heads = []
    for h, rs in enumerate(ref_sel):
        tally.decisions += 1
        g = np.asarray(gpu_sel[h])
        g = g[g >= 0]
        if gaps[h] <= NEAR_TIE_SCORE:
            tally.near_ties += 1
            tally.notes.append(f"{name} head {h}: near-tie page boundary")
            ok_heads.append(False)
            continue
        if not np.array_equal(g, np.asarray(rs)):
            raise AssertionError(f"{name} head {h}: selected pages differ: gpu {g.tolist()} oracle {list(rs)}")
        ok_heads.append(True)
    return ok_heads


def compare_sampling(name, gpu_x, gpu_out, gpu_nacc, ref, tally: Tally):
    """Exact comparison of one sequence's draft draws, accept decisions and
    drawn token, leaving out everything downstream of a near-tie."""
    gamma = len(ref["x"])
    for i in range(gamma):
        tally.decisions += 1
        if ref["x_margin"][i] < NEAR_TIE_DRAW:
            tally.near_ties += 1
            tally.notes.append(f"{name}: near-tie draft draw {i}")
            return
        if int(gpu_x[i]) != int(ref["x"][i]):
            raise AssertionError(f"{name}: draft token {i} gpu {int(gpu_x[i])} oracle {int(ref['x'][i])}")
    n_ref = ref["n_acc"]
    for i in range(min(gamma, n_ref + 1)):
        tally.decisions += 1
        if ref["accept_margin"][i] < NEAR_TIE_DECISION:
            tally.near_ties += 1
            tally.notes.append(f"{name}: near-tie accept test {i}")
            return
    if int(gpu_nacc) != n_ref:
        raise AssertionError(f"{name}: n_acc gpu {int(gpu_nacc)} oracle {n_ref}")
    tally.decisions += 1
    if ref["sample_margin"] < NEAR_TIE_DRAW:
        tally.near_ties += 1
        tally.notes.append(f"{name}: near-tie draw")
        g = np.asarray(gpu_out)
        if not np.array_equal(g[:n_ref], ref["out_tokens"][:n_ref]) or np.any(g[n_ref + 1:] != -1):
            raise AssertionError(f"{name}: committed tokens around a near-tie draw differ")
        return
    if not np.array_equal(np.asarray(gpu_out), ref["out_tokens"]):
        raise AssertionError(f"{name}: out_tokens gpu {np.asarray(gpu_out).tolist()} "
                             f"oracle {ref['out_tokens'].tolist()}")
