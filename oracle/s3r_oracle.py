"""Float64 CPU oracle for one S3R decode step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or
executes this module; only the tests, the smoke check and the benchmark's CPU
baseline leg do. It shares no code with the CUDA path: the two meet only in
the seeded inputs of ``self_sparse_speculative_b200.workloads``, which hold no
arithmetic of the method.

Source of every definition: the S3R page ("S3R: Fast and Faithful RL Rollouts
via Self-Sparse Speculative Decoding", weekinpapers.com, Abstract) states the
method in one paragraph: draft tokens with sparse attention, generate through
full-attention verification and exact speculative sampling, with drafter and
verifier sharing one set of parameters, so that the committed tokens follow
the dense policy. The pieces it builds on are named on the mlsanity.com page's
reference list: Quest (query-aware page sparsity from per-page key min/max),
PagedAttention (block tables), and the two speculative-sampling papers ("Fast
Inference from Transformers via Speculative Decoding"; "Accelerating Large
Language Model Decoding with Speculative Sampling"). The accept/residual rule
is also restated on the ai.info SpecRoll page ("Exactness is preserved").

Every function is the plain definition: numpy float64, no blocking, fusion or
reordering beyond the definition. Readings where the pages are silent are
marked "reading:".

Pins (tests/test_oracle_pins.py): sparse == dense at full budget; attention ==
torch's scaled_dot_product_attention in float64 and hand-derived closed forms;
summaries bound every key; top-B == exhaustive subset search; q == p accepts
everything; chi-square of committed tokens against p over 1e6 trials;
acceptance rate == sum_x min(p, q); exact rational enumeration of the
committed-sequence distribution. Temperature (tests/test_oracle_temperature.py):
hand-derived cases at T = 0.5 and 0.7, chi-square and the acceptance rate at
T = 0.7, planted temperature slips caught. KV upkeep (tests/test_oracle_kv.py):
a dense per-sequence model over random rounds. Tree verification
(tests/test_oracle_tree.py): a chain equals ordinary speculative sampling and
causal verification; tree attention == SDPA with the ancestor mask; the
multi-draft rule by rational enumeration; chi-square over a two-level tree.
Parity unpinned (readings fixed by this build, not by the pages): the GQA
aggregation of the page score (sum over the query heads of a KV group) and
the absence of forced sink/recent pages in the top-B.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------- (a1) summaries
def page_summaries(k_cache, block_table, context_lens, page_size, tail_only=False,
                   kmin=None, kmax=None):
    """Per-page key minima and maxima (Quest's page metadata).

    kmin[p, h, d] = min over the valid tokens t of page p of K[p, h, t, d];
    kmax likewise. A sequence of length L uses tokens 0..L-1; its page i holds
    tokens i*P .. i*P+P-1, of which only those < L are valid.
    tail_only: recompute only each sequence's last page (the one a decode step
    appends to); every other page keeps its value in kmin/kmax.

    k_cache: float64 [num_pages_total, Hkv, P, D]; returns float64 arrays
    [num_pages_total, Hkv, D] (pages no sequence uses stay NaN unless given).
    """
    n_tot, H, P, D = k_cache.shape
    assert P == page_size
    kmin = np.full((n_tot, H, D), np.nan) if kmin is None else np.array(kmin, dtype=np.float64)
    kmax = np.full((n_tot, H, D), np.nan) if kmax is None else np.array(kmax, dtype=np.float64)
    for b, L in enumerate(np.asarray(context_lens).tolist()):
        n_b = -(-L // P)
        pages = [n_b - 1] if tail_only else range(n_b)
        for i in pages:
            phys = int(block_table[b, i])
            valid = min(P, L - i * P)
            kmin[phys] = k_cache[phys, :, :valid, :].min(axis=1)
            kmax[phys] = k_cache[phys, :, :valid, :].max(axis=1)
    return kmin, kmax


# ----------------------------------------------------------------- (a2) score + top-B
def page_scores(q, kmin_pages, kmax_pages, group):
    """Quest upper bound of q.k over a page, aggregated over a GQA group.

    For KV head h and page p:
        s(p) = sum_{g in group(h)} sum_d max(q[g,d] * kmin[p,h,d], q[g,d] * kmax[p,h,d])
    Each term bounds q[g,d]*k[t,d] for every token t of the page, so s(p)
    bounds the sum over the group of q_g . k_t. Reading: sum over the G query
    heads of the group, unscaled (1/sqrt(D) does not change the order).

    q: [Hq, D]; kmin_pages/kmax_pages: [n, Hkv, D]. Returns [Hkv, n].
    """
    n, H, D = kmin_pages.shape
    out = np.empty((H, n))
    for h in range(H):
        qg = q[h * group:(h + 1) * group]                        # [G, D]
        lo = qg[None, :, :] * kmin_pages[:, h, None, :]          # [n, G, D]
        hi = qg[None, :, :] * kmax_pages[:, h, None, :]
        out[h] = np.maximum(lo, hi).sum(axis=(1, 2))
    return out


def select_top_pages(scores, budget):
    """The `budget` highest-scoring pages, ascending by page index.

    Ties go to the lower page index. If there are no more pages than the
    budget, all pages are taken. Reading: no page (sink or most recent) is
    forced in. Also returns the gap between the last chosen and the first
    rejected score (inf when nothing is rejected) for near-tie accounting.
    """
    n = len(scores)
    if n <= budget:
        return np.arange(n, dtype=np.int64), np.inf
    order = sorted(range(n), key=lambda p: (-scores[p], p))
    chosen = np.array(sorted(order[:budget]), dtype=np.int64)
    gap = float(scores[order[budget - 1]] - scores[order[budget]])
    return chosen, gap


# ----------------------------------------------------------------- attention
def attend(q_rows, keys, values, valid, scale):
    """softmax(q k^T * scale) v over the valid keys of each row.

    q_rows [r, D], keys/values [n, D], valid bool [r, n]. Returns out [r, D]
    and the natural-log log-sum-exp lse [r] of the scaled scores. A row with no
    valid key gets out = 0 and lse = -inf.
    """
    s = (q_rows @ keys.T) * scale
    s = np.where(valid, s, NEG_INF)
    m = s.max(axis=1, initial=NEG_INF)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.where(valid, np.exp(s - m_safe[:, None]), 0.0)
    l = w.sum(axis=1)
    out = np.where(l[:, None] > 0, (w @ values) / np.where(l > 0, l, 1.0)[:, None], 0.0)
    lse = np.where(l > 0, m_safe + np.log(np.where(l > 0, l, 1.0)), NEG_INF)
    return out, lse


def _gather_tokens(cache, block_table, b, h, pages, L, P):
    """Rows of head h for the tokens of the listed logical pages of sequence b,
    with their token positions (only positions < L)."""
    rows, pos = [], []
    for lp in pages:
        phys = int(block_table[b, int(lp)])
        valid = min(P, L - int(lp) * P)
        rows.append(cache[phys, h, :valid, :])
        pos.append(int(lp) * P + np.arange(valid))
    return np.concatenate(rows), np.concatenate(pos)


def paged_attention(q, k_cache, v_cache, block_table, context_lens, scale,
                    page_lists=None):
    """Causal attention of the last R positions of each sequence over its paged cache.

    q: [S, R, Hq, D]; row r of sequence b sits at position L_b - R + r and sees
    keys at positions <= its own (causal). R = 1 is single-token decode at
    position L_b - 1.
    page_lists: None for all pages (dense); else page_lists[b][h] lists the
    logical pages KV head h may read (sparse drafting: only those pages).
    GQA: query head hq reads KV head hq // (Hq // Hkv).
    Returns out [S, R, Hq, D], lse [S, R, Hq].
    """
    S, R, Hq, D = q.shape
    H, P = k_cache.shape[1], k_cache.shape[2]
    G = Hq // H
    out = np.zeros((S, R, Hq, D))
    lse = np.zeros((S, R, Hq))
    for b in range(S):
        L = int(context_lens[b])
        n_b = -(-L // P)
        for h in range(H):
            pages = range(n_b) if page_lists is None else page_lists[b][h]
            K, pos = _gather_tokens(k_cache, block_table, b, h, pages, L, P)
            V, _ = _gather_tokens(v_cache, block_table, b, h, pages, L, P)
            heads = range(h * G, (h + 1) * G)
            qr = np.stack([q[b, r, hq] for r in range(R) for hq in heads])      # [R*G, D]
            qpos = np.array([L - R + r for r in range(R) for _ in heads])
            valid = pos[None, :] <= qpos[:, None]
            o, s = attend(qr, K, V, valid, scale)
            i = 0
            for r in range(R):
                for hq in heads:
                    out[b, r, hq] = o[i]
                    lse[b, r, hq] = s[i]
                    i += 1
    return out, lse


def dense_decode(q, k_cache, v_cache, block_table, context_lens, scale):
    """Single-query dense decode: q [S, Hq, D] at position L_b - 1."""
    o, l = paged_attention(q[:, None], k_cache, v_cache, block_table, context_lens, scale)
    return o[:, 0], l[:, 0]


def sparse_draft_select(q, kmin, kmax, block_table, context_lens, page_size, budget, group,
                        return_scores=False):
    """Step (a2) for every sequence: selected [S][Hkv] arrays of logical page ids
    (ascending) and the boundary score gaps [S, Hkv] relative to the largest
    |score| of the head. With return_scores, also the page scores [S] of
    [Hkv, n_b] arrays (for checking a choice at a near-tie boundary)."""
    S = q.shape[0]
    H = kmin.shape[1]
    sel, gaps, scores = [], np.full((S, H), np.inf), []
    for b in range(S):
        n_b = -(-int(context_lens[b]) // page_size)
        phys = block_table[b, :n_b]
        sc = page_scores(q[b], kmin[phys], kmax[phys], group)
        row = []
        for h in range(H):
            c, gap = select_top_pages(sc[h], budget)
            row.append(c)
            gaps[b, h] = gap / max(1e-300, float(np.abs(sc[h]).max()))
        sel.append(row)
        scores.append(sc)
    if return_scores:
        return sel, gaps, scores
    return sel, gaps


def sparse_draft_attn(q, k_cache, v_cache, block_table, context_lens, selected, scale):
    """Step (a3): decode at position L_b - 1 over the selected pages only."""
    o, l = paged_attention(q[:, None], k_cache, v_cache, block_table, context_lens, scale,
                           page_lists=selected)
    return o[:, 0], l[:, 0]


def verify_attn(q, k_cache, v_cache, block_table, context_lens, scale):
    """Step (a4): the R = gamma+1 verify rows, dense and causal over the whole history."""
    return paged_attention(q, k_cache, v_cache, block_table, context_lens, scale)


# ----------------------------------------------------------------- (a5) sampling
def softmax_t(logits, temperature):
    """softmax(logits / T) over the last axis."""
    x = np.asarray(logits, dtype=np.float64) / temperature
    m = x.max(axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=-1, keepdims=True)


def inverse_cdf(weights, u):
    """Inverse-CDF draw from unnormalised non-negative weights, one row per u.

    With C the running sum of the weights, returns the smallest k with
    C(k) > u * C(V-1), so zero-weight entries never win. If rounding leaves no
    such k, the last index with positive weight. Also returns the distance of
    u from the nearer boundary C(k-1)/C(V-1), C(k)/C(V-1) of the chosen token.
    weights [N, V], u [N] -> (k [N], margin [N]).
    """
    w = np.atleast_2d(np.asarray(weights, dtype=np.float64))
    u = np.atleast_1d(np.asarray(u, dtype=np.float64))
    C = np.cumsum(w, axis=1)
    total = C[:, -1]
    k = (C <= (u * total)[:, None]).sum(axis=1)
    V = w.shape[1]
    for i in np.nonzero(k >= V)[0]:
        k[i] = int(np.nonzero(w[i] > 0)[0][-1])
    lo = np.where(k > 0, C[np.arange(len(k)), np.maximum(k - 1, 0)], 0.0) / total
    hi = C[np.arange(len(k)), k] / total
    margin = np.minimum(np.abs(u - lo), np.abs(u - hi))
    return k.astype(np.int64), margin


def sample_rows(logits, u, temperature):
    """One token per row from softmax(logits / T) by inverse CDF (the drafter's
    own sampling of x_i ~ q_i). logits [N, V], u [N]."""
    return inverse_cdf(softmax_t(logits, temperature), u)


def residual_weights(p_j, q_j):
    """The distribution drawn from after a rejection at position j: the
    residual max(p_j - q_j, 0) (unnormalised; the draw normalises it), or p_j
    itself where the residual is zero everywhere (reading: p = q makes a
    rejection a probability-0 event, so any choice keeps the output exact).
    Works row-wise over the last axis."""
    resid = np.maximum(p_j - q_j, 0.0)
    return np.where(resid.sum(axis=-1, keepdims=True) > 0, resid, p_j)


def spec_sample(target_logits, draft_logits, draft_tokens, u_accept, u_sample, temperature):
    """Exact speculative sampling of one round, for every sequence.

    p_i = softmax(target_i / T) for i = 0..gamma, q_i = softmax(draft_i / T)
    for i < gamma. For i = 0..gamma-1 in order: accept x_i iff
    u_accept[i] < p_i(x_i) / q_i(x_i) (min(1, .) is moot for u < 1; reading:
    q_i(x_i) = 0 rejects). At the first rejection j, draw from the residual
    max(p_j - q_j, 0) normalised (reading: from p_j if the residual is all
    zero); if every draft is accepted, draw the bonus token from p_gamma. The
    draw is inverse_cdf with u_sample[j].

    target_logits [S, R, V], draft_logits [S, gamma, V], draft_tokens
    [S, gamma], u_accept [S, gamma], u_sample [S, R].
    Returns out_tokens [S, R] (committed tokens then -1), n_acc [S], and the
    decision margins: accept_margin [S, gamma] = |u - p/q| (NaN where not
    tested) and sample_margin [S].
    """
    S, R, V = target_logits.shape
    gamma = R - 1
    p = softmax_t(target_logits, temperature)                 # [S, R, V]
    q = softmax_t(draft_logits, temperature)                  # [S, gamma, V]
    x = np.asarray(draft_tokens, dtype=np.int64)
    si = np.arange(S)[:, None]
    gi = np.arange(gamma)[None, :]
    px = p[si, gi, x]
    qx = q[si, gi, x]
    ratio = np.where(qx > 0, px / np.where(qx > 0, qx, 1.0), 0.0)
    ua = np.asarray(u_accept, dtype=np.float64)
    accept = ua < ratio
    # number of leading accepts
    n_acc = np.cumprod(accept, axis=1).sum(axis=1).astype(np.int64)
    tested = gi <= n_acc[:, None]                              # tests actually made
    tested &= gi < gamma
    accept_margin = np.where(tested, np.abs(ua - ratio), np.nan)
    # the distribution of the token drawn at position n_acc
    j = n_acc
    p_j = p[np.arange(S), j]                                   # [S, V]
    q_j = q[np.arange(S), np.minimum(j, gamma - 1)]            # unused where j == gamma
    w = np.where((j == gamma)[:, None], p_j, residual_weights(p_j, q_j))
    us = np.asarray(u_sample, dtype=np.float64)[np.arange(S), j]
    k, sample_margin = inverse_cdf(w, us)
    out = np.where(gi < j[:, None], x, -1)
    out = np.concatenate([out, np.full((S, 1), -1, dtype=np.int64)], axis=1)
    out[np.arange(S), j] = k
    return out, n_acc, accept_margin, sample_margin


# ----------------------------------------------------------------- KV cache upkeep of a round
# The S3R page (Abstract) has the drafter and the verifier share the policy's
# parameters and its KV cache: a draft step adds its token's keys and values
# to the cache, verification recomputes the round's positions with dense
# attention (its keys and values replace the drafter's), and speculative
# sampling commits only the accepted prefix plus one drawn token, so the
# positions after it leave the cache. Reading: the round's positions are
# L - R .. L - 1 (verify row r at L - R + r, as above); a write refreshes the
# summaries of every page it touches (their valid tokens after the write).

def kv_append(k_cache, v_cache, block_table, context_lens, k_new, v_new, overwrite, page_size,
              kmin=None, kmax=None):
    """Write n new rows per sequence and refresh the touched pages' summaries.

    For sequence b with length L: the rows go to positions
    L - overwrite .. L - overwrite + n - 1 (overwrite = 0 appends at the end;
    overwrite > 0 first replaces the last `overwrite` positions), and the new
    length is L - overwrite + n. k_new, v_new: [S, n, Hkv, D]. The summaries of
    every page holding a written position are recomputed over the page's valid
    tokens under the new length (page_summaries' definition).
    Returns new k_cache, v_cache, context_lens, kmin, kmax (copies).
    """
    K = np.array(k_cache, dtype=np.float64)
    V = np.array(v_cache, dtype=np.float64)
    lens = np.array(context_lens, dtype=np.int64)
    S, n = k_new.shape[0], k_new.shape[1]
    n_tot, H, P, D = K.shape
    kmin = np.full((n_tot, H, D), np.nan) if kmin is None else np.array(kmin, dtype=np.float64)
    kmax = np.full((n_tot, H, D), np.nan) if kmax is None else np.array(kmax, dtype=np.float64)
    for b in range(S):
        start = int(lens[b]) - overwrite
        for t in range(n):
            pos = start + t
            phys = int(block_table[b, pos // P])
            K[phys, :, pos % P, :] = k_new[b, t]
            V[phys, :, pos % P, :] = v_new[b, t]
        new_len = start + n
        lens[b] = new_len
        for i in range(start // P, (new_len - 1) // P + 1) if n > 0 else ():
            phys = int(block_table[b, i])
            valid = min(P, new_len - i * P)
            kmin[phys] = K[phys, :, :valid, :].min(axis=1)
            kmax[phys] = K[phys, :, :valid, :].max(axis=1)
    return K, V, lens, kmin, kmax


def kv_rollback(k_cache, block_table, context_lens, num_accepted, rows, page_size, kmin, kmax):
    """Keep the committed prefix of a round and refresh the new tail page.

    After a round whose R = rows positions end the cache (length L), n_acc
    drafts accepted: the committed length is L - R + n_acc + 1 (the round's
    first position, whose token was committed by the previous round, plus the
    accepted drafts). The summary of the page holding the new last position is
    recomputed over its valid tokens. Returns new context_lens, kmin, kmax.
    """
    K = np.asarray(k_cache, dtype=np.float64)
    P = page_size
    lens = np.array(context_lens, dtype=np.int64)
    kmin = np.array(kmin, dtype=np.float64)
    kmax = np.array(kmax, dtype=np.float64)
    for b in range(len(lens)):
        new_len = int(lens[b]) - rows + int(num_accepted[b]) + 1
        lens[b] = new_len
        i = (new_len - 1) // P
        phys = int(block_table[b, i])
        valid = new_len - i * P
        kmin[phys] = K[phys, :, :valid, :].min(axis=1)
        kmax[phys] = K[phys, :, :valid, :].max(axis=1)
    return lens, kmin, kmax


# ----------------------------------------------------------------- tree verification
# The ai.info SpecRoll page (another speculative method for RL rollouts)
# verifies a sparse tree of proposals instead of a chain: each round gives a
# response a node budget N_t = clip(floor(C_hw / B_t), N_min, N_max) (C_hw the
# profiled capacity, B_t the unfinished responses), and exact rejection
# sampling with the target-residual fallback stays authoritative at every
# visited node, so the committed tokens still follow the target policy.
# Readings: a tree of R nodes in topological order (parent[0] = -1 is the
# round's first position, parent[i] < i), stored in the cache at the round's
# R positions in node order; node i attends to the committed history and to
# its ancestors and itself; the children of a node were drawn i.i.d. from
# that node's draft distribution and are tried in index order (each
# rejection replaces the target by its normalised residual), the sampling
# rule the speculative-sampling papers give for several drafts.

def node_budget(capacity, active, n_min, n_max):
    """N_t = clip(floor(C_hw / B_t), N_min, N_max)."""
    return int(min(max(capacity // active, n_min), n_max))


def tree_ancestor_masks(parents):
    """Bit j of mask[i] is set iff node j is node i or one of its ancestors."""
    R = len(parents)
    masks = [0] * R
    for i in range(R):
        m, v = 0, i
        while v >= 0:
            m |= 1 << v
            v = int(parents[v])
        masks[i] = m
    return masks


def tree_verify_attn(q, k_cache, v_cache, block_table, context_lens, parents, scale):
    """Dense attention of the R tree nodes of each sequence: node i sits at
    slot L - R + i and sees every key before L - R and the slots of its
    ancestors and itself. q [S, R, Hq, D], parents [S, R].
    Returns out [S, R, Hq, D], lse [S, R, Hq]."""
    S, R, Hq, D = q.shape
    H, P = k_cache.shape[1], k_cache.shape[2]
    G = Hq // H
    out = np.zeros((S, R, Hq, D))
    lse = np.zeros((S, R, Hq))
    for b in range(S):
        L = int(context_lens[b])
        n_b = -(-L // P)
        masks = tree_ancestor_masks(parents[b])
        for h in range(H):
            K, pos = _gather_tokens(k_cache, block_table, b, h, range(n_b), L, P)
            V, _ = _gather_tokens(v_cache, block_table, b, h, range(n_b), L, P)
            heads = range(h * G, (h + 1) * G)
            qr = np.stack([q[b, r, hq] for r in range(R) for hq in heads])
            node = np.array([r for r in range(R) for _ in heads])
            j = pos[None, :] - (L - R)                                     # tree slot of each key (< 0: history)
            m = np.array(masks, dtype=np.uint64)[node][:, None]                # up to 64 nodes: unsigned
            valid = (j < 0) | ((m >> np.maximum(j, 0).astype(np.uint64)) & np.uint64(1)).astype(bool)
            o, s = attend(qr, K, V, valid, scale)
            i = 0
            for r in range(R):
                for hq in heads:
                    out[b, r, hq] = o[i]
                    lse[b, r, hq] = s[i]
                    i += 1
    return out, lse


def tree_spec_sample(target_logits, draft_logits, tokens, parents, u_accept, u_sample, temperature):
    """Exact speculative sampling over a tree, per sequence.

    p_v = softmax(target_logits[v] / T), q_v = softmax(draft_logits[v] / T)
    (the distribution node v's children were drawn from). From the root:
    at node v the children c (ascending index) are tested in turn, accept c iff
    u_accept[c] < p'(x_c) / q_v(x_c) with p' = p_v at first and, after each
    rejection, p' = max(p' - q_v, 0) normalised (p' itself where that is all
    zero); an accepted child commits its token and becomes v. When no child
    is accepted (or v has none) the token drawn from p' with u_sample[v]
    (inverse CDF) is committed and the round ends.
    target_logits, draft_logits [S, R, V]; tokens, parents, u_accept,
    u_sample [S, R]. Returns out_tokens [S, R] (committed tokens, then -1),
    n_acc [S] (accepted nodes), path [S, R] (the accepted nodes, then -1), and
    the margins of every accept test and of the final draw (for near-ties).
    """
    S, R, V = target_logits.shape
    p = softmax_t(target_logits, temperature)
    q = softmax_t(draft_logits, temperature)
    out = np.full((S, R), -1, dtype=np.int64)
    path = np.full((S, R), -1, dtype=np.int64)
    n_acc = np.zeros(S, dtype=np.int64)
    accept_margins = [[] for _ in range(S)]
    draw_margin = np.zeros(S)
    for b in range(S):
        v, depth = 0, 0
        while True:
            children = [c for c in range(R) if int(parents[b, c]) == v]
            pr = p[b, v]
            nxt = None
            for c in children:
                x = int(tokens[b, c])
                qx = q[b, v, x]
                ratio = pr[x] / qx if qx > 0 else 0.0
                accept_margins[b].append(abs(float(u_accept[b, c]) - ratio))
                if float(u_accept[b, c]) < ratio:
                    nxt = c
                    break
                resid = residual_weights(pr, q[b, v])
                pr = resid / resid.sum()
            if nxt is None:
                k, margin = inverse_cdf(pr[None], np.array([float(u_sample[b, v])]))
                out[b, depth] = int(k[0])
                draw_margin[b] = float(margin[0])
                break
            out[b, depth] = int(tokens[b, nxt])
            path[b, depth] = nxt
            depth += 1
            v = nxt
        n_acc[b] = depth
    return out, n_acc, path, accept_margins, draw_margin


def chain_parents(R):
    """The chain tree (ordinary speculative decoding): parent[i] = i - 1."""
    return np.arange(-1, R - 1)


def build_tree(n_nodes, branching):
    """A tree of n_nodes in breadth-first order: every node of depth d gets
    branching[d] children (the last entry repeats) until n_nodes exist.
    Returns parents [n_nodes]. Reading: SpecRoll picks the tree from its
    heads' candidate probabilities; without those heads the shape is given."""
    parents = [-1]
    frontier = [0]
    d = 0
    while len(parents) < n_nodes and frontier:
        k = branching[min(d, len(branching) - 1)]
        nxt = []
        for v in frontier:
            for _ in range(k):
                if len(parents) >= n_nodes:
                    break
                parents.append(v)
                nxt.append(len(parents) - 1)
        frontier = nxt
        d += 1
    return np.array(parents, dtype=np.int64)
