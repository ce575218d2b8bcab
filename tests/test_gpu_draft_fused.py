"""The sparse draft call against the float64 oracle, on shapes that reach each
path of the fused kernel (page scoring, top-B and attention in one launch):
units cut into pieces over clusters of two and four CTAs, budgets on both
sides of 32 pages, pieces that keep no page, bad
lengths and page ids, and queries and tail-page keys written by the caller's
own kernels right before the call; plus launches with more units than SMs,
which take the selection kernel (persistent CTAs claiming units from a
workspace counter) and the split-KV attention kernel. Every GPU
result comes from the C ABI (libs3r.so)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from self_sparse_speculative_b200 import s3r                      # noqa: E402
from self_sparse_speculative_b200.step import DecodeStep          # noqa: E402
from self_sparse_speculative_b200.workloads import (               # noqa: E402
    Workload, custom_spec, round_to_bf16_bits, to_float64)

import oracle as O                                                 # noqa: E402
import oracle.reference_run as RR                                  # noqa: E402


def _ragged(n, lo, hi, seed):
    return np.random.default_rng(seed).integers(lo, hi, size=n).tolist()


CASES = {
    # 400 units, more than the SMs: the selection kernel and the split-KV
    # attention kernel; 16-token pages (eight pages per stage)
    "many-units-p16": (custom_spec(1, num_seqs=200, num_q_heads=8, num_kv_heads=2, page_size=16, gamma=2,
                                   budget_pages=5, vocab=512), _ragged(200, 40, 700, 1)),
    # one unit: cut into four pieces of 200 pages each
    "long-chunks": (custom_spec(1, num_seqs=1, num_q_heads=4, num_kv_heads=1, page_size=16, gamma=1,
                                budget_pages=9, vocab=512), [800 * 16 - 5]),
    # split units whose kept-page list is shorter than the number of pieces
    "empty-pieces": (custom_spec(1, num_seqs=2, num_q_heads=8, num_kv_heads=2, page_size=64, gamma=1,
                                 budget_pages=4, vocab=512), [100, 64 * 9 + 3]),
    # budgets between 32 and 64 pages (the 64-key bitonic selection): units
    # cut into four pieces with up to ~940 pages each, some below the budget
    "top64-clusters": (custom_spec(1, num_seqs=3, num_q_heads=8, num_kv_heads=4, page_size=16, gamma=1,
                                   budget_pages=48, vocab=512), [1000, 9000, 15000]),
    # the same budgets through the selection kernel (160 units)
    "top64-selection-kernel": (custom_spec(1, num_seqs=80, num_q_heads=4, num_kv_heads=2, page_size=16, gamma=1,
                                           budget_pages=64, vocab=512), _ragged(80, 700, 9000, 3)),
    # 640 units, more than the selection kernel's resident CTAs: CTAs claim
    # further units from the workspace counter (ragged lengths)
    "selection-claims": (custom_spec(1, num_seqs=320, num_q_heads=4, num_kv_heads=2, page_size=16, gamma=2,
                                     budget_pages=6, vocab=512), _ragged(320, 50, 3000, 5)),
    # the selection kernel, 16-token pages and a 34-page budget: units end
    # mid-stage inside the split-KV attention's 41-page CTA ranges
    "selection-p16-budget34": (custom_spec(1, num_seqs=100, num_q_heads=8, num_kv_heads=2, page_size=16, gamma=1,
                                           budget_pages=34, vocab=512), _ragged(100, 16 * 6, 16 * 60, 11)),
    # D = 64 through the selection kernel (200 units), budget 40 (the 64-key select)
    "d64-selection-top64": (custom_spec(1, num_seqs=100, num_q_heads=16, num_kv_heads=2, head_dim=64, page_size=64,
                                        gamma=1, budget_pages=40, vocab=512), _ragged(100, 1500, 6400, 6)),
    # D = 64, G = 8: 60 units, each cut into two pieces (clusters of two CTAs)
    "d64-g8-pairs": (custom_spec(1, num_seqs=30, num_q_heads=16, num_kv_heads=2, head_dim=64, page_size=64,
                                 gamma=1, budget_pages=3, vocab=512), _ragged(30, 130, 2000, 2)),
}


def _check(name, wl, st, steps):
    tally = RR.Tally()
    sel = st.selected.cpu().numpy()
    out = st.draft_out.float().cpu().numpy()
    lse = st.draft_lse.cpu().numpy()
    for b in range(wl.spec.num_seqs):
        ref = RR.oracle_attention_seq(wl, b, draft_steps=steps)
        n_b = int(wl.pages_per_seq[b])
        for i, d in ref["draft"].items():
            ok = RR.compare_selection(f"{name} seq {b} draft {i}", sel[i, b], d["selected"], d["gaps"], tally,
                                      scores=d["scores"])
            assert np.all(sel[i, b][:, min(n_b, wl.spec.budget_pages):] == -1)
            if all(ok):
                RR.assert_close(f"{name} seq {b} draft {i} out", out[i, b], d["out"], "bf16")
                RR.assert_close(f"{name} seq {b} draft {i} lse", lse[i, b], d["lse"], "bf16")
    assert tally.near_ties <= max(0, int(1e-4 * tally.decisions)), tally.notes


@pytest.mark.parametrize("name", list(CASES))
def test_fused_draft_matches_oracle(name):
    s, lens = CASES[name]
    wl = Workload(s, seed=4, context_lens=lens)
    st = DecodeStep(wl)
    st.summaries(tail_only=False)
    for i in range(s.gamma):
        st.draft(i)
    torch.cuda.synchronize()
    assert s3r.s3r_device_status(st.ws_draft) == (s3r.S3R_OK, 0)
    _check(name, wl, st, list(range(s.gamma)))
    # a second call on the same workspace (tickets and lists reset by the first)
    st.draft(0)
    torch.cuda.synchronize()
    assert s3r.s3r_device_status(st.ws_draft) == (s3r.S3R_OK, 0)
    _check(name, wl, st, [0])


@pytest.mark.parametrize("num_seqs", [3, 100], ids=["fused", "selection-kernel"])
def test_fused_draft_flags_bad_inputs_without_faulting(num_seqs):
    """A bad context length and an out-of-range block-table entry are recorded
    in the status word; the unusable unit gets zeros, lse -inf and no pages,
    and the other sequences are unaffected (one fused kernel, or with more
    units than SMs the selection kernel and the split-KV attention)."""
    s = custom_spec(1, num_seqs=num_seqs, num_q_heads=8, num_kv_heads=2, budget_pages=2, vocab=512)
    wl = Workload(s, seed=2, context_lens=([300, 200, 330] + [150 + 7 * i for i in range(num_seqs - 3)]))
    st = DecodeStep(wl)
    st.summaries()
    torch.cuda.synchronize()
    st.context_lens[1] = 0
    st.block_table[2, 1] = wl.num_pages_total + 5
    st.draft(0)
    status, bits = s3r.s3r_device_status(st.ws_draft)
    assert status == s3r.S3R_ERR_DEVICE_CHECK
    assert bits & s3r.S3R_DEV_BAD_CONTEXT_LEN and bits & s3r.S3R_DEV_BAD_PAGE_ID
    assert not bits & s3r.S3R_DEV_WAIT_TIMEOUT
    assert np.all(st.selected[0, 1].cpu().numpy() == -1)
    out = st.draft_out[0].float().cpu().numpy()
    lse = st.draft_lse[0].cpu().numpy()
    assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(out[2]))
    ref = RR.oracle_attention_seq(wl, 0, draft_steps=[0])
    d = ref["draft"][0]
    tally = RR.Tally()
    if all(RR.compare_selection("seq 0", st.selected[0, 0].cpu().numpy(), d["selected"], d["gaps"], tally,
                                scores=d["scores"])):
        RR.assert_close("seq 0 draft out", out[0], d["out"], "bf16")
    # the same workspace is clean again once the inputs are
    st.context_lens[1] = 200
    st.block_table[2, 1] = int(wl.block_table[2, 1])
    st.draft(0)
    assert s3r.s3r_device_status(st.ws_draft) == (s3r.S3R_OK, 0)


def test_caller_written_tail_keys_and_query_are_seen():
    """Kernels of the caller's (torch copies on the same stream, no sync)
    write a new key into every sequence's tail page and a new draft query
    right before the call: the selection and the outputs follow the new
    values (oracle on the same host-side values)."""
    s = custom_spec(1, num_seqs=3, num_q_heads=8, num_kv_heads=2, budget_pages=3, vocab=512)
    lens = [700, 64 * 7 + 1, 1000]
    wl = Workload(s, seed=9, context_lens=lens)
    st = DecodeStep(wl)
    st.summaries(tail_only=False)
    torch.cuda.synchronize()
    rng = np.random.default_rng(31)
    H, P, D, Hq = s.num_kv_heads, s.page_size, s.head_dim, s.num_q_heads
    K = wl.kv_cache("K").copy()                       # bf16 bit patterns [pages, H, P, D]
    V = wl.kv_cache("V")
    new_q = round_to_bf16_bits(rng.standard_normal((s.num_seqs, Hq, D), dtype=np.float32))
    for b, L in enumerate(lens):
        n = int(wl.pages_per_seq[b])
        ph = int(wl.block_table[b, n - 1])
        t = (L - 1) % P
        # a key aligned with the new query rows of each head, scaled up: the
        # tail page's summary moves, so its score does
        qh = to_float64(new_q[b], "bf16").reshape(H, Hq // H, D).sum(axis=1)
        row = round_to_bf16_bits((4.0 * np.sign(qh) + 0.5 * rng.standard_normal((H, D))).astype(np.float32))
        K[ph, :, t, :] = row
        st.k_cache[ph, :, t, :] = torch.from_numpy(row.view(np.int16)).view(torch.bfloat16).cuda(non_blocking=True)
    st.q_draft[0].copy_(torch.from_numpy(new_q.view(np.int16)).view(torch.bfloat16).cuda(non_blocking=True))
    st.draft(0)                                        # same stream, no synchronisation in between
    torch.cuda.synchronize()
    assert s3r.s3r_device_status(st.ws_draft) == (s3r.S3R_OK, 0)
    # oracle on the same values
    bt = wl.block_table.astype(np.int64)
    K64, V64 = to_float64(K, "bf16"), to_float64(V, "bf16")
    q64 = to_float64(new_q, "bf16")
    cl = np.asarray(lens)
    kmin, kmax = O.page_summaries(K64, bt, cl, P)
    sel, gaps, scores = O.sparse_draft_select(q64, kmin, kmax, bt, cl, P, s.budget_pages, s.group,
                                              return_scores=True)
    out, lse = O.sparse_draft_attn(q64, K64, V64, bt, cl, sel, RR.f32(wl.scale))
    tally = RR.Tally()
    gsel = st.selected[0].cpu().numpy()
    gout = st.draft_out[0].float().cpu().numpy()
    moved = 0
    for b in range(s.num_seqs):
        n = int(wl.pages_per_seq[b])
        moved += sum(int(n - 1 in sel[b][h]) for h in range(H))
        if all(RR.compare_selection(f"seq {b}", gsel[b], sel[b], gaps[b], tally, scores=scores[b])):
            RR.assert_close(f"seq {b} out", gout[b], out[b], "bf16")
    assert moved > 0                                   # the new keys changed the selection


@pytest.mark.parametrize("num_seqs,heads,budget", [(2, 2, 5), (40, 2, 3), (100, 2, 4)],
                         ids=["clusters", "one-cta-per-unit", "selection-kernel"])
def test_exact_ties_go_to_the_lower_page(num_seqs, heads, budget):
    """Every page of a sequence but the tail is a copy of its first page, so
    their page scores are exactly equal: float32 cannot order them and the
    float64 re-scoring with ties to the lower page decides. The kept pages
    are exactly the oracle's (the lowest page ids, plus the tail page when
    it scores higher); the outputs follow."""
    s = custom_spec(1, num_seqs=num_seqs, num_q_heads=4 * heads, num_kv_heads=heads, page_size=64, gamma=1,
                    budget_pages=budget, vocab=512)
    lens = _ragged(num_seqs, 64 * 6, 64 * 20, 7)
    wl = Workload(s, seed=12, context_lens=lens)
    st = DecodeStep(wl)
    K = wl.kv_cache("K").copy()                       # bf16 bit patterns [pages, H, P, D]
    V = wl.kv_cache("V")
    bt = wl.block_table.astype(np.int64)
    for b in range(num_seqs):
        n = int(wl.pages_per_seq[b])
        for j in range(1, n - 1):
            K[bt[b, j]] = K[bt[b, 0]]
    st.k_cache.copy_(torch.from_numpy(K.view(np.int16)).view(torch.bfloat16).cuda())
    st.summaries(tail_only=False)
    st.draft(0)
    torch.cuda.synchronize()
    assert s3r.s3r_device_status(st.ws_draft) == (s3r.S3R_OK, 0)
    K64, V64 = to_float64(K, "bf16"), to_float64(V, "bf16")
    q64 = to_float64(wl.q_draft[0], "bf16")
    cl = np.asarray(lens)
    kmin, kmax = O.page_summaries(K64, bt, cl, s.page_size)
    sel, _ = O.sparse_draft_select(q64, kmin, kmax, bt, cl, s.page_size, budget, s.group)
    out, lse = O.sparse_draft_attn(q64, K64, V64, bt, cl, sel, RR.f32(wl.scale))
    gsel = st.selected[0].cpu().numpy()
    gout = st.draft_out[0].float().cpu().numpy()
    ties = 0
    for b in range(num_seqs):
        for h in range(heads):
            assert gsel[b, h].tolist() == list(sel[b][h]), (b, h, gsel[b, h].tolist(), list(sel[b][h]))
            ties += int(1 in sel[b][h])
        RR.assert_close(f"seq {b} out", gout[b], out[b], "bf16")
    assert ties > 0                                    # the tie rule decided


@pytest.mark.parametrize("num_seqs,heads,budget", [(2, 2, 5), (40, 2, 3), (100, 2, 4)],
                         ids=["clusters", "one-cta-per-unit", "selection-kernel"])
def test_near_ties_inside_the_float32_band_follow_float64(num_seqs, heads, budget):
    """Pages that float32 cannot order but float64 can: every page but the
    tail copies the first page, then page j raises the largest key of one
    channel by j bf16 ulps, and every query head weighs that channel by 2^-16.
    The page scores then differ by ~1e-9 of their size: well inside the
    float32 rounding band (so the float64 re-scoring decides) and far above
    the comparison's near-tie threshold (1e-12), so the kept pages must be
    exactly the oracle's: the highest raises (and the tail page when it
    scores higher)."""
    s = custom_spec(1, num_seqs=num_seqs, num_q_heads=4 * heads, num_kv_heads=heads, page_size=64, gamma=1,
                    budget_pages=budget, vocab=512)
    lens = _ragged(num_seqs, 64 * 6, 64 * 20, 9)
    wl = Workload(s, seed=13, context_lens=lens)
    st = DecodeStep(wl)
    c0 = 5                                            # the raised channel
    K = wl.kv_cache("K").copy()                       # bf16 bit patterns [pages, H, P, D]
    V = wl.kv_cache("V")
    bt = wl.block_table.astype(np.int64)
    Kf = to_float64(K, "bf16")
    for b in range(num_seqs):
        n = int(wl.pages_per_seq[b])
        p0 = bt[b, 0]
        for j in range(1, n - 1):
            K[bt[b, j]] = K[p0]
            for h in range(heads):
                t = int(np.argmax(Kf[p0, h, :, c0]))
                x = int(K[p0, h, t, c0])
                assert x < 0x8000                      # a positive largest key: its bits grow with it
                K[bt[b, j], h, t, c0] = np.uint16(x + j)
    q = wl.q_draft[0].copy()                          # [S, Hq, D] bf16 bits
    q[:, :, c0] = np.uint16(0x3780)                   # 2^-16
    st.k_cache.copy_(torch.from_numpy(K.view(np.int16)).view(torch.bfloat16).cuda())
    st.q_draft[0].copy_(torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).cuda())
    st.summaries(tail_only=False)
    st.draft(0)
    torch.cuda.synchronize()
    assert s3r.s3r_device_status(st.ws_draft) == (s3r.S3R_OK, 0)
    K64, V64 = to_float64(K, "bf16"), to_float64(V, "bf16")
    q64 = to_float64(q, "bf16")
    cl = np.asarray(lens)
    kmin, kmax = O.page_summaries(K64, bt, cl, s.page_size)
    sel, gaps = O.sparse_draft_select(q64, kmin, kmax, bt, cl, s.page_size, budget, s.group)
    out, lse = O.sparse_draft_attn(q64, K64, V64, bt, cl, sel, RR.f32(wl.scale))
    gsel = st.selected[0].cpu().numpy()
    gout = st.draft_out[0].float().cpu().numpy()
    decided = 0
    for b in range(num_seqs):
        n = int(wl.pages_per_seq[b])
        for h in range(heads):
            assert gaps[b][h] > RR.NEAR_TIE_SCORE      # not a near-tie: an exact comparison
            assert gsel[b, h].tolist() == list(sel[b][h]), (b, h, gsel[b, h].tolist(), list(sel[b][h]))
            decided += int(n > budget and (n - 2) in set(int(x) for x in sel[b][h]))
        RR.assert_close(f"seq {b} out", gout[b], out[b], "bf16")
    assert decided > 0                                # the raises decided


@pytest.mark.parametrize("num_seqs,heads,budget", [(2, 2, 5), (40, 2, 3), (100, 2, 34)],
                         ids=["clusters", "one-cta-per-unit", "selection-kernel-top64"])
def test_zero_queries_keep_the_lowest_pages(num_seqs, heads, budget):
    """All-zero queries: every page scores exactly 0 (the rounding bound is 0
    too, and the band's edges are the two zeros), so the float64 tie rule
    keeps the lowest pages; attention over them gives the mean of their
    values (uniform weights)."""
    s = custom_spec(1, num_seqs=num_seqs, num_q_heads=4 * heads, num_kv_heads=heads, page_size=16, gamma=1,
                    budget_pages=budget, vocab=512)
    lens = _ragged(num_seqs, 16 * 6, 16 * 60, 11)
    wl = Workload(s, seed=14, context_lens=lens)
    st = DecodeStep(wl)
    st.q_draft[0].zero_()
    st.summaries(tail_only=False)
    st.draft(0)
    torch.cuda.synchronize()
    assert s3r.s3r_device_status(st.ws_draft) == (s3r.S3R_OK, 0)
    K64, V64 = to_float64(wl.kv_cache("K"), "bf16"), to_float64(wl.kv_cache("V"), "bf16")
    q64 = np.zeros_like(to_float64(wl.q_draft[0], "bf16"))
    bt = wl.block_table.astype(np.int64)
    cl = np.asarray(lens)
    kmin, kmax = O.page_summaries(K64, bt, cl, s.page_size)
    sel, _ = O.sparse_draft_select(q64, kmin, kmax, bt, cl, s.page_size, budget, s.group)
    out, lse = O.sparse_draft_attn(q64, K64, V64, bt, cl, sel, RR.f32(wl.scale))
    gsel = st.selected[0].cpu().numpy()
    gout = st.draft_out[0].float().cpu().numpy()
    for b in range(num_seqs):
        n = int(wl.pages_per_seq[b])
        for h in range(heads):
            assert list(sel[b][h]) == list(range(min(n, budget)))
            assert gsel[b, h].tolist()[:min(n, budget)] == list(range(min(n, budget))), (b, h, gsel[b, h].tolist())
        RR.assert_close(f"seq {b} out", gout[b], out[b], "bf16")
