"""GPU vs float64 oracle on small workloads that the oracle finishes in
seconds: several tiles, several splits, ragged and partial pages, both the
M=64 and M=128 tensor-core tiles, head_dim 64/128, page 16/64, fp32 and bf16.
Every GPU result comes from the C ABI (libs3r.so)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from self_sparse_speculative_b200 import s3r                      # noqa: E402
from self_sparse_speculative_b200.step import DecodeStep          # noqa: E402
from self_sparse_speculative_b200.workloads import Workload, custom_spec, spec, to_float64  # noqa: E402

import oracle.reference_run as RR                                  # noqa: E402

CASES = {
    # the tiny fp32 workload itself
    "tiny-fp32": (spec(0), None),
    # bf16, D128, P64, G4, R5 -> 20 packed rows (M=64 tile); a sequence with
    # fewer pages than the budget, a partial tail page, several splits
    "bf16-d128-p64": (custom_spec(1, num_seqs=3, num_q_heads=8, num_kv_heads=2, budget_pages=4, vocab=1000),
                      [130, 64, 1007 + 1024]),
    # G8 x R9 = 72 packed rows -> M=128 tile
    "bf16-g8-r9": (custom_spec(1, num_seqs=2, num_q_heads=16, num_kv_heads=2, gamma=8, budget_pages=3,
                               vocab=2048), [300, 777]),
    # D64 with 16-token pages (four pages per 64-token stage)
    "bf16-d64-p16": (custom_spec(1, num_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=64, page_size=16,
                                 gamma=3, budget_pages=6, vocab=999), [500, 33, 16 * 40 + 5]),
    # 16-token pages (eight per 128-token stage), many short ragged units:
    # a CTA's range of more than 32 pages holds three or more units, and a
    # unit ending mid-stage inside it must not move the page-id windows past
    # the next unit's first page (20 rows, then 72 rows)
    "bf16-p16-wide": (custom_spec(1, num_seqs=200, num_q_heads=8, num_kv_heads=2, page_size=16, gamma=4,
                                  budget_pages=13, vocab=512),
                      np.random.default_rng(21).integers(96, 600, size=200).tolist()),
    "bf16-p16-wide-r9": (custom_spec(1, num_seqs=160, num_q_heads=16, num_kv_heads=2, page_size=16, gamma=8,
                                     budget_pages=5, vocab=512),
                         np.random.default_rng(22).integers(150, 700, size=160).tolist()),
    # fp32 with D128, P64 and fp32 logits
    "f32-d128-p64": (custom_spec(0, num_seqs=2, num_q_heads=6, num_kv_heads=2, head_dim=128, page_size=64,
                                 budget_pages=2, vocab=777), [200, 4 * 64 + 1]),
    # the largest packed tile: G8 x R16 = 128 rows
    "bf16-g8-r16": (custom_spec(1, num_seqs=2, num_q_heads=16, num_kv_heads=2, gamma=15, budget_pages=2,
                                vocab=1536), [200, 64 * 5]),
    # shortest legal history: L = R for verify
    "bf16-min-len": (custom_spec(1, num_seqs=2, num_q_heads=4, num_kv_heads=1, gamma=2, budget_pages=1,
                                 vocab=512), [3, 70]),
}


def _run(name):
    s, lens = CASES[name]
    wl = Workload(s, seed=1, context_lens=lens)
    st = DecodeStep(wl)
    st.summaries(tail_only=False)
    st.round()
    torch.cuda.synchronize()
    return wl, st


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    return request.param, _run(request.param)


def test_device_status_clean(case):
    name, (wl, st) = case
    for ws_name, (status, bits) in st.device_checks().items():
        assert status == s3r.S3R_OK, f"{name} {ws_name}: device status bits {bits:#x}"


def test_summaries_bit_exact(case):
    name, (wl, st) = case
    dt = wl.spec.kv_dtype
    kmin = st.kmin.float().cpu().numpy().astype(np.float64)
    kmax = st.kmax.float().cpu().numpy().astype(np.float64)
    for b in range(wl.spec.num_seqs):
        ref = RR.oracle_attention_seq(wl, b, draft_steps=[])
        assert np.array_equal(kmin[ref["phys"]], ref["kmin"]), f"{name} seq {b} kmin"
        assert np.array_equal(kmax[ref["phys"]], ref["kmax"]), f"{name} seq {b} kmax"


def test_selection_and_attention(case):
    name, (wl, st) = case
    ws = wl.spec
    dt = ws.kv_dtype
    tally = RR.Tally()
    sel = st.selected.cpu().numpy()
    dout = st.draft_out.float().cpu().numpy()
    dlse = st.draft_lse.cpu().numpy()
    vout = st.verify_out.float().cpu().numpy()
    vlse = st.verify_lse.cpu().numpy()
    for b in range(ws.num_seqs):
        ref = RR.oracle_attention_seq(wl, b)
        for i, d in ref["draft"].items():
            ok = RR.compare_selection(f"{name} seq {b} draft {i}", sel[i, b], d["selected"], d["gaps"], tally,
                                      scores=d["scores"])
            n_b = int(wl.pages_per_seq[b])
            assert np.all(sel[i, b][:, min(n_b, ws.budget_pages):] == -1)
            if all(ok):
                RR.assert_close(f"{name} seq {b} draft {i} out", dout[i, b], d["out"], dt)
                RR.assert_close(f"{name} seq {b} draft {i} lse", dlse[i, b], d["lse"], dt)
        RR.assert_close(f"{name} seq {b} verify out", vout[b], ref["verify_out"], dt)
        RR.assert_close(f"{name} seq {b} verify lse", vlse[b], ref["verify_lse"], dt)
    assert tally.near_ties <= max(0, int(1e-4 * tally.decisions)), tally.notes


def test_sampling_round(case):
    """Draft draws, accept/reject and the drawn token of the GPU round."""
    name, (wl, st) = case
    tally = RR.Tally()
    x = st.draft_tokens.cpu().numpy()
    out = st.out_tokens.cpu().numpy()
    nacc = st.num_accepted.cpu().numpy()
    for b in range(wl.spec.num_seqs):
        ref = RR.oracle_sampling_seq(wl, b)
        RR.compare_sampling(f"{name} seq {b}", x[b], out[b], nacc[b], ref, tally)
    assert tally.near_ties <= max(0, int(1e-4 * tally.decisions)), tally.notes


def test_spec_sample_with_oracle_drafts(case):
    """s3r_spec_sample fed the oracle's own draft tokens."""
    name, (wl, st) = case
    ws = wl.spec
    refs = [RR.oracle_sampling_seq(wl, b) for b in range(ws.num_seqs)]
    xo = torch.from_numpy(np.stack([r["x"] for r in refs]).astype(np.int32)).cuda()
    st.draft_tokens.copy_(xo)
    st.sample()
    torch.cuda.synchronize()
    out = st.out_tokens.cpu().numpy()
    nacc = st.num_accepted.cpu().numpy()
    tally = RR.Tally()
    for b, r in enumerate(refs):
        # the draws are the oracle's, so only accept decisions and the draw count
        r2 = dict(r, x_margin=np.full_like(r["x_margin"], 1.0))
        RR.compare_sampling(f"{name} seq {b}", r["x"], out[b], nacc[b], r2, tally)
    assert tally.near_ties <= max(0, int(1e-4 * tally.decisions)), tally.notes


def test_tail_only_summaries_touch_only_tail_pages(case):
    name, (wl, st) = case
    st.kmin.zero_()
    st.kmax.zero_()
    st.summaries(tail_only=True)
    torch.cuda.synchronize()
    kmin = st.kmin.float().cpu().numpy().astype(np.float64)
    tails = set()
    for b in range(wl.spec.num_seqs):
        n = int(wl.pages_per_seq[b])
        tails.add(int(wl.block_table[b, n - 1]))
        ref = RR.oracle_attention_seq(wl, b, draft_steps=[])
        assert np.array_equal(kmin[ref["phys"][n - 1]], ref["kmin"][n - 1])
    others = [p for p in range(wl.num_pages_total) if p not in tails]
    assert np.all(kmin[others] == 0.0)
    st.summaries(tail_only=False)
    torch.cuda.synchronize()


def test_q_equals_p_accepts_every_draft_on_gpu():
    """Identical draft and target logits: every draft is accepted, the bonus
    token is drawn from p_gamma (the degenerate case of the accept rule)."""
    ws = custom_spec(1, num_seqs=6, gamma=5, vocab=4096)
    wl = Workload(ws, seed=5)
    t, _ = wl.logits()
    tl = torch.from_numpy(t.view(np.int16)).view(torch.bfloat16).cuda()
    dl = tl[:, :ws.gamma].contiguous()
    S, g, V = ws.num_seqs, ws.gamma, ws.vocab
    x = torch.empty((S, g), dtype=torch.int32, device="cuda")
    wt = torch.zeros(s3r.s3r_sample_workspace_bytes(S * g, 0, V), dtype=torch.uint8, device="cuda")
    s3r.s3r_sample_tokens(dl, "bf16", S * g, V, 1.0, torch.from_numpy(wl.u_draft).cuda(), x, wt)
    out = torch.empty((S, g + 1), dtype=torch.int32, device="cuda")
    n = torch.empty((S,), dtype=torch.int32, device="cuda")
    w = torch.zeros(s3r.s3r_sample_workspace_bytes(S, g, V), dtype=torch.uint8, device="cuda")
    s3r.s3r_spec_sample(tl, dl, "bf16", x, torch.from_numpy(wl.u_accept).cuda(), torch.from_numpy(wl.u_sample).cuda(),
                        S, g, V, 1.0, out, n, w)
    torch.cuda.synchronize()
    assert torch.all(n == g)
    assert torch.equal(out[:, :g], x)
    assert int(out[:, g].min()) >= 0


def test_device_checks_flag_bad_inputs_without_faulting():
    """A bad context length and a bad page id are recorded in the status word;
    the kernels skip them and the context stays usable."""
    ws = custom_spec(1, num_seqs=3, num_q_heads=8, num_kv_heads=2, budget_pages=2, vocab=512)
    wl = Workload(ws, seed=2, context_lens=[300, 200, 130])
    st = DecodeStep(wl)
    st.summaries()
    torch.cuda.synchronize()
    # sequence 1: length 0 (unusable); sequence 2: a block-table entry out of range
    st.context_lens[1] = 0
    st.block_table[2, 1] = wl.num_pages_total + 5
    st.verify()
    status, bits = s3r.s3r_device_status(st.ws_verify)
    assert status == s3r.S3R_ERR_DEVICE_CHECK
    assert bits & s3r.S3R_DEV_BAD_CONTEXT_LEN and bits & s3r.S3R_DEV_BAD_PAGE_ID
    out = st.verify_out.float().cpu().numpy()
    lse = st.verify_lse.cpu().numpy()
    assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(out[0])) and np.all(np.isfinite(out[2]))
    # sequence 0 is untouched by the bad entries of the others
    ref = RR.oracle_attention_seq(wl, 0, draft_steps=[])
    RR.assert_close("seq 0 verify", out[0], ref["verify_out"], "bf16")
    # the next call on the same workspace starts clean
    st.context_lens[1] = 200
    st.block_table[2, 1] = int(wl.block_table[2, 1])
    st.verify()
    assert s3r.s3r_device_status(st.ws_verify) == (s3r.S3R_OK, 0)


def test_status_word_is_sticky_until_read():
    """A device-check bit survives later clean calls on the same workspace and
    is cleared by reading it (no call clears the workspace itself)."""
    ws = custom_spec(1, num_seqs=2, num_q_heads=8, num_kv_heads=2, budget_pages=2, vocab=512)
    wl = Workload(ws, seed=3, context_lens=[300, 200])
    st = DecodeStep(wl)
    st.summaries()
    torch.cuda.synchronize()
    st.context_lens[1] = 0
    st.verify()
    st.context_lens[1] = 200
    st.verify()
    status, bits = s3r.s3r_device_status(st.ws_verify)
    assert status == s3r.S3R_ERR_DEVICE_CHECK and bits & s3r.S3R_DEV_BAD_CONTEXT_LEN
    assert s3r.s3r_device_status(st.ws_verify) == (s3r.S3R_OK, 0)
    # the clean call's results are right
    ref = RR.oracle_attention_seq(wl, 1, draft_steps=[])
    RR.assert_close("seq 1 verify", st.verify_out[1].float().cpu().numpy(), ref["verify_out"], "bf16")


def test_draft_summarises_the_tail_page_itself():
    """The sparse draft call takes the tail page's summary from K, not from
    kmin/kmax: with the stored tail summaries wiped, the selection and the
    draft outputs still match the oracle (whose summaries come from K)."""
    s, lens = CASES["bf16-d128-p64"]
    wl = Workload(s, seed=1, context_lens=lens)
    st = DecodeStep(wl)
    st.summaries(tail_only=False)
    torch.cuda.synchronize()
    tails = [int(wl.block_table[b, int(wl.pages_per_seq[b]) - 1]) for b in range(wl.spec.num_seqs)]
    st.kmin[tails] = -100.0                     # stale values that would make every tail page win
    st.kmax[tails] = 100.0
    for i in range(wl.spec.gamma):
        st.draft(i)
    torch.cuda.synchronize()
    sel = st.selected.cpu().numpy()
    tally = RR.Tally()
    for b in range(wl.spec.num_seqs):
        ref = RR.oracle_attention_seq(wl, b)
        for i, d in ref["draft"].items():
            ok = RR.compare_selection(f"seq {b} draft {i}", sel[i, b], d["selected"], d["gaps"], tally,
                                      scores=d["scores"])
            if all(ok):
                RR.assert_close(f"seq {b} draft {i} out", st.draft_out[i, b].float().cpu().numpy(), d["out"], "bf16")
    assert tally.near_ties <= max(0, int(1e-4 * tally.decisions)), tally.notes
