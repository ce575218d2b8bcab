"""A decode round captured into one CUDA graph (γ drafts, verify, sampling;
the kernels chained by programmatic dependent launch inside it) must give
exactly the eager round's outputs on every replay (the kernels are
deterministic, with fixed merge orders, and the workspaces reset
themselves), and those outputs match the float64 oracle, the benchmark's
full-size 16 x 16K round included."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from self_sparse_speculative_b200.step import DecodeStep                        # noqa: E402
from self_sparse_speculative_b200.workloads import Workload, custom_spec, spec  # noqa: E402

import oracle.reference_run as RR                                               # noqa: E402

OUTPUTS = ("selected", "draft_out", "draft_lse", "verify_out", "verify_lse", "draft_tokens", "out_tokens",
           "num_accepted")


def _snapshot(st):
    return {k: getattr(st, k).detach().clone() for k in OUTPUTS}


@pytest.mark.parametrize("base,over", [(1, dict(num_seqs=3, context=4096 + 64 * 5 + 17, vocab=5000)),
                                       (3, dict(num_seqs=2, context=8192 + 33, vocab=4000)),
                                       (4, dict(num_seqs=5, context=1024 + 7, vocab=3001))])
def test_captured_round_matches_eager(base, over):
    wl = Workload(custom_spec(base, **over), seed=5)
    st = DecodeStep(wl)
    st.summaries()
    st.round()
    torch.cuda.synchronize()
    ref = _snapshot(st)
    for k in OUTPUTS:
        getattr(st, k).fill_(-7)
    graph = st.capture_round()
    for _ in range(3):
        graph.replay()
        torch.cuda.synchronize()
        for k in OUTPUTS:
            assert torch.equal(getattr(st, k), ref[k]), k
        for k in OUTPUTS:
            getattr(st, k).fill_(-7)
    assert all(v == (0, 0) for v in st.device_checks().values())
    del graph


def _check_against_oracle(name, wl, st, seqs, attention=True):
    """The replayed round's outputs against the float64 oracle: selections,
    draft and verify attention of the listed sequences, and every sequence's
    draws, accept decisions and drawn token."""
    ws = wl.spec
    dt = ws.kv_dtype
    tally = RR.Tally()
    if attention:
        sel = st.selected.cpu().numpy()
        for b in seqs:
            ref = RR.oracle_attention_seq(wl, b)
            for i, d in ref["draft"].items():
                ok = RR.compare_selection(f"{name} seq {b} draft {i}", sel[i, b], d["selected"], d["gaps"], tally,
                                          scores=d["scores"])
                if all(ok):
                    RR.assert_close(f"{name} seq {b} draft {i}", st.draft_out[i, b].float().cpu().numpy(), d["out"], dt)
            RR.assert_close(f"{name} seq {b} verify", st.verify_out[b].float().cpu().numpy(), ref["verify_out"], dt)
    x = st.draft_tokens.cpu().numpy()
    out = st.out_tokens.cpu().numpy()
    nacc = st.num_accepted.cpu().numpy()
    for b in range(ws.num_seqs):
        RR.compare_sampling(f"{name} seq {b}", x[b], out[b], nacc[b], RR.oracle_sampling_seq(wl, b), tally)
    assert tally.near_ties <= max(0, int(1e-4 * tally.decisions)), tally.notes


@pytest.mark.parametrize("base,over", [(1, dict(num_seqs=3, context=4096 + 64 * 5 + 17, vocab=5000)),
                                       (4, dict(num_seqs=5, context=1024 + 7, vocab=3001))])
def test_replayed_round_matches_oracle(base, over):
    wl = Workload(custom_spec(base, **over), seed=8)
    st = DecodeStep(wl)
    st.summaries()
    graph = st.capture_round()
    for _ in range(2):
        for k in OUTPUTS:
            getattr(st, k).fill_(-7)
        graph.replay()
        torch.cuda.synchronize()
        _check_against_oracle(f"{wl.spec.name.split(':')[0]}", wl, st, range(wl.spec.num_seqs))
    assert all(v == (0, 0) for v in st.device_checks().values())
    del graph


def test_replayed_round_full_size_matches_oracle():
    """The benchmark's own headline: the 16 x 16K Qwen3-8B-shaped round,
    replayed from its graph, against the oracle (attention on two sampled
    sequences, sampling on all sixteen)."""
    wl = Workload(spec(1), seed=0)
    st = DecodeStep(wl)
    st.summaries()
    graph = st.capture_round()
    for k in OUTPUTS:
        getattr(st, k).fill_(-7)
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    _check_against_oracle("qwen3-8b-layer replay", wl, st, [0, 15])
    assert all(v == (0, 0) for v in st.device_checks().values())
    del graph
    del st
    torch.cuda.empty_cache()
