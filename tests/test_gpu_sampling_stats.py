"""The draft rows' statistics handed from the drafter's draw to speculative
sampling (s3r_sample_tokens_ex -> s3r_spec_sample_ex): the statistics equal
the float64 definition, and sampling with them commits the oracle's tokens,
as sampling without them does. Every GPU result comes from the C ABI."""
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
    "bf16-v151936": (custom_spec(1, num_seqs=6, num_q_heads=8, num_kv_heads=2, budget_pages=2), [300, 200, 130, 700, 64, 90]),
    "f32-t0.7-ragged-vocab": (custom_spec(4, num_seqs=5, num_q_heads=8, num_kv_heads=2, budget_pages=2, gamma=5,
                                          vocab=10007), [300, 200, 130, 700, 64]),
    "tiny-fp32": (spec(0), None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_draw_writes_exact_row_statistics(name):
    s, lens = CASES[name]
    wl = Workload(s, seed=3, context_lens=lens)
    st = DecodeStep(wl)
    st.draw_draft_tokens()
    torch.cuda.synchronize()
    stats = st.draft_stats.cpu().numpy()
    T = RR.f32(s.temperature)
    for b in range(s.num_seqs):
        _, d = wl.logits_for_seq(b)
        dl = to_float64(d, s.logit_dtype)
        for i in range(s.gamma):
            M = dl[i].max()
            Z = np.exp((dl[i] - M) / T).sum()
            assert stats[b, i, 0] == M, (name, b, i)
            assert abs(stats[b, i, 1] - Z) <= 1e-12 * Z, (name, b, i, stats[b, i, 1], Z)


@pytest.mark.parametrize("name", list(CASES))
def test_spec_sample_with_draft_statistics_matches_oracle(name):
    s, lens = CASES[name]
    wl = Workload(s, seed=5, context_lens=lens)
    st = DecodeStep(wl)
    st.draw_draft_tokens()
    results = {}
    for use in (True, False):
        st.sample(use_draft_stats=use)
        torch.cuda.synchronize()
        assert s3r.s3r_device_status(st.ws_sample) == (s3r.S3R_OK, 0)
        results[use] = (st.out_tokens.cpu().numpy().copy(), st.num_accepted.cpu().numpy().copy())
    x = st.draft_tokens.cpu().numpy()
    tally = RR.Tally()
    for use in (True, False):
        out, nacc = results[use]
        for b in range(s.num_seqs):
            RR.compare_sampling(f"{name} stats={use} seq {b}", x[b], out[b], nacc[b], RR.oracle_sampling_seq(wl, b),
                                tally)
    assert tally.near_ties <= max(0, int(1e-4 * tally.decisions)), tally.notes
