"""A decode round captured into one CUDA graph (γ drafts, verify, sampling;
the kernels chained by programmatic dependent launch inside it) must give
exactly the eager round's outputs on every replay: the kernels are
deterministic (fixed merge orders) and the workspaces reset themselves."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from self_sparse_speculative_b200.step import DecodeStep                        # noqa: E402
from self_sparse_speculative_b200.workloads import Workload, custom_spec        # noqa: E402

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
