"""s3r_spec_sample_noalloc: speculative sampling for callers that cannot
allocate device memory.

Code that runs inside a host framework whose device memory belongs to the
framework's own pooling allocator, or that must not allocate while a stream
is being captured, cannot hand the library a workspace. The no-alloc entry
point takes the same inputs and outputs as s3r_spec_sample but keeps its
scratch in a fixed 4 MiB device array owned by the library. These tests call
both entry points through the C ABI on the same inputs and require identical
committed tokens, on two no-alloc calls in a row (the array keeps the previous
call's contents, so the second call checks that everything that must start
from zero is cleared).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from self_sparse_speculative_b200 import s3r                                    # noqa: E402
from self_sparse_speculative_b200.step import _to_torch                         # noqa: E402
from self_sparse_speculative_b200.workloads import Workload, custom_spec, spec  # noqa: E402

CASES = {
    "small-bf16": custom_spec(1, num_seqs=5, vocab=3000),
    "small-f32-odd-vocab": custom_spec(4, num_seqs=3, gamma=5, vocab=999),
    "qwen3-8b-layer": spec(1),
}


def _inputs(ws, seed):
    wl = Workload(ws, seed=seed)
    t, d = wl.logits()
    dev = "cuda"
    tl = _to_torch(t, ws.logit_dtype, dev)
    dl = _to_torch(d, ws.logit_dtype, dev)
    S, g, V = ws.num_seqs, ws.gamma, ws.vocab
    x = torch.empty((S, g), dtype=torch.int32, device=dev)
    wtok = torch.zeros(s3r.s3r_sample_workspace_bytes(S * g, 0, V), dtype=torch.uint8, device=dev)
    s3r.s3r_sample_tokens(dl, ws.logit_dtype, S * g, V, ws.temperature,
                          torch.from_numpy(wl.u_draft).to(dev), x, wtok)
    ua = torch.from_numpy(wl.u_accept).to(dev)
    us = torch.from_numpy(wl.u_sample).to(dev)
    return tl, dl, x, ua, us


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry_point_on_two_calls(name):
    ws = CASES[name]
    S, g, V, T = ws.num_seqs, ws.gamma, ws.vocab, ws.temperature
    tl, dl, x, ua, us = _inputs(ws, seed=3)
    out_ref = torch.full((S, g + 1), -7, dtype=torch.int32, device="cuda")
    n_ref = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    work = torch.zeros(s3r.s3r_sample_workspace_bytes(S, g, V), dtype=torch.uint8, device="cuda")
    s3r.s3r_spec_sample(tl, dl, ws.logit_dtype, x, ua, us, S, g, V, T, out_ref, n_ref, work)
    for call in range(2):
        out = torch.full((S, g + 1), -7, dtype=torch.int32, device="cuda")
        n = torch.full((S,), -7, dtype=torch.int32, device="cuda")
        s3r.s3r_spec_sample_noalloc(tl, dl, ws.logit_dtype, x, ua, us, S, g, V, T, out, n)
        torch.cuda.synchronize()
        assert torch.equal(n, n_ref), (name, call)
        assert torch.equal(out, out_ref), (name, call)
    assert int(n_ref.min()) >= 0 and int(n_ref.max()) <= g


def test_noalloc_rejects_batches_beyond_its_array():
    # 2048 sequences x 33 rows of statistics need more than the 4 MiB array
    fake = 0x10000
    st = s3r.lib().s3r_spec_sample_noalloc(fake, fake, s3r.S3R_BF16, fake, fake, fake, 2048, 16, 151936,
                                           1.0, fake, fake, None)
    assert st == s3r.S3R_ERR_UNSUPPORTED
    assert s3r.s3r_sample_workspace_bytes(2048, 16, 151936) > (4 << 20)
