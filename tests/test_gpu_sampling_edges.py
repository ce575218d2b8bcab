"""Sampling on logits the synthetic workloads never produce.

The drawn token is the smallest k with C(k) > u * C(V-1) over the weights
exp((x - max)/T) (inverse CDF, the speculative-sampling rule restated on the
ai.info SpecRoll page). These rows spread their logits over more than 707 T,
so some float64 exponentials fall into the range the sampler's table-driven
exponential hands to its fix-up (subnormal weights, and weights that are
exactly 0); other rows are -inf except for a few tokens. Draws must equal the
float64 oracle's except where the oracle's own margin is below 1e-10 (a near
tie); with u = 0 the draw is the first token of positive weight, which the
GPU must find exactly (a subnormal weight still counts).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from oracle import s3r_oracle as O                                             # noqa: E402
from self_sparse_speculative_b200 import s3r                                   # noqa: E402
from self_sparse_speculative_b200.workloads import to_float64, to_storage      # noqa: E402

V = 4096 + 40          # two 2048-element pass-2 chunks and a ragged tail of whole vectors
DRAW_TIE = 1e-10
ACCEPT_TIE = 1e-6


def _edge_rows(rng):
    rows = []
    r = rng.normal(0.0, 1.0, V).astype(np.float32)
    r[:16] = -720.0                      # exp(-724) is subnormal at T = 1, 0 at T = 0.7
    r[100:200] = -800.0                  # 0 in float64
    rows.append(r)
    r = np.full(V, -np.inf, np.float32)  # three tokens only
    r[[5, V // 2, V - 1]] = [0.5, 1.0, -2.0]
    rows.append(r)
    rows.append((rng.normal(0.0, 1.0, V) * 300.0).astype(np.float32))   # spread of +-1000 (row WIDE)
    r = np.full(V, -np.inf, np.float32)  # one token only
    r[V - 3] = 7.0
    rows.append(r)
    r = rng.normal(0.0, 2.0, V).astype(np.float32)
    r[::7] = -760.0                      # zeros scattered through every vector
    rows.append(r)
    return np.stack(rows)


WIDE = 2   # its smallest positive weights sit at the float64 underflow edge, where either
           # side may round to 0: compared by margin only


def _dev(arr, dtype):
    st = to_storage(arr, dtype)
    t = torch.from_numpy(np.ascontiguousarray(st).view(np.int16 if dtype == "bf16" else np.float32))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.cuda()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("temperature", [1.0, 0.7])
def test_draws_on_wide_and_sparse_logits(dtype, temperature):
    rng = np.random.default_rng(7)
    base = _edge_rows(rng)
    us = np.array([0.0, 0.5, 0.999999, 0.123457], dtype=np.float32)
    logits = np.repeat(base, len(us), axis=0)                     # every row with every u
    u = np.tile(us, len(base)).astype(np.float32)
    n = logits.shape[0]
    x64 = to_float64(to_storage(logits, dtype), dtype)
    k_ref, margin = O.sample_rows(x64, u.astype(np.float64), temperature)
    p = O.softmax_t(x64, temperature)

    ws = torch.zeros(s3r.s3r_sample_workspace_bytes(n, 0, V), dtype=torch.uint8, device="cuda")
    toks = torch.empty(n, dtype=torch.int32, device="cuda")
    s3r.s3r_sample_tokens(_dev(logits, dtype), dtype, n, V, temperature, torch.from_numpy(u).cuda(), toks, ws)
    torch.cuda.synchronize()
    k = toks.cpu().numpy()
    assert s3r.s3r_device_status(ws) == (0, 0)
    for i in range(n):
        row = i // len(us)
        if u[i] == 0.0:
            if row == WIDE:
                continue
            first = int(np.nonzero(p[i] > 0)[0][0])
            assert k[i] == first, f"row {i} (u = 0): {k[i]} != first positive weight {first}"
        elif margin[i] >= DRAW_TIE:
            assert k[i] == k_ref[i], f"row {i} u {u[i]}: gpu {k[i]} oracle {k_ref[i]} (margin {margin[i]:.2e})"
        assert p[i, k[i]] > 0, f"row {i}: drew token {k[i]} of zero probability"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_spec_sample_on_wide_logits(dtype):
    """Residual and bonus draws where p and q span over 707 T; drafts drawn
    from q by the oracle, so every decision has a defined reference."""
    rng = np.random.default_rng(11)
    temperature = 1.0
    gamma, S = 3, 4
    R = gamma + 1
    tgt = np.stack([_edge_rows(rng)[[0, 2, 4, 0]] for _ in range(S)])             # [S, R, V]
    drf = tgt[:, :gamma] + rng.normal(0.0, 0.5, (S, gamma, V)).astype(np.float32)
    drf[1] = tgt[1, :gamma]                                                     # q = p: every draft accepted
    t64 = to_float64(to_storage(tgt, dtype), dtype)
    d64 = to_float64(to_storage(drf, dtype), dtype)
    ud = rng.random((S, gamma))
    x, _ = O.sample_rows(d64.reshape(S * gamma, V), ud.reshape(-1), temperature)
    x = x.reshape(S, gamma).astype(np.int32)
    ua = rng.random((S, gamma)).astype(np.float32)
    us = rng.random((S, R)).astype(np.float32)
    out_ref, nacc_ref, amargin, smargin = O.spec_sample(t64, d64, x, ua, us, temperature)

    ws = torch.zeros(s3r.s3r_sample_workspace_bytes(S, gamma, V), dtype=torch.uint8, device="cuda")
    out = torch.empty((S, R), dtype=torch.int32, device="cuda")
    nacc = torch.empty(S, dtype=torch.int32, device="cuda")
    s3r.s3r_spec_sample(_dev(tgt, dtype), _dev(drf, dtype), dtype, torch.from_numpy(x).cuda(),
                        torch.from_numpy(ua).cuda(), torch.from_numpy(us).cuda(), S, gamma, V, temperature,
                        out, nacc, ws)
    torch.cuda.synchronize()
    assert s3r.s3r_device_status(ws) == (0, 0)
    out, nacc = out.cpu().numpy(), nacc.cpu().numpy()
    assert nacc[1] == gamma, "q = p must accept every draft"
    for b in range(S):
        tested = amargin[b][~np.isnan(amargin[b])]
        if np.any(tested < ACCEPT_TIE):
            continue                                        # a near-tie decision: either outcome is valid
        assert nacc[b] == nacc_ref[b], f"seq {b}: accepted {nacc[b]} != {nacc_ref[b]}"
        assert np.array_equal(out[b, :nacc[b]], x[b, :nacc[b]])
        assert np.all(out[b, nacc[b] + 1:] == -1)
        if smargin[b] >= DRAW_TIE:
            assert out[b, nacc[b]] == out_ref[b, nacc_ref[b]], f"seq {b}: drew {out[b, nacc[b]]}"
