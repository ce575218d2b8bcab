"""KV-cache upkeep of a round on the GPU (s3r_kv_append, s3r_kv_rollback)
against the float64 oracle: random draft appends, verification overwrites
and rollbacks across page boundaries (cache rows, lengths and page
summaries bit-exact), every acceptance count from 0 to gamma, bad inputs
flagged without faulting, and whole rounds with the cache upkept (draft
steps appending, verification overwriting, sampling, rollback). Every GPU
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


def _dev(x, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _host64(t, dtype):
    a = t.cpu()
    if dtype == "bf16":
        return to_float64(a.view(torch.int16).numpy().view(np.uint16), "bf16")
    return a.numpy().astype(np.float64)


def _store(x, dtype, rng_shape=None):
    return round_to_bf16_bits(x.astype(np.float32)) if dtype == "bf16" else x.astype(np.float32)


class Cache:
    """A small paged cache on the GPU and its float64 twin for the oracle."""

    def __init__(self, rng, dtype, S, H, P, D, lens, cap):
        total = S * cap + 5
        perm = rng.permutation(total)
        self.bt = perm[:S * cap].reshape(S, cap).astype(np.int32)
        self.dtype, self.P = dtype, P
        k = _store(rng.standard_normal((total, H, P, D)), dtype)
        v = _store(rng.standard_normal((total, H, P, D)), dtype)
        self.K = to_float64(k, dtype) if dtype == "bf16" else k.astype(np.float64)
        self.V = to_float64(v, dtype) if dtype == "bf16" else v.astype(np.float64)
        self.lens = np.asarray(lens, dtype=np.int64)
        self.kmin, self.kmax = O.page_summaries(self.K, self.bt, self.lens, P)
        self.k_dev, self.v_dev = _dev(k, dtype), _dev(v, dtype)
        self.bt_dev = torch.from_numpy(self.bt).cuda()
        self.lens_dev = torch.from_numpy(self.lens.astype(np.int32)).cuda()
        self.kv = s3r.paged_kv(self.k_dev, self.v_dev, self.bt_dev, self.lens_dev, H)
        self.kmin_dev = torch.zeros((total, H, D), dtype=self.k_dev.dtype, device="cuda")
        self.kmax_dev = torch.zeros_like(self.kmin_dev)
        s3r.s3r_page_summaries(self.kv, 0, self.kmin_dev, self.kmax_dev)
        self.ws = torch.zeros(s3r.s3r_kv_workspace_bytes(S), dtype=torch.uint8, device="cuda")

    def append(self, rng, n, overwrite):
        S, H, D = self.bt.shape[0], self.K.shape[1], self.K.shape[3]
        kn = _store(rng.standard_normal((S, n, H, D)), self.dtype)
        vn = _store(rng.standard_normal((S, n, H, D)), self.dtype)
        s3r.s3r_kv_append(self.kv, self.lens_dev, _dev(kn, self.dtype), _dev(vn, self.dtype), n, overwrite,
                          self.kmin_dev, self.kmax_dev, self.ws)
        k64 = to_float64(kn, self.dtype) if self.dtype == "bf16" else kn.astype(np.float64)
        v64 = to_float64(vn, self.dtype) if self.dtype == "bf16" else vn.astype(np.float64)
        self.K, self.V, self.lens, self.kmin, self.kmax = O.kv_append(
            self.K, self.V, self.bt, self.lens, k64, v64, overwrite, self.P, self.kmin, self.kmax)

    def rollback(self, n_acc, rows):
        s3r.s3r_kv_rollback(self.kv, self.lens_dev, torch.from_numpy(np.asarray(n_acc, np.int32)).cuda(), rows,
                            self.kmin_dev, self.kmax_dev, self.ws)
        self.lens, self.kmin, self.kmax = O.kv_rollback(self.K, self.bt, self.lens, n_acc, rows, self.P,
                                                        self.kmin, self.kmax)

    def check(self, tag):
        torch.cuda.synchronize()
        assert s3r.s3r_device_status(self.ws) == (s3r.S3R_OK, 0), tag
        lens = self.lens_dev.cpu().numpy()
        assert lens.tolist() == self.lens.tolist(), (tag, lens, self.lens)
        K, V = _host64(self.k_dev, self.dtype), _host64(self.v_dev, self.dtype)
        mn, mx = _host64(self.kmin_dev, self.dtype), _host64(self.kmax_dev, self.dtype)
        P = self.P
        for b, L in enumerate(self.lens):
            for t in range(int(L)):
                ph = self.bt[b, t // P]
                assert np.array_equal(K[ph, :, t % P], self.K[ph, :, t % P]), (tag, b, t)
                assert np.array_equal(V[ph, :, t % P], self.V[ph, :, t % P]), (tag, b, t)
            for i in range(-(-int(L) // P)):
                ph = self.bt[b, i]
                assert np.array_equal(mn[ph], self.kmin[ph]) and np.array_equal(mx[ph], self.kmax[ph]), (tag, b, i)


@pytest.mark.parametrize("dtype,P,D,seed", [("bf16", 64, 128, 0), ("bf16", 16, 64, 1), ("f32", 16, 128, 2),
                                            ("bf16", 16, 128, 3)])
def test_rounds_of_appends_overwrites_rollbacks_match_oracle(dtype, P, D, seed):
    rng = np.random.default_rng(seed)
    S, H, cap = 4, 2, 24
    c = Cache(rng, dtype, S, H, P, D, rng.integers(1, 6 * P, size=S), cap)
    c.check("initial")
    for rnd in range(4):
        gamma = int(rng.integers(1, 9))
        for i in range(gamma):
            c.append(rng, 1, 0)
            c.check(f"round {rnd} draft {i}")
        c.append(rng, gamma + 1, gamma)
        c.check(f"round {rnd} verify")
        n_acc = rng.integers(0, gamma + 1, size=S)
        c.rollback(n_acc, gamma + 1)
        c.check(f"round {rnd} rollback {n_acc.tolist()}")


def test_rollback_for_every_acceptance_count():
    """One sequence per n_acc in 0..gamma, rounds ending on both sides of a
    page boundary."""
    rng = np.random.default_rng(7)
    gamma, P, H, D = 6, 16, 2, 128
    S = 2 * (gamma + 1)
    base = [16 * 3 - 2] * (gamma + 1) + [16 * 5 + 3] * (gamma + 1)
    c = Cache(rng, "bf16", S, H, P, D, base, 10)
    for i in range(gamma):
        c.append(rng, 1, 0)
    c.append(rng, gamma + 1, gamma)
    c.check("before rollback")
    n_acc = np.array(list(range(gamma + 1)) * 2)
    c.rollback(n_acc, gamma + 1)
    c.check("after rollback")
    assert c.lens.tolist() == [b + 1 + int(a) for b, a in zip(base, n_acc)]


def test_bad_lengths_are_flagged_and_left_unchanged():
    rng = np.random.default_rng(11)
    c = Cache(rng, "bf16", 3, 2, 16, 128, [40, 5, 70], 8)
    # overwrite more rows than sequence 1 holds: it is skipped, the others are written
    kn = torch.zeros((3, 7, 2, 128), dtype=torch.bfloat16, device="cuda")
    s3r.s3r_kv_append(c.kv, c.lens_dev, kn, kn, 7, 6, c.kmin_dev, c.kmax_dev, c.ws)
    torch.cuda.synchronize()
    st, bits = s3r.s3r_device_status(c.ws)
    assert st == s3r.S3R_ERR_DEVICE_CHECK and bits & s3r.S3R_DEV_BAD_CONTEXT_LEN
    assert c.lens_dev.cpu().tolist() == [41, 5, 71]
    # an acceptance count out of range leaves that sequence unchanged
    s3r.s3r_kv_rollback(c.kv, c.lens_dev, torch.tensor([0, 0, 9], dtype=torch.int32, device="cuda"), 7,
                        c.kmin_dev, c.kmax_dev, c.ws)
    torch.cuda.synchronize()
    st, bits = s3r.s3r_device_status(c.ws)
    assert st == s3r.S3R_ERR_DEVICE_CHECK and bits & s3r.S3R_DEV_BAD_CONTEXT_LEN
    assert c.lens_dev.cpu().tolist() == [35, 5, 71]
    # the workspace is clean again for good inputs
    s3r.s3r_kv_rollback(c.kv, c.lens_dev, torch.tensor([0, 0, 0], dtype=torch.int32, device="cuda"), 1,
                        c.kmin_dev, c.kmax_dev, c.ws)
    torch.cuda.synchronize()
    assert s3r.s3r_device_status(c.ws) == (s3r.S3R_OK, 0)


KV_ROUNDS = {
    "bf16-d128-p64": (custom_spec(1, num_seqs=3, num_q_heads=8, num_kv_heads=2, budget_pages=3, vocab=1000),
                      [700, 64 * 7 + 2, 1200]),
    "bf16-d64-p16-g8": (custom_spec(1, num_seqs=3, num_q_heads=16, num_kv_heads=2, head_dim=64, page_size=16,
                                    gamma=7, budget_pages=5, vocab=777), [300, 16 * 9 + 8, 130]),
    "f32-tiny": (custom_spec(0, num_seqs=2, budget_pages=3), [200, 257]),
}


@pytest.mark.parametrize("name", list(KV_ROUNDS))
def test_round_with_kv_upkeep_matches_oracle(name):
    s, lens = KV_ROUNDS[name]
    wl = Workload(s, seed=6, context_lens=lens)
    st = DecodeStep(wl)
    st.context_lens.copy_(st.lens_committed)
    st.summaries()                                  # summaries of the committed cache
    st.round_with_kv()
    torch.cuda.synchronize()
    for k, (status, bits) in st.device_checks().items():
        assert status == s3r.S3R_OK, (name, k, bits)
    dt = s.kv_dtype
    tally = RR.Tally()
    sel = st.selected.cpu().numpy()
    x = st.draft_tokens.cpu().numpy()
    out = st.out_tokens.cpu().numpy()
    nacc = st.num_accepted.cpu().numpy()
    lens_after = st.context_lens.cpu().numpy()
    K, V = _host64(st.k_cache, dt), _host64(st.v_cache, dt)
    mn, mx = _host64(st.kmin, dt), _host64(st.kmax, dt)
    for b in range(s.num_seqs):
        ref = RR.oracle_kv_round_seq(wl, b)
        for i, d in ref["draft"].items():
            ok = RR.compare_selection(f"{name} seq {b} draft {i}", sel[i, b], d["selected"], d["gaps"], tally,
                                      scores=d["scores"])
            if all(ok):
                RR.assert_close(f"{name} seq {b} draft {i}", st.draft_out[i, b].float().cpu().numpy(), d["out"], dt)
        RR.assert_close(f"{name} seq {b} verify", st.verify_out[b].float().cpu().numpy(), ref["verify_out"], dt)
        RR.compare_sampling(f"{name} seq {b}", x[b], out[b], nacc[b], ref["sampling"], tally)
        if int(nacc[b]) == ref["sampling"]["n_acc"]:
            assert int(lens_after[b]) == ref["len_after"], (name, b)
        # the round's rows in the cache (the verifier's), and the summaries of
        # every page the sequence now uses
        phys, P = ref["phys"], s.page_size
        for t in range(ref["start"], ref["start"] + s.rows):
            lp = t // P
            assert np.array_equal(K[phys[lp], :, t % P], ref["K"][lp, :, t % P]), (name, b, t)
            assert np.array_equal(V[phys[lp], :, t % P], ref["V"][lp, :, t % P]), (name, b, t)
        for lp in range(-(-int(lens_after[b]) // P)):
            assert np.array_equal(mn[phys[lp]], ref["kmin"][lp]) and np.array_equal(mx[phys[lp]], ref["kmax"][lp]), \
                (name, b, lp)
    assert tally.near_ties <= max(0, int(1e-4 * tally.decisions)), tally.notes
