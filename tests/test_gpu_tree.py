"""Tree verification on the GPU (s3r_verify_attn_tree, s3r_tree_spec_sample)
against the float64 oracle: ancestor-masked attention over paged caches
(bf16 token-major tiles and the fp32 kernel, several splits, ragged pages,
the shortest history L = R, up to 64 nodes), the tree walk of exact
speculative sampling (random and breadth-first trees, repeated sibling
tokens, vectorised and scalar vocab layouts, full vocabulary size), the
chain tree against the ordinary calls, and bad trees or tokens flagged
without a fault. Every GPU result comes from the C ABI (libs3r.so)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from self_sparse_speculative_b200 import s3r                      # noqa: E402
from self_sparse_speculative_b200.workloads import round_to_bf16_bits, to_float64  # noqa: E402

import oracle as O                                                 # noqa: E402
import oracle.reference_run as RR                                  # noqa: E402

ACCEPT_TIE, DRAW_TIE = 1e-6, 1e-10


def _store(x, dtype):
    return round_to_bf16_bits(x.astype(np.float32)) if dtype == "bf16" else np.asarray(x, dtype=np.float32)


def _wide(x, dtype):
    return to_float64(x, dtype) if dtype == "bf16" else np.asarray(x, dtype=np.float64)


def _dev(x, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _i32(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()


def random_tree(rng, R):
    par = np.full(R, -1, dtype=np.int64)
    for c in range(1, R):
        par[c] = rng.integers(0, c)
    return par


# ------------------------------------------------------------------ attention

class Paged:
    def __init__(self, rng, dtype, S, Hq, H, P, D, lens):
        n_pages = [-(-L // P) for L in lens]
        cap = max(n_pages) + 1
        total = S * cap + 3
        perm = rng.permutation(total)
        self.bt = np.full((S, cap), -1, dtype=np.int32)
        off = 0
        for b, n in enumerate(n_pages):
            self.bt[b, :n] = perm[off:off + n]
            off += n
        k = _store(rng.standard_normal((total, H, P, D)), dtype)
        v = _store(rng.standard_normal((total, H, P, D)), dtype)
        self.K, self.V = _wide(k, dtype), _wide(v, dtype)
        self.lens = np.asarray(lens, dtype=np.int64)
        self.k_dev, self.v_dev = _dev(k, dtype), _dev(v, dtype)
        self.bt_dev, self.lens_dev = _i32(self.bt), _i32(self.lens)
        self.kv = s3r.paged_kv(self.k_dev, self.v_dev, self.bt_dev, self.lens_dev, Hq)
        self.dtype = dtype


ATTN_CASES = [
    # dtype, S, Hq, H, P, D, nodes, lens, branching (None: random tree)
    ("bf16", 3, 8, 2, 64, 128, 9, [130, 9, 2100], [3, 2, 1]),
    ("bf16", 2, 8, 2, 16, 64, 16, [700, 16 * 9 + 3], None),
    ("bf16", 2, 8, 1, 64, 128, 8, [77, 1500], [2]),                # G = 8: 64 packed rows
    ("bf16", 2, 2, 2, 64, 64, 64, [64, 3000], None),               # 64 nodes, G = 1
    ("f32", 2, 6, 2, 64, 128, 10, [200, 4 * 64 + 1], [4, 1]),
    ("f32", 2, 4, 2, 16, 64, 64, [64, 900], None),                 # G * R = 128 on the fp32 kernel
]


def _attn_case(case, seed):
    dtype, S, Hq, H, P, D, R, lens, br = case
    rng = np.random.default_rng(seed)
    c = Paged(rng, dtype, S, Hq, H, P, D, lens)
    par = np.stack([O.build_tree(R, br) if br else random_tree(rng, R) for _ in range(S)])
    q = _store(rng.standard_normal((S, R, Hq, D)), dtype)
    return c, par, q


@pytest.mark.parametrize("case", ATTN_CASES, ids=[f"{c[0]}-g{c[2] // c[3]}-r{c[6]}-p{c[4]}-d{c[5]}" for c in ATTN_CASES])
def test_tree_attention_matches_oracle(case):
    c, par, q = _attn_case(case, 11)
    S, R, Hq, D = q.shape
    scale = 1.0 / np.sqrt(D)
    out = torch.empty((S, R, Hq, D), dtype=c.k_dev.dtype, device="cuda")
    lse = torch.empty((S, R, Hq), dtype=torch.float32, device="cuda")
    ws = torch.zeros(s3r.s3r_attn_workspace_bytes(c.kv, R, 0), dtype=torch.uint8, device="cuda")
    s3r.s3r_verify_attn_tree(c.kv, _dev(q, c.dtype), R, _i32(par), scale, out, lse, ws)
    assert s3r.s3r_device_status(ws) == (s3r.S3R_OK, 0)
    ref_o, ref_l = O.tree_verify_attn(_wide(q, c.dtype), c.K, c.V, c.bt, c.lens, par, RR.f32(scale))
    RR.assert_close("tree out", out.float().cpu().numpy(), ref_o, c.dtype)
    RR.assert_close("tree lse", lse.cpu().numpy(), ref_l, c.dtype)


@pytest.mark.parametrize("case", [ATTN_CASES[0], ATTN_CASES[1], ATTN_CASES[4]], ids=["bf16-p64", "bf16-p16", "f32"])
def test_chain_tree_is_bitwise_the_causal_verify(case):
    c, _, q = _attn_case(case, 12)
    S, R, Hq, D = q.shape
    chain = np.broadcast_to(O.chain_parents(R), (S, R))
    ws = torch.zeros(s3r.s3r_attn_workspace_bytes(c.kv, R, 0), dtype=torch.uint8, device="cuda")
    qd = _dev(q, c.dtype)
    o1 = torch.empty((S, R, Hq, D), dtype=c.k_dev.dtype, device="cuda")
    o2 = torch.empty_like(o1)
    l1 = torch.empty((S, R, Hq), dtype=torch.float32, device="cuda")
    l2 = torch.empty_like(l1)
    s3r.s3r_verify_attn_tree(c.kv, qd, R, _i32(chain), 0.125, o1, l1, ws)
    s3r.s3r_verify_attn(c.kv, qd, R, 0.125, o2, l2, ws)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16) if c.dtype == "bf16" else o1, o2.view(torch.int16) if c.dtype == "bf16" else o2)
    assert torch.equal(l1, l2)


def test_bad_tree_is_flagged_and_unsupported_shapes_refused():
    c, par, q = _attn_case(ATTN_CASES[0], 13)
    S, R, Hq, D = q.shape
    bad = par.copy()
    bad[1, 5] = 7                                            # a parent after its child
    out = torch.empty((S, R, Hq, D), dtype=c.k_dev.dtype, device="cuda")
    ws = torch.zeros(s3r.s3r_attn_workspace_bytes(c.kv, R, 0), dtype=torch.uint8, device="cuda")
    s3r.s3r_verify_attn_tree(c.kv, _dev(q, c.dtype), R, _i32(bad), 0.1, out, None, ws)
    st, bits = s3r.s3r_device_status(ws)
    assert st == s3r.S3R_ERR_DEVICE_CHECK and bits & s3r.S3R_DEV_BAD_TREE
    # 65 nodes, or more than 64 packed bf16 rows, are refused before any launch
    with pytest.raises(s3r.S3RError, match="UNSUPPORTED"):
        s3r.s3r_verify_attn_tree(c.kv, _dev(q, c.dtype), 65, _i32(np.zeros((S, 65))), 0.1, out, None, ws)
    with pytest.raises(s3r.S3RError, match="UNSUPPORTED"):
        s3r.s3r_verify_attn_tree(c.kv, _dev(q, c.dtype), 9 * 2, _i32(np.zeros((S, 18))), 0.1, out, None, ws)


# ------------------------------------------------------------------ sampling

def _sample_inputs(rng, dtype, S, R, V, T, trees, noise=0.6, leaf_nan=True):
    """Target and draft logits for every node, and node tokens drawn from
    the parent's draft distribution (some siblings forced to repeat)."""
    t = _store(2.0 * rng.standard_normal((S, R, V)), dtype)
    t64 = _wide(t, dtype)
    d = _store(t64 + noise * rng.standard_normal((S, R, V)), dtype)
    d64 = _wide(d, dtype)
    tokens = np.zeros((S, R), dtype=np.int64)
    for b in range(S):
        for c in range(1, R):
            v = int(trees[b, c])
            k, _ = O.sample_rows(d64[b, v][None], np.array([rng.random()]), T)
            tokens[b, c] = int(k[0])
            sib = [s for s in range(1, c) if trees[b, s] == v]
            if sib and rng.random() < 0.3:
                tokens[b, c] = tokens[b, sib[-1]]
    if leaf_nan:
        # the draft rows of leaves are never read: poison them on the device copy
        for b in range(S):
            leaves = [v for v in range(R) if not np.any(trees[b] == v)]
            for v in leaves:
                d[b, v] = _store(np.full(V, np.nan), dtype)
    return t, d, t64, d64, tokens


def _run_tree_gpu(dtype, t, d, tokens, par, ua, us, T):
    S, R, V = t.shape
    out = torch.empty((S, R), dtype=torch.int32, device="cuda")
    nacc = torch.empty(S, dtype=torch.int32, device="cuda")
    path = torch.empty((S, R), dtype=torch.int32, device="cuda")
    ws = torch.zeros(s3r.s3r_tree_sample_workspace_bytes(S, R, V), dtype=torch.uint8, device="cuda")
    s3r.s3r_tree_spec_sample(_dev(t, dtype), _dev(d, dtype), dtype, _i32(tokens), _i32(par),
                             torch.from_numpy(ua.astype(np.float32)).cuda(), torch.from_numpy(us.astype(np.float32)).cuda(),
                             S, R, V, T, out, nacc, path, ws)
    status = s3r.s3r_device_status(ws)
    return out.cpu().numpy(), nacc.cpu().numpy(), path.cpu().numpy(), status


def _check_walk(name, out, nacc, path, par, tokens, V, ref, tally):
    r_out, r_n, r_path, r_am, r_dm = ref
    S, R = out.shape
    for b in range(S):
        n = int(nacc[b])
        # always: a valid walk down the tree
        assert 0 <= n < R, (name, b, n)
        prev = 0
        for i in range(n):
            c = int(path[b, i])
            assert par[b, c] == prev and out[b, i] == tokens[b, c], (name, b, path[b].tolist())
            prev = c
        assert 0 <= out[b, n] < V and np.all(out[b, n + 1:] == -1) and np.all(path[b, n:] == -1), (name, b)
        tally.decisions += len(r_am[b]) + 1
        if (r_am[b] and min(r_am[b]) < ACCEPT_TIE) or r_dm[b] < DRAW_TIE:
            tally.near_ties += 1
            tally.notes.append(f"{name} seq {b}: near tie, walk validity checked only")
            continue
        assert n == r_n[b], (name, b, n, int(r_n[b]))
        assert np.array_equal(path[b], r_path[b]), (name, b, path[b].tolist(), r_path[b].tolist())
        assert np.array_equal(out[b], r_out[b]), (name, b, out[b].tolist(), r_out[b].tolist())


SAMPLE_CASES = [
    # dtype, S, R, V, T, tree kind
    ("bf16", 8, 10, 1024, 1.0, "bfs"),          # vectorised rows
    ("bf16", 8, 13, 1001, 0.7, "random"),       # odd vocab: scalar path
    ("f32", 6, 16, 2048, 1.3, "random"),
    ("f32", 4, 64, 520, 1.0, "random"),         # the largest tree
    ("bf16", 6, 1, 777, 1.0, "root"),           # a root alone: a plain draw from p_0
]


@pytest.mark.parametrize("case", SAMPLE_CASES, ids=[f"{c[0]}-s{c[1]}-r{c[2]}-v{c[3]}-{c[5]}" for c in SAMPLE_CASES])
def test_tree_sampling_matches_oracle(case):
    dtype, S, R, V, T, kind = case
    rng = np.random.default_rng(100 + SAMPLE_CASES.index(case))
    if kind == "bfs":
        par = np.stack([O.build_tree(R, [3, 2, 1]) for _ in range(S)])
    elif kind == "root":
        par = np.full((S, 1), -1)
    else:
        par = np.stack([random_tree(rng, R) for _ in range(S)])
    tally = RR.Tally()
    for rep in range(3):
        t, d, t64, d64, tokens = _sample_inputs(rng, dtype, S, R, V, T, par)
        ua, us = rng.random((S, R)), rng.random((S, R))
        ua32, us32 = ua.astype(np.float32), us.astype(np.float32)
        out, nacc, path, status = _run_tree_gpu(dtype, t, d, tokens, par, ua32, us32, T)
        assert status == (s3r.S3R_OK, 0)
        ref = O.tree_spec_sample(t64, d64, tokens, par, ua32.astype(np.float64), us32.astype(np.float64), RR.f32(T))
        _check_walk(f"{case} rep {rep}", out, nacc, path, par, tokens, V, ref, tally)
    assert tally.near_ties <= max(0, int(1e-3 * tally.decisions)), tally.notes


def test_acceptance_is_exercised_when_draft_equals_target():
    """q = p: every first child is accepted (ratio 1 > u), so the walk goes
    down to a leaf and draws there."""
    dtype, S, R, V, T = "bf16", 4, 9, 512, 1.0
    rng = np.random.default_rng(21)
    par = np.stack([O.build_tree(R, [2]) for _ in range(S)])
    t = _store(rng.standard_normal((S, R, V)), dtype)
    tokens = rng.integers(0, V, (S, R))
    ua, us = rng.random((S, R)).astype(np.float32) * 0.999, rng.random((S, R)).astype(np.float32)
    out, nacc, path, status = _run_tree_gpu(dtype, t, t, tokens, par, ua, us, T)
    assert status == (s3r.S3R_OK, 0)
    for b in range(S):
        # first children all the way down: 0 -> 1 -> 3 -> 7
        assert path[b, :nacc[b]].tolist() == [1, 3, 7][:nacc[b]] and nacc[b] == 3
    ref = O.tree_spec_sample(_wide(t, dtype), _wide(t, dtype), tokens, par, ua.astype(np.float64), us.astype(np.float64), RR.f32(T))
    _check_walk("q = p", out, nacc, path, par, tokens, V, ref, RR.Tally())


@pytest.mark.parametrize("dtype,V", [("bf16", 4096), ("f32", 1000)])
def test_chain_tree_equals_speculative_sampling(dtype, V):
    """Chain parents, node i + 1 carrying draft x_i: the tree walk commits
    what s3r_spec_sample commits on the same logits and uniforms."""
    rng = np.random.default_rng(31)
    S, gamma, T = 8, 6, 0.9
    R = gamma + 1
    par = np.broadcast_to(O.chain_parents(R), (S, R)).copy()
    t, d, t64, d64, tokens = _sample_inputs(rng, dtype, S, R, V, T, par, leaf_nan=False)
    ua, us = rng.random((S, R)).astype(np.float32), rng.random((S, R)).astype(np.float32)
    out, nacc, path, status = _run_tree_gpu(dtype, t, d, tokens, par, ua, us, T)
    assert status == (s3r.S3R_OK, 0)
    # the same round through s3r_spec_sample: drafts x_i = tokens[i + 1], u_accept[i] = ua[i + 1]
    o2 = torch.empty((S, R), dtype=torch.int32, device="cuda")
    n2 = torch.empty(S, dtype=torch.int32, device="cuda")
    ws = torch.zeros(s3r.s3r_sample_workspace_bytes(S, gamma, V), dtype=torch.uint8, device="cuda")
    s3r.s3r_spec_sample(_dev(t, dtype), _dev(np.ascontiguousarray(d[:, :gamma]), dtype), dtype,
                        _i32(tokens[:, 1:]), torch.from_numpy(np.ascontiguousarray(ua[:, 1:])).cuda(),
                        torch.from_numpy(us).cuda(), S, gamma, V, T, o2, n2, ws)
    ref = O.tree_spec_sample(t64, d64, tokens, par, ua.astype(np.float64), us.astype(np.float64), RR.f32(T))
    tally = RR.Tally()
    _check_walk("chain", out, nacc, path, par, tokens, V, ref, tally)
    o2, n2 = o2.cpu().numpy(), n2.cpu().numpy()
    for b in range(S):
        if (ref[3][b] and min(ref[3][b]) < ACCEPT_TIE) or ref[4][b] < DRAW_TIE:
            continue
        assert np.array_equal(out[b], o2[b]) and nacc[b] == n2[b], (b, out[b].tolist(), o2[b].tolist())


def test_bad_tree_and_bad_token_are_flagged():
    dtype, S, R, V, T = "f32", 3, 6, 300, 1.0
    rng = np.random.default_rng(41)
    par = np.stack([O.build_tree(R, [2]) for _ in range(S)])
    t, d, _, _, tokens = _sample_inputs(rng, dtype, S, R, V, T, par, leaf_nan=False)
    ua, us = rng.random((S, R)).astype(np.float32), rng.random((S, R)).astype(np.float32)
    bad = par.copy()
    bad[2, 0] = 0                                             # the root must have parent -1
    out, nacc, path, status = _run_tree_gpu(dtype, t, d, tokens, bad, ua, us, T)
    assert status[0] == s3r.S3R_ERR_DEVICE_CHECK and status[1] & s3r.S3R_DEV_BAD_TREE
    assert nacc[2] == 0 and 0 <= out[2, 0] < V                  # drawn at the root
    tok = tokens.copy()
    tok[1, 1] = V + 5
    out, nacc, path, status = _run_tree_gpu(dtype, t, d, tok, par, ua, us, T)
    assert status[0] == s3r.S3R_ERR_DEVICE_CHECK and status[1] & s3r.S3R_DEV_BAD_TOKEN_ID
    assert path[1, 0] != 1                                    # the bad token is never accepted


def test_full_vocab_tree_round_matches_oracle():
    """16 sequences, a 16-node tree, 151936-entry bf16 vocabulary."""
    dtype, S, R, V, T = "bf16", 16, 16, 151936, 1.0
    rng = np.random.default_rng(51)
    par = np.stack([O.build_tree(R, [4, 2, 1]) for _ in range(S)])
    t, d, t64, d64, tokens = _sample_inputs(rng, dtype, S, R, V, T, par, noise=0.3)
    ua, us = rng.random((S, R)).astype(np.float32), rng.random((S, R)).astype(np.float32)
    out, nacc, path, status = _run_tree_gpu(dtype, t, d, tokens, par, ua, us, T)
    assert status == (s3r.S3R_OK, 0)
    ref = O.tree_spec_sample(t64, d64, tokens, par, ua.astype(np.float64), us.astype(np.float64), RR.f32(T))
    tally = RR.Tally()
    _check_walk("full vocab", out, nacc, path, par, tokens, V, ref, tally)
    assert tally.near_ties <= 1, tally.notes
