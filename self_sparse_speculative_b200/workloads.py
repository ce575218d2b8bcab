"""Seeded synthetic inputs for one S3R decode step.

This module only draws and stores inputs. It holds none of the method's
arithmetic: no attention, no page scoring, no softmax, no sampling. Both the
CUDA path (through the Python binding) and the float64 oracle take their
inputs from here, so that the two compute on the same bits.

What the inputs stand in for: the S3R page ("S3R: Fast and Faithful RL
Rollouts via Self-Sparse Speculative Decoding", Abstract) profiles long-context
mathematical-reasoning RLVR rollouts on Qwen3 models. No dataset or weights are
used; the shapes follow Qwen3-8B/14B attention layers (GQA 32q/8kv and 40q/8kv,
head_dim 128) over a paged KV cache (PagedAttention, cited on the same page's
reference list), and the value distributions are the ones each workload below
states.

Recipe (every stream is an independent numpy PCG64 generator keyed by
``SeedSequence(seed, spawn_key=(workload index, stream id, ...))``):

* physical page ids: a seeded permutation of all pages, so a sequence's pages
  are scattered in the cache as a real allocator leaves them;
* K and V: drawn per physical page (all KV heads of the page at once), i.i.d.
  N(0,1); the bf16 workloads add a per-head low-rank outlier component on 8
  seeded channels: ``x[t, h, c_h] += z[t, h] * w_h`` with ``z ~ N(0, 2^2)`` and
  ``w_h ~ N(0, 1)^8 / sqrt(8)`` (K and V have independent channels, w and z);
* queries: i.i.d. N(0,1); one query tensor per draft step and one for verify;
* logits: per sequence; target ``N(0, s_t^2)``, draft ``target + N(0, s_d^2)``
  (the tiny fp32 workload instead takes draft ``z`` and target ``z + 0.3 z'``);
* uniforms: float32 in [0, 1): one per draft token (drawing the draft token
  from q), one per accept test, one per sampling position.

Floating values are drawn in float32 and rounded once to the storage dtype
(round-to-nearest-even for bf16), so the GPU and the oracle see identical bits.
bf16 values are held as ``uint16`` bit patterns.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# stream ids for SeedSequence spawn keys
_S_K, _S_V, _S_OUT_K, _S_OUT_V = 1, 2, 3, 4
_S_QDRAFT, _S_QVERIFY, _S_LOGITS, _S_UNIF, _S_PERM, _S_LENS = 5, 6, 7, 8, 9, 10
_S_ROUND_KV = 11


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    index: int
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    context: int            # every sequence's length; 0 means ragged
    ragged_lo: int
    ragged_hi: int
    budget_pages: int       # sparse draft budget B, in pages
    gamma: int              # drafts per round
    vocab: int
    temperature: float
    kv_dtype: str           # "f32" or "bf16"
    logit_dtype: str        # "f32" or "bf16"
    kv_outliers: bool
    target_std: float
    draft_noise_std: float
    tiny_logits: bool       # draft z, target z + 0.3 z'

    @property
    def rows(self) -> int:
        """Verify rows per sequence: the last committed token plus gamma drafts."""
        return self.gamma + 1

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


WORKLOADS = [
    WorkloadSpec(0, "tiny-fp32: 1 seq, 4q/1kv, D64, L256, page16, B=4 pages, gamma3, V1000",
                 1, 4, 1, 64, 16, 256, 0, 0, 4, 3, 1000, 1.0, "f32", "f32",
                 False, 1.0, 0.0, True),
    WorkloadSpec(1, "qwen3-8b-layer: 16 seq, 32q/8kv, D128, L16384, page64, B=32 pages, gamma4, V151936 bf16",
                 16, 32, 8, 128, 64, 16384, 0, 0, 32, 4, 151936, 1.0, "bf16", "bf16",
                 True, 2.0, 0.5, False),
    WorkloadSpec(2, "ragged: 64 seq, 32q/8kv, D128, L~U[4096,32768], page64, B=32 pages, gamma4, V151936 bf16",
                 64, 32, 8, 128, 64, 0, 4096, 32768, 32, 4, 151936, 1.0, "bf16", "bf16",
                 True, 2.0, 0.5, False),
    WorkloadSpec(3, "tail: 4 seq, 32q/8kv, D128, L65536, page64, B=64 pages, gamma6, V151936 bf16",
                 4, 32, 8, 128, 64, 65536, 0, 0, 64, 6, 151936, 1.0, "bf16", "bf16",
                 True, 2.0, 1.0, False),
    WorkloadSpec(4, "wide: 256 seq, 40q/8kv, D128, L8192, page64, B=16 pages, gamma8, V151936 fp32 logits T0.7",
                 256, 40, 8, 128, 64, 8192, 0, 0, 16, 8, 151936, 0.7, "bf16", "f32",
                 True, 2.0, 0.3, False),
]


def spec(index: int) -> WorkloadSpec:
    return WORKLOADS[index]


def custom_spec(base: int = 0, **overrides) -> WorkloadSpec:
    """A workload with some fields replaced (small parity cases, edge cases)."""
    return dataclasses.replace(WORKLOADS[base], **overrides)


# ---------------------------------------------------------------- storage dtypes
def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_float32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16_bits(x)
    return np.ascontiguousarray(x, dtype=np.float32)


def to_float64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Widen stored values exactly to float64."""
    if dtype == "bf16":
        return bf16_bits_to_float32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def storage_itemsize(dtype: str) -> int:
    return 2 if dtype == "bf16" else 4


# ---------------------------------------------------------------- the workload
def _threads() -> int:
    return max(1, min(32, len(os.sched_getaffinity(0))))


class Workload:
    """All inputs of one decode step for one workload spec and seed.

    Small tensors are drawn eagerly; the KV cache and the logits are drawn on
    demand (per physical page, per sequence) so that large workloads can be
    streamed to the GPU and sampled by the oracle without holding everything
    in host memory at once.
    """

    def __init__(self, ws: WorkloadSpec, seed: int = 0, context_lens=None):
        self.spec = ws
        self.seed = seed
        S, P = ws.num_seqs, ws.page_size
        if context_lens is not None:
            lens = np.asarray(context_lens, dtype=np.int64)
            assert lens.shape == (S,)
        elif ws.context:
            lens = np.full(S, ws.context, dtype=np.int64)
        else:
            u = self._rng(_S_LENS).uniform(ws.ragged_lo, ws.ragged_hi, size=S)
            lens = (np.floor(u / P) * P).astype(np.int64)
        if context_lens is None:
            lens = np.maximum(lens, ws.rows)
        self.context_lens = lens.astype(np.int32)
        self.pages_per_seq = ((lens + P - 1) // P).astype(np.int64)
        self.max_pages_per_seq = int(self.pages_per_seq.max())
        self.num_pages_total = int(self.pages_per_seq.sum())
        perm = self._rng(_S_PERM).permutation(self.num_pages_total).astype(np.int32)
        bt = np.full((S, self.max_pages_per_seq), -1, dtype=np.int32)
        off = 0
        for b in range(S):
            n = int(self.pages_per_seq[b])
            bt[b, :n] = perm[off:off + n]
            off += n
        self.block_table = bt
        # owner sequence and logical index of every physical page
        self.page_owner = np.empty(self.num_pages_total, dtype=np.int32)
        self.page_logical = np.empty(self.num_pages_total, dtype=np.int32)
        for b in range(S):
            n = int(self.pages_per_seq[b])
            self.page_owner[bt[b, :n]] = b
            self.page_logical[bt[b, :n]] = np.arange(n, dtype=np.int32)

        H, Hq, D, R, g = ws.num_kv_heads, ws.num_q_heads, ws.head_dim, ws.rows, ws.gamma
        self._outlier = {}
        if ws.kv_outliers:
            for which, sid in (("K", _S_OUT_K), ("V", _S_OUT_V)):
                rng = self._rng(sid)
                ch = np.stack([rng.choice(D, size=8, replace=False) for _ in range(H)])
                w = (rng.standard_normal((H, 8)) / math.sqrt(8.0)).astype(np.float32)
                self._outlier[which] = (ch, w)
        qd = self._rng(_S_QDRAFT).standard_normal((g, S, Hq, D), dtype=np.float32)
        qv = self._rng(_S_QVERIFY).standard_normal((S, R, Hq, D), dtype=np.float32)
        self.q_draft = to_storage(qd, ws.kv_dtype)      # [gamma, S, Hq, D]
        self.q_verify = to_storage(qv, ws.kv_dtype)     # [S, R, Hq, D]
        ur = self._rng(_S_UNIF)
        self.u_draft = ur.random((S, g), dtype=np.float32)
        self.u_accept = ur.random((S, g), dtype=np.float32)
        self.u_sample = ur.random((S, R), dtype=np.float32)
        self.scale = 1.0 / math.sqrt(D)

    # -- generators
    def _rng(self, *key) -> np.random.Generator:
        ss = np.random.SeedSequence(self.seed, spawn_key=(self.spec.index,) + tuple(int(k) for k in key))
        return np.random.Generator(np.random.PCG64(ss))

    # -- KV cache
    def _page_f32(self, which: str, phys: int) -> np.ndarray:
        ws = self.spec
        H, P, D = ws.num_kv_heads, ws.page_size, ws.head_dim
        rng = self._rng(_S_K if which == "K" else _S_V, phys)
        x = rng.standard_normal((H, P, D), dtype=np.float32)
        if ws.kv_outliers:
            ch, w = self._outlier[which]
            z = 2.0 * rng.standard_normal((H, P), dtype=np.float32)
            for h in range(H):
                x[h][:, ch[h]] += z[h][:, None] * w[h][None, :]
        return x

    def kv_pages(self, which: str, phys_pages) -> np.ndarray:
        """Stored values of the given physical pages: [n, Hkv, P, D]."""
        phys_pages = np.asarray(phys_pages, dtype=np.int64).reshape(-1)
        dt = self.spec.kv_dtype
        def one(p):
            return to_storage(self._page_f32(which, int(p)), dt)
        if len(phys_pages) > 64:
            with ThreadPoolExecutor(_threads()) as ex:
                parts = list(ex.map(one, phys_pages))
        else:
            parts = [one(p) for p in phys_pages]
        ws = self.spec
        if not parts:
            return np.zeros((0, ws.num_kv_heads, ws.page_size, ws.head_dim),
                            dtype=np.uint16 if dt == "bf16" else np.float32)
        return np.stack(parts)

    def kv_cache(self, which: str) -> np.ndarray:
        """The whole cache [num_pages_total, Hkv, P, D] (small workloads only)."""
        return self.kv_pages(which, np.arange(self.num_pages_total))

    def kv_bytes(self) -> int:
        ws = self.spec
        return 2 * self.num_pages_total * ws.num_kv_heads * ws.page_size * ws.head_dim * storage_itemsize(ws.kv_dtype)

    # -- the keys and values a round writes (a round over the last R positions)
    def round_kv(self, b: int):
        """Keys and values of sequence b's round, as the model would produce
        them: the drafter's rows of the gamma draft steps and the verifier's
        rows of the R = gamma + 1 round positions, [gamma, Hkv, D] and
        [R, Hkv, D] each for K and V, drawn like the cache (N(0, 1) plus the
        workload's outlier component), in the storage dtype."""
        ws = self.spec
        H, D, g, R = ws.num_kv_heads, ws.head_dim, ws.gamma, ws.rows
        out = []
        for which, sid in (("K", 0), ("V", 1)):
            rng = self._rng(_S_ROUND_KV, b, sid)
            x = rng.standard_normal((g + R, H, D), dtype=np.float32)
            if ws.kv_outliers:
                ch, w = self._outlier[which]
                z = 2.0 * rng.standard_normal((g + R, H), dtype=np.float32)
                for h in range(H):
                    x[:, h][:, ch[h]] += z[:, h][:, None] * w[h][None, :]
            out.append(to_storage(x, ws.kv_dtype))
        k, v = out
        return k[:g], v[:g], k[g:], v[g:]

    # -- logits
    def logits_for_seq(self, b: int):
        """(target [R, V], draft [gamma, V]) stored logits of sequence b."""
        ws = self.spec
        R, g, V = ws.rows, ws.gamma, ws.vocab
        rng = self._rng(_S_LOGITS, b)
        if ws.tiny_logits:
            z = rng.standard_normal((R, V), dtype=np.float32)
            z2 = rng.standard_normal((R, V), dtype=np.float32)
            tgt = z + np.float32(0.3) * z2
            drf = z[:g].copy()
        else:
            tgt = np.float32(ws.target_std) * rng.standard_normal((R, V), dtype=np.float32)
            drf = tgt[:g] + np.float32(ws.draft_noise_std) * rng.standard_normal((g, V), dtype=np.float32)
        return to_storage(tgt, ws.logit_dtype), to_storage(drf, ws.logit_dtype)

    def logits(self, seqs=None):
        """(target [n, R, V], draft [n, gamma, V]) for the given sequences."""
        seqs = range(self.spec.num_seqs) if seqs is None else seqs
        seqs = list(seqs)
        if len(seqs) > 4:
            with ThreadPoolExecutor(_threads()) as ex:
                parts = list(ex.map(self.logits_for_seq, seqs))
        else:
            parts = [self.logits_for_seq(b) for b in seqs]
        return np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts])


def algorithmic_bytes(wl: "Workload"):
    """Bytes one step of workload `wl` must move (what the method has to
    read/write): per draft call the summaries of every page plus the K/V
    of the selected pages, verify the K/V of every token, sampling the
    (2 gamma + 1) rows plus the 2 re-read rows, the drafter's draws
    gamma rows per sequence."""
    ws = wl.spec
    Hkv, D, P, B = ws.num_kv_heads, ws.head_dim, ws.page_size, ws.budget_pages
    elt = 2 if ws.kv_dtype == "bf16" else 4
    lelt = 2 if ws.logit_dtype == "bf16" else 4
    lens = wl.context_lens.astype(np.int64)
    n_b = wl.pages_per_seq
    kv_tok = 2 * Hkv * D * elt                                  # K + V per token
    # sparse draft: page summaries of every page (kmin+kmax) + selected KV
    sel_tokens = 0
    for L, n in zip(lens, n_b):
        k = min(int(n), B)
        # the selected pages are full except possibly the tail page
        sel_tokens += min(int(L), k * P)
    draft = int(n_b.sum()) * Hkv * 2 * D * elt + sel_tokens * kv_tok
    verify = int(lens.sum()) * kv_tok
    V, g = ws.vocab, ws.gamma
    sample = ws.num_seqs * ((2 * g + 1) * V * lelt + 2 * V * lelt)
    draw = ws.num_seqs * g * V * lelt
    return {"draft_per_call": draft, "verify": verify, "sample": sample, "draft_tokens": draw,
            "step": g * draft + verify + sample + draw}


def kv_append_bytes(lens, n, overwrite, page_size, kv_heads, head_dim, elt):
    """Bytes one s3r_kv_append must move: the n new K and V rows read and
    written per KV head, and for every page holding a written row its valid
    keys read and its kmin / kmax written. lens: lengths before the call."""
    P, D = page_size, head_dim
    total = 0
    for L in np.asarray(lens, dtype=np.int64):
        start = int(L) - overwrite
        new_len = start + n
        rows = 2 * 2 * n * D * elt                                    # K and V, read and written
        summ = 0
        for pg in range(start // P, (new_len - 1) // P + 1):
            valid = min(P, new_len - pg * P)
            summ += valid * D * elt + 2 * D * elt
        total += kv_heads * (rows + summ)
    return total


def kv_rollback_bytes(new_lens, page_size, kv_heads, head_dim, elt):
    """Bytes one s3r_kv_rollback must move: the new tail page's valid keys
    read and its kmin / kmax written, per KV head."""
    P, D = page_size, head_dim
    total = 0
    for L in np.asarray(new_lens, dtype=np.int64):
        pg = (int(L) - 1) // P
        total += kv_heads * ((int(L) - pg * P) * D * elt + 2 * D * elt)
    return total


def tree_sample_bytes(parents, num_accepted, path, vocab, elt):
    """Bytes a tree walk must read: the target row of every visited node and
    the draft row of every visited node that has children (the first pass over
    a node's rows; the later passes of the walk re-read them from L2)."""
    total = 0
    for b in range(parents.shape[0]):
        visited = [0] + [int(path[b, i]) for i in range(int(num_accepted[b]))]
        for v in visited:
            has_child = bool(np.any(parents[b] == v))
            total += vocab * elt * (2 if has_child else 1)
    return total


def breadth_first_tree(n_nodes, branching):
    """Parents of an n_nodes tree in breadth-first order, node d-deep getting
    branching[d] children (the last entry repeats)."""
    parents, frontier, d = [-1], [0], 0
    while len(parents) < n_nodes and frontier:
        k = branching[min(d, len(branching) - 1)]
        nxt = []
        for v in frontier:
            for _ in range(k):
                if len(parents) < n_nodes:
                    parents.append(v)
                    nxt.append(len(parents) - 1)
        frontier, d = nxt, d + 1
    return np.array(parents, dtype=np.int64)
