"""One S3R decode step driven through the C ABI.

This module owns device buffers (allocated with torch: plumbing only) and
issues the library calls of one round in order; it performs no arithmetic of
its own. A round, as the S3R page (weekinpapers.com, Abstract) describes it:

  draft   gamma times: score the pages (the tail page summarised from K
          inside the call, the others from the page summaries), keep the
          top-B per KV head and sparse-attend over them
          (s3r_sparse_draft_attn), and draw the draft token from the draft
          distribution (s3r_sample_tokens);
  verify  dense causal attention of the gamma+1 rows (s3r_verify_attn);
  commit  exact speculative sampling (s3r_spec_sample).

The synthetic single-layer step has no model between these calls: the
queries and logits are seeded inputs (workloads.Workload). The gamma draft
tokens are drawn in one batched call at the start of the round (the same work
as gamma single-row calls). capture_round() records the whole round into one
CUDA graph for replay.
"""
from __future__ import annotations

import numpy as np
import torch

from . import s3r
from .workloads import Workload, algorithmic_bytes


def _to_torch(arr: np.ndarray, dtype: str, device) -> torch.Tensor:
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device)


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


class DecodeStep:
    """Device-resident inputs, outputs and workspaces of one round."""

    def __init__(self, wl: Workload, device="cuda", upload_chunk_pages: int = 2048):
        self.wl = wl
        ws = wl.spec
        self.device = torch.device(device)
        dev = self.device
        S, Hq, Hkv, D, P = ws.num_seqs, ws.num_q_heads, ws.num_kv_heads, ws.head_dim, ws.page_size
        R, g, V, B = ws.rows, ws.gamma, ws.vocab, ws.budget_pages
        kdt = torch_dtype(ws.kv_dtype)
        ldt = torch_dtype(ws.logit_dtype)
        n = wl.num_pages_total
        self.k_cache = torch.empty((n, Hkv, P, D), dtype=kdt, device=dev)
        self.v_cache = torch.empty((n, Hkv, P, D), dtype=kdt, device=dev)
        for start in range(0, n, upload_chunk_pages):
            ids = np.arange(start, min(n, start + upload_chunk_pages))
            self.k_cache[start:start + len(ids)] = _to_torch(wl.kv_pages("K", ids), ws.kv_dtype, dev)
            self.v_cache[start:start + len(ids)] = _to_torch(wl.kv_pages("V", ids), ws.kv_dtype, dev)
        self.block_table = torch.from_numpy(wl.block_table).to(dev)
        self.context_lens = torch.from_numpy(wl.context_lens).to(dev)
        self.kv = s3r.paged_kv(self.k_cache, self.v_cache, self.block_table, self.context_lens, Hq)
        self.kmin = torch.zeros((n, Hkv, D), dtype=kdt, device=dev)
        self.kmax = torch.zeros((n, Hkv, D), dtype=kdt, device=dev)

        self.q_draft = _to_torch(wl.q_draft, ws.kv_dtype, dev)          # [g, S, Hq, D]
        self.q_verify = _to_torch(wl.q_verify, ws.kv_dtype, dev)        # [S, R, Hq, D]
        tgt, drf = [], []
        for b in range(S):
            t, d = wl.logits_for_seq(b)
            tgt.append(_to_torch(t, ws.logit_dtype, dev))
            drf.append(_to_torch(d, ws.logit_dtype, dev))
        self.target_logits = torch.stack(tgt)                           # [S, R, V]
        self.draft_logits = torch.stack(drf)                            # [S, g, V]
        self.u_draft = torch.from_numpy(wl.u_draft).to(dev)             # [S, g]
        self.u_accept = torch.from_numpy(wl.u_accept).to(dev)
        self.u_sample = torch.from_numpy(wl.u_sample).to(dev)

        self.selected = torch.empty((g, S, Hkv, B), dtype=torch.int32, device=dev)
        self.draft_out = torch.empty((g, S, Hq, D), dtype=kdt, device=dev)
        self.draft_lse = torch.empty((g, S, Hq), dtype=torch.float32, device=dev)
        self.verify_out = torch.empty((S, R, Hq, D), dtype=kdt, device=dev)
        self.verify_lse = torch.empty((S, R, Hq), dtype=torch.float32, device=dev)
        self.draft_tokens = torch.empty((S, g), dtype=torch.int32, device=dev)
        self.draft_stats = torch.empty((S, g, 2), dtype=torch.float64, device=dev)   # {max, Z} of each q_i
        self.out_tokens = torch.empty((S, R), dtype=torch.int32, device=dev)
        self.num_accepted = torch.empty((S,), dtype=torch.int32, device=dev)

        # the round's own keys and values (drafter rows per step, verifier rows)
        kd, vd, kvr, vvr = zip(*(wl.round_kv(b) for b in range(S)))
        self.k_round_draft = _to_torch(np.stack(kd, axis=1), ws.kv_dtype, dev)[:, :, None]   # [g, S, 1, Hkv, D]
        self.v_round_draft = _to_torch(np.stack(vd, axis=1), ws.kv_dtype, dev)[:, :, None]
        self.k_round_verify = _to_torch(np.stack(kvr), ws.kv_dtype, dev)                       # [S, R, Hkv, D]
        self.v_round_verify = _to_torch(np.stack(vvr), ws.kv_dtype, dev)
        self.k_round_draft = [self.k_round_draft[i].contiguous() for i in range(g)]
        self.v_round_draft = [self.v_round_draft[i].contiguous() for i in range(g)]
        self.lens_committed = self.context_lens - R                                             # C = L - R
        self.ws_kv = self._ws(s3r.s3r_kv_workspace_bytes(S))
        self.ws_draft = self._ws(s3r.s3r_attn_workspace_bytes(self.kv, 1, B))
        self.ws_verify = self._ws(s3r.s3r_attn_workspace_bytes(self.kv, R, 0))
        self.ws_tokens = self._ws(s3r.s3r_sample_workspace_bytes(S * g, 0, V))
        self.ws_sample = self._ws(s3r.s3r_sample_workspace_bytes(S, g, V))
        self.scale = wl.scale

    def _ws(self, nbytes: int) -> torch.Tensor:
        assert nbytes > 0, "workspace query rejected the shapes"
        return torch.zeros(nbytes, dtype=torch.uint8, device=self.device)

    # ---------------------------------------------------------------- calls
    def summaries(self, tail_only: bool = False, stream=None):
        s3r.s3r_page_summaries(self.kv, int(tail_only), self.kmin, self.kmax, stream)

    def draw_draft_tokens(self, stream=None):
        ws = self.wl.spec
        s3r.s3r_sample_tokens(self.draft_logits, ws.logit_dtype, ws.num_seqs * ws.gamma, ws.vocab,
                              ws.temperature, self.u_draft, self.draft_tokens, self.ws_tokens, stream=stream,
                              row_stats=self.draft_stats)

    def draft(self, i: int, stream=None):
        """Draft step i: page scores and top-B (the tail page summarised from K
        inside the call), then sparse attention."""
        ws = self.wl.spec
        s3r.s3r_sparse_draft_attn(self.kv, self.kmin, self.kmax, self.q_draft[i], ws.budget_pages, self.scale,
                                  self.selected[i], self.draft_out[i], self.draft_lse[i], self.ws_draft,
                                  stream=stream)

    def verify(self, stream=None):
        s3r.s3r_verify_attn(self.kv, self.q_verify, self.wl.spec.rows, self.scale, self.verify_out,
                            self.verify_lse, self.ws_verify, stream=stream)

    def sample(self, stream=None, use_draft_stats=True):
        """Exact speculative sampling; by default with the draft rows' statistics written by
        draw_draft_tokens (s3r_spec_sample_ex), else computed inside the call."""
        ws = self.wl.spec
        s3r.s3r_spec_sample(self.target_logits, self.draft_logits, ws.logit_dtype, self.draft_tokens,
                            self.u_accept, self.u_sample, ws.num_seqs, ws.gamma, ws.vocab, ws.temperature,
                            self.out_tokens, self.num_accepted, self.ws_sample, stream=stream,
                            draft_stats=self.draft_stats if use_draft_stats else None)

    def round(self, stream=None):
        """One whole decode step: gamma drafts, verify, commit."""
        self.draw_draft_tokens(stream)
        for i in range(self.wl.spec.gamma):
            self.draft(i, stream)
        self.verify(stream)
        self.sample(stream)

    def round_with_kv(self, stream=None):
        """One round with the cache kept: from the committed lengths C = L - R,
        each draft step writes its keys and values at the end of the cache
        (s3r_kv_append) before its sparse attention; verification writes the
        verifier's R rows over the round's positions before dense attention;
        sampling commits and s3r_kv_rollback keeps the committed prefix. The
        lengths start from C on every call (a copy on the stream), so rounds
        can be repeated and captured."""
        ws = self.wl.spec
        g, R = ws.gamma, ws.rows
        st = torch.cuda.current_stream(self.device) if stream is None else stream
        with torch.cuda.stream(st):
            self.context_lens.copy_(self.lens_committed)
        self.draw_draft_tokens(stream)
        for i in range(g):
            s3r.s3r_kv_append(self.kv, self.context_lens, self.k_round_draft[i], self.v_round_draft[i], 1, 0,
                              self.kmin, self.kmax, self.ws_kv, stream=stream)
            self.draft(i, stream)
        s3r.s3r_kv_append(self.kv, self.context_lens, self.k_round_verify, self.v_round_verify, R, g,
                          self.kmin, self.kmax, self.ws_kv, stream=stream)
        self.verify(stream)
        self.sample(stream)
        s3r.s3r_kv_rollback(self.kv, self.context_lens, self.num_accepted, R, self.kmin, self.kmax, self.ws_kv,
                            stream=stream)

    def capture_round(self):
        """One whole round captured into a CUDA graph. The library's kernels
        chain by programmatic dependent launch, which the capture keeps as
        programmatic edges; graph.replay() reruns the round on the same
        buffers (the workspaces need no reset between rounds)."""
        dev = self.device
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            self.round(side)
        torch.cuda.current_stream(dev).wait_stream(side)
        return graph

    def device_checks(self):
        """Status words of every workspace (synchronises)."""
        return {name: s3r.s3r_device_status(getattr(self, name))
                for name in ("ws_draft", "ws_verify", "ws_tokens", "ws_sample", "ws_kv")}

    # ---------------------------------------------------------------- bytes
    def algorithmic_bytes(self):
        """Bytes each step must move (what the method has to read/write)."""
        return algorithmic_bytes(self.wl)
