#!/usr/bin/env python
"""Benchmark of one S3R decode step on B200 (verified tokens/s, KV GB/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ours|reference]

A step is one whole round of the hot path on one batch: gamma sparse-draft
calls (tail-page summary + page scoring/top-B, then split-KV attention),
the drafter's token draws, dense causal verification of the gamma+1 rows, and
exact speculative sampling. Inputs are seeded synthetic tensors shaped like
the Qwen3-8B layer workload (16 sequences x 16384 tokens, 32q/8kv heads,
head_dim 128, 64-token pages, B = 32 pages, gamma = 4, vocab 151936, bf16),
resident in HBM before timing. Metric: verified (committed) tokens per second
= sum over sequences of (accepted drafts + 1) / step time.

With one process and steps larger than L2, the round is also captured once
into a CUDA graph (DecodeStep.capture_round) and replayed K times, device-timed
inside the clock-sampling window; those replays give the headline value
("timed": "cuda graph replay of the round") and the eager steps, which also
give the per-call phases, are reported under "eager". Otherwise, or if the
capture fails (its error is reported under "graph"), the eager steps are the
headline. --no-graph skips the capture.

Multi-GPU (torchrun, one rank per GPU): sequences are independent, so every
rank runs its own full batch (weak scaling, no data-path collective); the
step time is the max over ranks.

--impl reference times the float64 CPU oracle on the host cores instead (a
bounded sample of the same workload per step).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import signal
import statistics
import subprocess
import sys
import tempfile
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402

METRIC = "verified tokens/s per decode step on 1 B200; KV-read GB/s as % of HBM peak"
L2_BYTES = 126 * 2 ** 20
FLUSH_BYTES = 256 * 2 ** 20
UNIT = "tokens/s"


def _peaks():
    try:
        with open(os.path.join(HERE, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------- CPU oracle
def _oracle_seq_worker(args):
    """One sequence's float64 oracle round in a worker process. Its inputs
    are generated first, outside the timer; only the oracle's arithmetic
    (summaries, gamma selections and sparse drafts, verify, draft draws and
    speculative sampling) is timed. Returns (committed tokens, seconds)."""
    idx, seed, b = args
    from self_sparse_speculative_b200.workloads import Workload, spec
    import oracle.reference_run as RR
    wl = Workload(spec(idx), seed=seed)
    inp = RR.sequence_inputs(wl, b)
    t0 = time.perf_counter()
    RR.oracle_attention(inp)
    s = RR.oracle_sampling(inp)
    return s["n_acc"] + 1, time.perf_counter() - t0


# one BLAS thread per oracle process (the processes already take one core
# each); set in the environment the spawned processes start with, since the
# BLAS library reads it when numpy is first imported
_ONE_THREAD = {"OMP_NUM_THREADS": "1", "OPENBLAS_NUM_THREADS": "1", "MKL_NUM_THREADS": "1"}


class OracleRunner:
    """A pool of `workers` single-threaded processes (spawned, so it is safe
    whether or not the parent holds a CUDA context) that runs the oracle on
    one sequence per process. A step's time is the slowest process's
    arithmetic time: the processes run at once, one per core."""

    def __init__(self, workers):
        import multiprocessing as mp
        self.workers = workers
        self.pool = None
        if workers > 1:
            saved = {k: os.environ.get(k) for k in _ONE_THREAD}
            os.environ.update(_ONE_THREAD)
            try:
                self.pool = mp.get_context("spawn").Pool(workers)
            finally:
                for k, v in saved.items():
                    if v is None:
                        os.environ.pop(k, None)
                    else:
                        os.environ[k] = v

    def step(self, idx, seed, seqs):
        jobs = [(idx, seed, b) for b in seqs]
        res = self.pool.map(_oracle_seq_worker, jobs, chunksize=1) if self.pool else \
            [_oracle_seq_worker(j) for j in jobs]
        if self.pool is None:
            return sum(r[0] for r in res), sum(r[1] for r in res)
        # the processes run at once: the slowest one, or the arithmetic spread
        # over the processes when sequences outnumber them
        per = [r[1] for r in res]
        return sum(r[0] for r in res), max(max(per), sum(per) / self.workers)

    def close(self):
        if self.pool is not None:
            self.pool.close()
            self.pool.join()


def cpu_cores():
    return len(os.sched_getaffinity(0))


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample_note(ws, seqs, steps, cores):
    return (f"float64 oracle round (summaries, {ws.gamma} sparse drafts, verify, draft draws, speculative "
            f"sampling) of {len(seqs)} of {ws.num_seqs} sequences per step, {steps} step(s), one process "
            f"per sequence on {cores} of {cpu_cores()} host cores ({cpu_model()}); inputs generated "
            f"before the timer, only the oracle arithmetic timed")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.send_signal(signal.SIGTERM)
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- our arm
# sources of the verify kernel; the committed ncu summary records their hash
VERIFY_SOURCES = ("s3r_attn_tok.cu", "s3r_tok_common.cuh", "s3r_attn_sched.cuh", "s3r_attn_common.cuh", "s3r_device.cuh")
VERIFY_PROFILE = os.path.join(HERE, "profiles", "verify_attn_tok_qwen3-8b-layer.md")


def _code_only(text):
    """Source text without comments, trailing blanks and empty lines, so that
    the hash identifies the compiled code, not its commentary."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


# where the host-side launch code of the attention kernel file begins (the
# hash below covers the device code before it)
HOST_SECTION = "cudaError_t launch_tok("


def verify_source_hash():
    """Hash of the verify kernel's device code (comments removed) that a
    committed ncu summary names; traffic figures from another build are not
    reported."""
    import hashlib
    h = hashlib.sha256()
    for f in VERIFY_SOURCES:
        with open(os.path.join(HERE, "self_sparse_speculative_b200", "csrc", f), encoding="utf-8") as fh:
            text = fh.read()
        if f == "s3r_attn_tok.cu":
            text = text[:text.index(HOST_SECTION)]
        h.update(_code_only(text).encode())
    return h.hexdigest()[:16]


def verify_traffic(workload=None):
    """DRAM bytes (read + write) per verify launch from the committed ncu
    summary, or None when it was taken on other kernel sources or (given a
    workload name) on another workload."""
    try:
        kv = {}
        with open(VERIFY_PROFILE) as f:
            for line in f:
                if line.startswith("- ") and ":" in line:
                    k, v = line[2:].split(":", 1)
                    kv[k.strip()] = v.strip().strip("`")
        if kv.get("source hash", "").split("`")[0].strip() != verify_source_hash():
            return None
        if workload is not None and kv.get("workload") != workload:
            return None
        return int(kv["dram bytes per launch"])
    except Exception:
        return None


def launches_per_step(ws, draft_kernels=2):
    """Library kernels per step: the drafter's draws (1), gamma draft calls of
    draft_kernels each (one fused kernel, or selection then attention),
    verify (1), sampling (statistics, normalisers, draw)."""
    return 1 + draft_kernels * ws.gamma + 1 + 3


def l2_note(step_bytes):
    if step_bytes > L2_BYTES:
        return "not flushed: each step reads %.2f GB > 126 MB L2" % (step_bytes / 1e9)
    return "flushed before every timed step (256 MB write outside the timed spans)"


def config_of(ws, world, seed, step_bytes=None):
    return {"workload": ws.name, "sequences_per_gpu": ws.num_seqs, "context": ws.context,
            "q_heads": ws.num_q_heads, "kv_heads": ws.num_kv_heads, "head_dim": ws.head_dim,
            "page": ws.page_size, "budget_pages": ws.budget_pages, "gamma": ws.gamma,
            "vocab": ws.vocab, "parallelism": f"replicas x{world} (sequence-sharded, no collective)",
            "l2": l2_note(step_bytes) if step_bytes is not None else "host memory", "seed": seed}


def over_ranks(ms, tokens, world, device):
    """(max over ranks of a device time in ms, sum over ranks of a token count).
    Every rank must call it at the same point (two collectives)."""
    if world <= 1:
        return float(ms), float(tokens)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    k = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(k, op=dist.ReduceOp.SUM)
    return float(t.item()), float(k.item())


def cpu_baseline_leg(a, ws):
    """The oracle timed on the host cores (rank 0 at N = 1 only): a bounded
    sample of the workload's sequences, the same runner as the reference arm."""
    seqs = list(range(min(ws.num_seqs, a.cpu_seqs)))
    workers = max(1, min(len(seqs), cpu_cores()))
    runner = OracleRunner(workers)
    try:
        runner.step(a.workload, a.seed, [0])                      # warm-up: worker start, imports
        tok, secs = runner.step(a.workload, a.seed, seqs)
    finally:
        runner.close()
    return {"value": round(tok / secs, 3), "unit": UNIT, "cores": workers, "kind": "oracle",
            "sample": oracle_sample_note(ws, seqs, 1, workers) + f", {secs:.2f} s"}


def _tensor_peak():
    try:
        with open(os.path.join(HERE, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def gamma_policy_note(ws, st, hbm_gbs):
    """The library's draft-length policy on this workload: acceptance
    measured from the step's counts, round costs from its roofline model at
    the HBM peak used above and the bf16 tensor peak; the draft length it
    would choose next (0: drafting off) and the rate gain over plain decoding."""
    from self_sparse_speculative_b200 import s3r
    tf = _tensor_peak()
    L = float(np.mean(st.wl.context_lens))
    kvb = 2 if ws.kv_dtype == "bf16" else 4
    lb = 2 if ws.logit_dtype == "bf16" else 4
    gmax = 8 if ws.gamma <= 8 else ws.gamma
    cost = [s3r.s3r_round_cost_us(ws.num_seqs, ws.num_q_heads, ws.num_kv_heads, ws.head_dim, ws.page_size, kvb, L,
                                  ws.budget_pages, ws.vocab, lb, g, hbm_gbs, tf) for g in range(gmax + 1)]
    pol = s3r.GammaPolicyHandle(gmax, 0.9, 0.5, 1.0, cost)
    pol.update(st.num_accepted.cpu().tolist(), ws.gamma)
    g, alpha, rate = pol.choose()
    return {"acceptance_estimate": round(alpha, 4), "gamma_next": g,
            "model_rate_gain_vs_plain_decode": round(rate * cost[0], 3),
            "cost_model": f"roofline at {hbm_gbs:.0f} GB/s and {tf:.0f} TFLOP/s"}


def next_rows_measure(st, ws, stream, peak, steps, seed):
    """The calls beyond the five-part step on the same cache: the KV upkeep
    of a round (a drafter row appended, the verifier's rows written over the
    round's positions, the rollback to the committed prefix) and tree
    verification (a tree of N_t nodes, N_t from the concurrency-aware budget
    with one node per sequence and head group of capacity, the tree's
    ancestor-masked attention over the whole cache, and the tree walk of
    exact speculative sampling). Each: microseconds per call (mean of
    `steps` calls, CUDA events on the launching stream) and algorithmic
    bytes over that time against the HBM peak."""
    import torch
    from self_sparse_speculative_b200 import s3r
    from self_sparse_speculative_b200 import workloads as W
    S, Hq, Hkv, D, P, V = ws.num_seqs, ws.num_q_heads, ws.num_kv_heads, ws.head_dim, ws.page_size, ws.vocab
    g, R = ws.gamma, ws.rows
    elt = 2 if ws.kv_dtype == "bf16" else 4
    lelt = 2 if ws.logit_dtype == "bf16" else 4
    lens_full = st.context_lens.clone()
    lens0 = st.lens_committed.cpu().numpy()
    out = {}

    def timed(fn, n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for e0, e1 in evs:
            fn(e0, e1)
        torch.cuda.synchronize()
        return sum(e0.elapsed_time(e1) for e0, e1 in evs) / n * 1e3     # us

    def entry(us, nbytes):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us_per_call": round(us, 2), "algorithmic_bytes": int(nbytes), "gbs": round(gbs, 1),
                "frac_of_peak": round(gbs / peak, 4)}

    # ---- KV upkeep: a round's appends and rollback, from the committed lengths
    t_app, t_ver, t_rb = [], [], []

    def one_round(e0, e1):
        st.context_lens.copy_(st.lens_committed)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        s3r.s3r_kv_append(st.kv, st.context_lens, st.k_round_draft[0], st.v_round_draft[0], 1, 0, st.kmin, st.kmax,
                          st.ws_kv, stream=stream)
        a1.record(stream)
        t_app.append((a0, a1))
        for i in range(1, g):
            s3r.s3r_kv_append(st.kv, st.context_lens, st.k_round_draft[i], st.v_round_draft[i], 1, 0, st.kmin,
                              st.kmax, st.ws_kv, stream=stream)
        e0.record(stream)
        s3r.s3r_kv_append(st.kv, st.context_lens, st.k_round_verify, st.v_round_verify, R, g, st.kmin, st.kmax,
                          st.ws_kv, stream=stream)
        e1.record(stream)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        s3r.s3r_kv_rollback(st.kv, st.context_lens, st.num_accepted, R, st.kmin, st.kmax, st.ws_kv, stream=stream)
        r1.record(stream)
        t_rb.append((r0, r1))

    for _ in range(3):
        one_round(torch.cuda.Event(), torch.cuda.Event())
    t_app.clear(); t_rb.clear()
    us_ver = timed(one_round, steps)
    us_app = sum(a.elapsed_time(b) for a, b in t_app) / len(t_app) * 1e3
    us_rb = sum(a.elapsed_time(b) for a, b in t_rb) / len(t_rb) * 1e3
    new_lens = lens0 + st.num_accepted.cpu().numpy() + 1
    out["kv_append_draft_row"] = entry(us_app, W.kv_append_bytes(lens0, 1, 0, P, Hkv, D, elt))
    out["kv_append_verify_rows"] = entry(us_ver, W.kv_append_bytes(lens0 + g, R, g, P, Hkv, D, elt))
    out["kv_rollback"] = entry(us_rb, W.kv_rollback_bytes(new_lens, P, Hkv, D, elt))
    # the cache's lengths and tail summaries as before
    st.context_lens.copy_(lens_full)
    st.summaries(tail_only=True)
    torch.cuda.synchronize()

    # ---- tree verification: node budget, attention, tree walk
    G = Hq // Hkv
    n_max = min(64, 64 // G) if ws.kv_dtype == "bf16" else min(64, 128 // G)
    n_t = s3r.s3r_tree_node_budget(S * n_max, S, 2, n_max)
    parents = np.broadcast_to(W.breadth_first_tree(n_t, [4, 2, 1]), (S, n_t)).copy()
    gen = torch.Generator(device=st.device).manual_seed(seed + 1234)
    dt = st.k_cache.dtype
    q = torch.randn((S, n_t, Hq, D), generator=gen, device=st.device, dtype=torch.float32).to(dt)
    par_d = torch.from_numpy(parents.astype(np.int32)).to(st.device)
    o = torch.empty((S, n_t, Hq, D), dtype=dt, device=st.device)
    lse = torch.empty((S, n_t, Hq), dtype=torch.float32, device=st.device)
    wsv = torch.zeros(s3r.s3r_attn_workspace_bytes(st.kv, n_t, 0), dtype=torch.uint8, device=st.device)

    def tree_attn(e0, e1):
        e0.record(stream)
        s3r.s3r_verify_attn_tree(st.kv, q, n_t, par_d, st.scale, o, lse, wsv, stream=stream)
        e1.record(stream)

    for _ in range(3):
        tree_attn(torch.cuda.Event(), torch.cuda.Event())
    us_tv = timed(tree_attn, steps)
    kv_bytes = int(st.wl.context_lens.astype(np.int64).sum()) * 2 * Hkv * D * elt
    out["tree_verify_attn"] = dict(entry(us_tv, kv_bytes), nodes=n_t, node_budget="N_t = clip(floor(C_hw / B_t), 2, "
                                   f"{n_max}) with C_hw = {S * n_max}, B_t = {S}")
    # logits of every node after the workload's recipe (target N(0, s^2), draft
    # = target + noise); children's tokens drawn from their parent's draft row
    ldt = st.target_logits.dtype
    sigma, noise = (1.0, 0.3) if ws.tiny_logits else (ws.target_std, ws.draft_noise_std)
    tgt = (sigma * torch.randn((S, n_t, V), generator=gen, device=st.device)).to(ldt)
    drf = (tgt.float() + noise * torch.randn((S, n_t, V), generator=gen, device=st.device)).to(ldt)
    child_rows = drf[:, torch.from_numpy(np.maximum(parents[0, 1:], 0)).to(st.device)].reshape(S * (n_t - 1), V)
    u_tok = torch.rand((S * (n_t - 1),), generator=gen, device=st.device)
    tok = torch.empty((S * (n_t - 1),), dtype=torch.int32, device=st.device)
    wst = torch.zeros(s3r.s3r_sample_workspace_bytes(S * (n_t - 1), 0, V), dtype=torch.uint8, device=st.device)
    s3r.s3r_sample_tokens(child_rows.contiguous(), ws.logit_dtype, S * (n_t - 1), V, ws.temperature, u_tok, tok, wst,
                          stream=stream)
    tokens = torch.cat([torch.zeros((S, 1), dtype=torch.int32, device=st.device), tok.view(S, n_t - 1)], 1)
    ua = torch.rand((S, n_t), generator=gen, device=st.device)
    us = torch.rand((S, n_t), generator=gen, device=st.device)
    o_tok = torch.empty((S, n_t), dtype=torch.int32, device=st.device)
    n_acc = torch.empty((S,), dtype=torch.int32, device=st.device)
    path = torch.empty((S, n_t), dtype=torch.int32, device=st.device)
    wss = torch.zeros(s3r.s3r_tree_sample_workspace_bytes(S, n_t, V), dtype=torch.uint8, device=st.device)

    def tree_walk(e0, e1):
        e0.record(stream)
        s3r.s3r_tree_spec_sample(tgt, drf, ws.logit_dtype, tokens, par_d, ua, us, S, n_t, V, ws.temperature, o_tok,
                                 n_acc, path, wss, stream=stream)
        e1.record(stream)

    for _ in range(3):
        tree_walk(torch.cuda.Event(), torch.cuda.Event())
    us_ts = timed(tree_walk, steps)
    na, pa = n_acc.cpu().numpy(), path.cpu().numpy()
    out["tree_spec_sample"] = dict(entry(us_ts, W.tree_sample_bytes(parents, na, pa, V, lelt)),
                                   mean_accepted_nodes=round(float(na.mean()), 3))
    bad = {k: v for k, v in (("tree_attn", s3r.s3r_device_status(wsv)), ("tree_walk", s3r.s3r_device_status(wss)),
                             ("kv", s3r.s3r_device_status(st.ws_kv))) if v[0] != s3r.S3R_OK}
    if bad:
        raise RuntimeError(f"device checks failed in the next-row calls: {bad}")
    return out


def run_ours(a):
    world0 = int(os.environ.get("WORLD_SIZE", "1"))
    # the CPU leg first, before this process touches the GPU
    cpu_line = None
    if not a.no_cpu_baseline and world0 == 1:
        from self_sparse_speculative_b200.workloads import spec as _spec
        cpu_line = cpu_baseline_leg(a, _spec(a.workload))
    import torch
    import torch.distributed as dist
    from self_sparse_speculative_b200.step import DecodeStep
    from self_sparse_speculative_b200.workloads import Workload, spec
    from self_sparse_speculative_b200 import s3r

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    ws = spec(a.workload)
    wl = Workload(ws, seed=a.seed + rank)
    st = DecodeStep(wl, device=f"cuda:{local}")
    stream = torch.cuda.current_stream()
    st.summaries(tail_only=False)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- warm-up
    for _ in range(a.warmup):
        st.round()
    barrier()

    # ---- device-timed steps, with per-phase events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(a.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    # a step that reads less than the 126 MB L2 gets it flushed before every
    # timed step (a 256 MB write outside the timed spans)
    flush = None if st.algorithmic_bytes()["step"] > L2_BYTES else torch.empty(
        FLUSH_BYTES, dtype=torch.uint8, device=f"cuda:{local}")
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(a.steps):
        e = ev[k]
        if flush is not None:
            flush.zero_()
        e[0].record(stream)
        st.draw_draft_tokens()
        e[1].record(stream)
        for i in range(ws.gamma):
            st.draft(i)
        e[2].record(stream)
        st.verify()
        e[3].record(stream)
        st.sample()
        e[4].record(stream)
    end.record(stream)
    barrier()
    total_ms = start.elapsed_time(end) if flush is None else sum(e[0].elapsed_time(e[4]) for e in ev)
    t_draw = sum(e[0].elapsed_time(e[1]) for e in ev) / a.steps
    t_draft = sum(e[1].elapsed_time(e[2]) for e in ev) / a.steps / ws.gamma
    t_verify = sum(e[2].elapsed_time(e[3]) for e in ev) / a.steps
    t_sample = sum(e[3].elapsed_time(e[4]) for e in ev) / a.steps
    # inputs are the same every step, so every step commits the same tokens
    n_acc_total = int(st.num_accepted.sum().item()) * a.steps
    tokens = n_acc_total + ws.num_seqs * a.steps             # (n_acc + 1) per sequence per step
    status = st.device_checks()
    bad = {k: v for k, v in status.items() if v[0] != s3r.S3R_OK}
    if bad:
        raise RuntimeError(f"device checks failed: {bad}")

    total_ms_max, tokens_all = over_ranks(total_ms, tokens, world, f"cuda:{local}")

    # ---- the same round replayed from one captured CUDA graph (one process,
    # steps larger than L2, so back-to-back replays read HBM): device time per
    # replay; reported beside the eager value, which keeps the per-call phases
    graph_info = None
    graph_ms_total = None
    if world == 1 and flush is None and not a.no_graph:
        try:
            graph = st.capture_round()
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            g_s = torch.cuda.Event(enable_timing=True)
            g_e = torch.cuda.Event(enable_timing=True)
            g_s.record(stream)
            for _ in range(a.steps):
                graph.replay()
            g_e.record(stream)
            torch.cuda.synchronize()
            g_total = g_s.elapsed_time(g_e)
            g_ms = g_total / a.steps
            del graph
            gbad = {k: v for k, v in st.device_checks().items() if v[0] != s3r.S3R_OK}
            if gbad:
                raise RuntimeError(f"device checks failed after replays: {gbad}")
            graph_info = {"ms_per_step": round(g_ms, 4), "value": round(tokens / a.steps / (g_ms / 1e3), 1),
                          "unit": UNIT}
            graph_ms_total = g_total
        except Exception as exc:                       # reported, never fatal to the eager line
            graph_info = {"error": f"{type(exc).__name__}: {exc}"[:200]}
    clk = clocks.stop()                               # the sampling spans the eager and the replayed steps
    # the headline: the K replays of the captured round when they ran (the same
    # round and tokens per step, launched as one graph), else the eager steps
    eager_ms_max = total_ms_max
    if graph_ms_total is not None:
        total_ms_max = graph_ms_total

    # ---- end to end: every step's inputs are copied from pinned host memory
    # and its committed tokens read back, through the public API; the upload
    # of step k+1 (copy stream, second input set) overlaps the compute of step k
    e2e = None
    if not a.no_e2e:
        names = ("q_draft", "q_verify", "target_logits", "draft_logits", "u_draft", "u_accept", "u_sample")
        host = {n: getattr(st, n).cpu().pin_memory() for n in names}
        sets = [{n: getattr(st, n) for n in names}, {n: torch.empty_like(getattr(st, n)) for n in names}]
        out_h = torch.empty_like(st.out_tokens, device="cpu").pin_memory()
        nacc_h = torch.empty_like(st.num_accepted, device="cpu").pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = out_h.numel() * 4 + nacc_h.numel() * 4
        cs = torch.cuda.Stream()

        def e2e_steps(k_steps):
            up = [torch.cuda.Event(), torch.cuda.Event()]
            done = [torch.cuda.Event(), torch.cuda.Event()]
            cs.wait_stream(stream)
            with torch.cuda.stream(cs):
                for n in names:
                    sets[0][n].copy_(host[n], non_blocking=True)
                up[0].record(cs)
            for k in range(k_steps):
                if k + 1 < k_steps:
                    with torch.cuda.stream(cs):
                        if k >= 1:
                            cs.wait_event(done[(k + 1) % 2])       # step k-1 has finished with that set
                        for n in names:
                            sets[(k + 1) % 2][n].copy_(host[n], non_blocking=True)
                        up[(k + 1) % 2].record(cs)
                stream.wait_event(up[k % 2])
                for n in names:
                    setattr(st, n, sets[k % 2][n])
                st.round()
                done[k % 2].record(stream)
                out_h.copy_(st.out_tokens, non_blocking=True)
                nacc_h.copy_(st.num_accepted, non_blocking=True)
            for n in names:
                setattr(st, n, sets[0][n])

        e2e_steps(2)
        barrier()
        e_s = torch.cuda.Event(enable_timing=True)
        e_e = torch.cuda.Event(enable_timing=True)
        e_s.record(stream)
        e2e_steps(a.steps)
        e_e.record(stream)
        barrier()
        e2e_ms = e_s.elapsed_time(e_e)
        e2e_tokens = (int(nacc_h.sum().item()) + ws.num_seqs) * a.steps
        e2e_ms, e2e_tokens = over_ranks(e2e_ms, e2e_tokens, world, f"cuda:{local}")
        e2e = {"value": e2e_tokens / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h)}

    peak, peak_kind = _peaks()
    next_rows = None
    if not a.no_next_rows:
        next_rows = next_rows_measure(st, ws, stream, peak, a.steps, a.seed)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    nbytes = st.algorithmic_bytes()
    verify_gbs = nbytes["verify"] / (t_verify * 1e-3) / 1e9
    draft_gbs = nbytes["draft_per_call"] / (t_draft * 1e-3) / 1e9
    ms_per_step = total_ms_max / a.steps
    value = tokens_all / (total_ms_max / 1e3)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "impl": "ours",
        "config": config_of(ws, world, a.seed, nbytes["step"]),
        "roofline": {"bound": "hbm", "kernel": "verify attention (s3r_verify_attn)",
                     "achieved": round(verify_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(verify_gbs / peak, 4), "peak_kind": peak_kind,
                     "traffic": verify_traffic(ws.name),
                     "algorithmic_bytes_per_launch": nbytes["verify"]},
        "phases_ms": {"draft_token_draws": round(t_draw, 4), "sparse_draft_per_call": round(t_draft, 4),
                      "verify": round(t_verify, 4), "spec_sample": round(t_sample, 4)},
        "kv_gbs": {"sparse_draft": round(draft_gbs, 1), "sparse_draft_frac_of_8tbs": round(draft_gbs / 8000, 4),
                   "verify": round(verify_gbs, 1), "verify_frac_of_8tbs": round(verify_gbs / 8000, 4)},
        "acceptance": {"mean_accepted_per_seq": round(n_acc_total / (ws.num_seqs * a.steps), 4),
                       "committed_per_seq": round(tokens / (ws.num_seqs * a.steps), 4)},
        "gpu_launches": launches_per_step(ws, s3r.s3r_sparse_draft_kernels(st.kv, ws.budget_pages)) * a.steps,
        "clocks": clk,
    }
    line["timed"] = "cuda graph replay of the round" if graph_ms_total is not None else "eager launches"
    line["eager"] = {"value": round(tokens_all / (eager_ms_max / 1e3), 1),
                     "ms_per_step": round(eager_ms_max / a.steps, 4)}
    if graph_info is not None:
        line["graph"] = graph_info
    if e2e:
        line["e2e"] = {k: (round(v, 1) if isinstance(v, float) else v) for k, v in e2e.items()}
    line["gamma_policy"] = gamma_policy_note(ws, st, peak)
    if next_rows is not None:
        line["next_rows"] = next_rows
    if cpu_line is not None:
        line["cpu_baseline"] = cpu_line
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- reference arm
def run_reference(a):
    """The oracle as it stands, on the host cores, in the same metric and
    configuration as the GPU arm. Imports nothing that loads the CUDA library."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from self_sparse_speculative_b200.workloads import Workload, algorithmic_bytes, spec
    ws = spec(a.workload)
    step_bytes = algorithmic_bytes(Workload(ws, seed=a.seed))["step"]
    seqs_per_step = min(ws.num_seqs, a.cpu_seqs)
    workers = max(1, min(cpu_cores(), seqs_per_step))
    runner = OracleRunner(workers)
    try:
        runner.step(a.workload, a.seed, [0])                      # warm-up: worker start, imports
        toks, secs = 0, 0.0
        for k in range(a.steps):
            seqs = [(k * seqs_per_step + i) % ws.num_seqs for i in range(seqs_per_step)]
            t, w = runner.step(a.workload, a.seed, seqs)
            toks += t
            secs += w
    finally:
        runner.close()
    value = toks / secs
    seqs = list(range(seqs_per_step))
    line = {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": round(secs / a.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(ws, world, a.seed, step_bytes),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": workers, "kind": "oracle",
                             "sample": oracle_sample_note(ws, seqs, a.steps, workers)},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def launch_plan(gpus, env, argv, port=None):
    """How `bench.py --gpus N` runs: None to run in this process (N = 1, or
    already one rank of an N-rank torchrun launch), else the torchrun command
    that starts N ranks of this same command line. A WORLD_SIZE that
    disagrees with N is an error (SystemExit), so no run can report a GPU
    count it did not use."""
    world = env.get("WORLD_SIZE")
    if world is not None:
        if int(world) != gpus:
            raise SystemExit(f"bench.py: --gpus {gpus} but WORLD_SIZE={world}")
        return None
    if gpus < 1:
        raise SystemExit(f"bench.py: --gpus must be at least 1, got {gpus}")
    if gpus == 1:
        return None
    if port is None:
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.join(HERE, "bench.py")] + list(argv)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seqs", type=int, default=8, help="sequences in the CPU oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the KV-upkeep and tree-verification timings")
    a = ap.parse_args()
    cmd = launch_plan(a.gpus, os.environ, sys.argv[1:])
    if cmd is not None:
        # one process per GPU: relaunch this command line under torchrun
        sys.exit(subprocess.call(cmd))
    if a.impl == "ours":
        a.warmup = max(3, a.warmup)     # at least 3 untimed warm-up steps
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
