"""ctypes binding of libs3r (include/s3r.h): argument marshalling only.

Each function has the name of the C entry point it calls and takes torch
tensors (device memory) or raw device addresses; every step of the computation
runs in the library's CUDA kernels. A non-OK status raises S3RError. The
library must have been built (``python -m self_sparse_speculative_b200.build``);
if it is missing, importing this module raises ImportError - there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libs3r.so")

S3R_OK, S3R_ERR_INVALID_ARG, S3R_ERR_UNSUPPORTED, S3R_ERR_WORKSPACE, S3R_ERR_CUDA, S3R_ERR_DEVICE_CHECK = range(6)
S3R_F32, S3R_BF16 = 0, 1
S3R_DEV_BAD_CONTEXT_LEN, S3R_DEV_BAD_PAGE_ID, S3R_DEV_BAD_TOKEN_ID, S3R_DEV_WAIT_TIMEOUT = 0x1, 0x2, 0x4, 0x8
S3R_DEV_BAD_TREE = 0x10

EXPORTED = [
    "s3r_page_summaries", "s3r_page_summaries_checked", "s3r_sparse_draft_attn", "s3r_verify_attn",
    "s3r_spec_sample", "s3r_spec_sample_noalloc", "s3r_sample_tokens", "s3r_attn_workspace_bytes", "s3r_sample_workspace_bytes",
    "s3r_device_status", "s3r_status_str", "s3r_version", "s3r_sparse_draft_kernels",
    "s3r_sample_tokens_ex", "s3r_spec_sample_ex", "s3r_kv_append", "s3r_kv_rollback", "s3r_kv_workspace_bytes",
    "s3r_debug_exp64", "s3r_gamma_policy_init", "s3r_gamma_policy_update", "s3r_gamma_policy_choose",
    "s3r_attend_cost_us", "s3r_round_cost_us", "s3r_verify_attn_tree", "s3r_tree_spec_sample",
    "s3r_tree_sample_workspace_bytes", "s3r_tree_node_budget",
]


class S3RError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_str(status)}")


class GammaPolicy(ctypes.Structure):
    _fields_ = [("gamma_max", ctypes.c_int32), ("decay", ctypes.c_double), ("accepted", ctypes.c_double),
                ("tested", ctypes.c_double), ("cost_us", ctypes.c_double * 17)]


class PagedKV(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
        ("num_pages_total", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("context_lens", ctypes.c_void_p),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libs3r.so is not built ({LIB_PATH}); run python -m self_sparse_speculative_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t, ctypes.c_double
    kvp = ctypes.POINTER(PagedKV)
    sig = {
        "s3r_page_summaries": ([kvp, i32, vp, vp, vp], i32),
        "s3r_page_summaries_checked": ([kvp, i32, vp, vp, vp, vp], i32),
        "s3r_sparse_draft_attn": ([kvp, vp, vp, vp, i32, f32, vp, vp, vp, vp, sz, vp], i32),
        "s3r_verify_attn": ([kvp, vp, i32, f32, vp, vp, vp, sz, vp], i32),
        "s3r_spec_sample": ([vp, vp, i32, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp, sz, vp], i32),
        "s3r_spec_sample_noalloc": ([vp, vp, i32, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp], i32),
        "s3r_sample_tokens": ([vp, i32, i32, i32, f32, vp, vp, vp, sz, vp], i32),
        "s3r_sample_tokens_ex": ([vp, i32, i32, i32, f32, vp, vp, vp, vp, sz, vp], i32),
        "s3r_spec_sample_ex": ([vp, vp, i32, vp, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp, sz, vp], i32),
        "s3r_kv_append": ([kvp, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp], i32),
        "s3r_kv_rollback": ([kvp, vp, vp, i32, vp, vp, vp, sz, vp], i32),
        "s3r_kv_workspace_bytes": ([i32], sz),
        "s3r_debug_exp64": ([vp, vp, vp, i32, vp], i32),
        "s3r_gamma_policy_init": ([ctypes.POINTER(GammaPolicy), i32, f64, f64, f64, ctypes.POINTER(f64)], i32),
        "s3r_gamma_policy_update": ([ctypes.POINTER(GammaPolicy), ctypes.POINTER(i32), i32, i32], i32),
        "s3r_gamma_policy_choose": ([ctypes.POINTER(GammaPolicy), ctypes.POINTER(i32), ctypes.POINTER(f64),
                                     ctypes.POINTER(f64)], i32),
        "s3r_attend_cost_us": ([i32, i32, i32, i32, i32, f64, i32, f64, f64], f64),
        "s3r_round_cost_us": ([i32, i32, i32, i32, i32, i32, f64, i32, i32, i32, i32, f64, f64], f64),
        "s3r_attn_workspace_bytes": ([kvp, i32, i32], sz),
        "s3r_sample_workspace_bytes": ([i32, i32, i32], sz),
        "s3r_device_status": ([vp, ctypes.POINTER(ctypes.c_uint32), vp], i32),
        "s3r_status_str": ([i32], ctypes.c_char_p),
        "s3r_sparse_draft_kernels": ([kvp, i32], i32),
        "s3r_version": ([], i32),
        "s3r_verify_attn_tree": ([kvp, vp, i32, vp, f32, vp, vp, vp, sz, vp], i32),
        "s3r_tree_sample_workspace_bytes": ([i32, i32, i32], sz),
        "s3r_tree_spec_sample": ([vp, vp, i32, vp, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp, vp, sz, vp], i32),
        "s3r_tree_node_budget": ([ctypes.c_int64, i32, i32, i32], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()


def lib():
    return _lib


def status_str(status: int) -> str:
    return _lib.s3r_status_str(int(status)).decode()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, st):
    if st != S3R_OK:
        raise S3RError(fn, st)


def dtype_code(dt) -> int:
    import torch
    if dt in (torch.bfloat16, "bf16", S3R_BF16):
        return S3R_BF16
    if dt in (torch.float32, "f32", S3R_F32):
        return S3R_F32
    raise ValueError(f"unsupported dtype {dt}")


def paged_kv(k_cache, v_cache, block_table, context_lens, num_q_heads: int) -> PagedKV:
    """Describe a cache [num_pages_total, Hkv, P, D] with its block table."""
    n, h, p, d = k_cache.shape
    return PagedKV(int(block_table.shape[0]), int(num_q_heads), int(h), int(d), int(p),
                   int(block_table.shape[1]), int(n), dtype_code(k_cache.dtype),
                   _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(context_lens))


def s3r_attn_workspace_bytes(kv: PagedKV, rows: int, budget_pages: int) -> int:
    return int(_lib.s3r_attn_workspace_bytes(ctypes.byref(kv), rows, budget_pages))


def s3r_sample_workspace_bytes(num_seqs: int, gamma: int, vocab: int) -> int:
    return int(_lib.s3r_sample_workspace_bytes(num_seqs, gamma, vocab))


def s3r_page_summaries(kv: PagedKV, tail_only: int, kmin, kmax, stream=None, status_word=None):
    if status_word is None:
        st = _lib.s3r_page_summaries(ctypes.byref(kv), int(tail_only), _ptr(kmin), _ptr(kmax), _stream(stream))
    else:
        st = _lib.s3r_page_summaries_checked(ctypes.byref(kv), int(tail_only), _ptr(kmin), _ptr(kmax),
                                             _ptr(status_word), _stream(stream))
    _check("s3r_page_summaries", st)


def s3r_sparse_draft_attn(kv: PagedKV, kmin, kmax, q, budget_pages: int, scale: float, selected, out,
                          lse, workspace, workspace_bytes=None, stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = _lib.s3r_sparse_draft_attn(ctypes.byref(kv), _ptr(kmin), _ptr(kmax), _ptr(q), int(budget_pages),
                                    float(scale), _ptr(selected), _ptr(out), _ptr(lse), _ptr(workspace), wb,
                                    _stream(stream))
    _check("s3r_sparse_draft_attn", st)


def s3r_verify_attn(kv: PagedKV, q, rows: int, scale: float, out, lse, workspace, workspace_bytes=None,
                    stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = _lib.s3r_verify_attn(ctypes.byref(kv), _ptr(q), int(rows), float(scale), _ptr(out), _ptr(lse),
                              _ptr(workspace), wb, _stream(stream))
    _check("s3r_verify_attn", st)


def s3r_verify_attn_tree(kv: PagedKV, q, nodes: int, parents, scale: float, out, lse, workspace,
                         workspace_bytes=None, stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = _lib.s3r_verify_attn_tree(ctypes.byref(kv), _ptr(q), int(nodes), _ptr(parents), float(scale), _ptr(out),
                                   _ptr(lse), _ptr(workspace), wb, _stream(stream))
    _check("s3r_verify_attn_tree", st)


def s3r_tree_sample_workspace_bytes(num_seqs: int, nodes: int, vocab: int) -> int:
    return int(_lib.s3r_tree_sample_workspace_bytes(num_seqs, nodes, vocab))


def s3r_tree_spec_sample(target_logits, draft_logits, logit_dtype, tokens, parents, u_accept, u_sample,
                         num_seqs: int, nodes: int, vocab: int, temperature: float, out_tokens, num_accepted,
                         path, workspace, workspace_bytes=None, stream=None):
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = _lib.s3r_tree_spec_sample(_ptr(target_logits), _ptr(draft_logits), dtype_code(logit_dtype), _ptr(tokens),
                                   _ptr(parents), _ptr(u_accept), _ptr(u_sample), int(num_seqs), int(nodes),
                                   int(vocab), float(temperature), _ptr(out_tokens), _ptr(num_accepted), _ptr(path),
                                   _ptr(workspace), wb, _stream(stream))
    _check("s3r_tree_spec_sample", st)


def s3r_tree_node_budget(capacity: int, active: int, n_min: int, n_max: int) -> int:
    """N_t = clip(floor(capacity / active), n_min, n_max); -1 for bad arguments."""
    return int(_lib.s3r_tree_node_budget(int(capacity), int(active), int(n_min), int(n_max)))


def s3r_spec_sample(target_logits, draft_logits, logit_dtype, draft_tokens, u_accept, u_sample,
                    num_seqs: int, gamma: int, vocab: int, temperature: float, out_tokens, num_accepted,
                    workspace, workspace_bytes=None, stream=None, draft_stats=None):
    """draft_stats (float64 [S, gamma, 2] from s3r_sample_tokens(..., row_stats=...)) selects
    s3r_spec_sample_ex."""
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    if draft_stats is None:
        st = _lib.s3r_spec_sample(_ptr(target_logits), _ptr(draft_logits), dtype_code(logit_dtype),
                                  _ptr(draft_tokens), _ptr(u_accept), _ptr(u_sample), int(num_seqs), int(gamma),
                                  int(vocab), float(temperature), _ptr(out_tokens), _ptr(num_accepted),
                                  _ptr(workspace), wb, _stream(stream))
        _check("s3r_spec_sample", st)
        return
    st = _lib.s3r_spec_sample_ex(_ptr(target_logits), _ptr(draft_logits), dtype_code(logit_dtype),
                                 _ptr(draft_tokens), _ptr(u_accept), _ptr(u_sample), _ptr(draft_stats),
                                 int(num_seqs), int(gamma), int(vocab), float(temperature), _ptr(out_tokens),
                                 _ptr(num_accepted), _ptr(workspace), wb, _stream(stream))
    _check("s3r_spec_sample_ex", st)


def s3r_spec_sample_noalloc(target_logits, draft_logits, logit_dtype, draft_tokens, u_accept, u_sample,
                            num_seqs: int, gamma: int, vocab: int, temperature: float, out_tokens,
                            num_accepted, stream=None):
    """s3r_spec_sample with the library's own static device scratch instead of a workspace
    (for callers that cannot allocate device memory; calls must not overlap on the GPU)."""
    st = _lib.s3r_spec_sample_noalloc(_ptr(target_logits), _ptr(draft_logits), dtype_code(logit_dtype),
                                      _ptr(draft_tokens), _ptr(u_accept), _ptr(u_sample), int(num_seqs),
                                      int(gamma), int(vocab), float(temperature), _ptr(out_tokens),
                                      _ptr(num_accepted), _stream(stream))
    _check("s3r_spec_sample_noalloc", st)


def s3r_sample_tokens(logits, logit_dtype, num_rows: int, vocab: int, temperature: float, u, tokens,
                      workspace, workspace_bytes=None, stream=None, row_stats=None):
    """row_stats (float64 [num_rows, 2]) selects s3r_sample_tokens_ex, which also writes each
    row's {max, exact Z}."""
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    if row_stats is None:
        st = _lib.s3r_sample_tokens(_ptr(logits), dtype_code(logit_dtype), int(num_rows), int(vocab),
                                    float(temperature), _ptr(u), _ptr(tokens), _ptr(workspace), wb,
                                    _stream(stream))
        _check("s3r_sample_tokens", st)
        return
    st = _lib.s3r_sample_tokens_ex(_ptr(logits), dtype_code(logit_dtype), int(num_rows), int(vocab),
                                   float(temperature), _ptr(u), _ptr(tokens), _ptr(row_stats), _ptr(workspace),
                                   wb, _stream(stream))
    _check("s3r_sample_tokens_ex", st)


def s3r_device_status(workspace, stream=None):
    """(status, bits) of the most recent call that used `workspace` (synchronises)."""
    bits = ctypes.c_uint32(0)
    st = _lib.s3r_device_status(_ptr(workspace), ctypes.byref(bits), _stream(stream))
    return int(st), int(bits.value)


def s3r_sparse_draft_kernels(kv: PagedKV, budget_pages: int) -> int:
    """Kernels one s3r_sparse_draft_attn call launches (1 fused, 2 select + attention)."""
    return int(_lib.s3r_sparse_draft_kernels(ctypes.byref(kv), int(budget_pages)))


def s3r_kv_workspace_bytes(num_seqs: int) -> int:
    return int(_lib.s3r_kv_workspace_bytes(int(num_seqs)))


def s3r_kv_append(kv: PagedKV, context_lens, k_new, v_new, n: int, overwrite: int, kmin, kmax, workspace,
                  workspace_bytes=None, stream=None):
    """Write n rows per sequence at L - overwrite.. (updating L and the touched pages' summaries)."""
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = _lib.s3r_kv_append(ctypes.byref(kv), _ptr(context_lens), _ptr(k_new), _ptr(v_new), int(n),
                            int(overwrite), _ptr(kmin), _ptr(kmax), _ptr(workspace), wb, _stream(stream))
    _check("s3r_kv_append", st)


def s3r_kv_rollback(kv: PagedKV, context_lens, num_accepted, rows: int, kmin, kmax, workspace,
                    workspace_bytes=None, stream=None):
    """L <- L - rows + n_acc + 1, and the new tail page's summary."""
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = _lib.s3r_kv_rollback(ctypes.byref(kv), _ptr(context_lens), _ptr(num_accepted), int(rows), _ptr(kmin),
                              _ptr(kmax), _ptr(workspace), wb, _stream(stream))
    _check("s3r_kv_rollback", st)


def s3r_debug_exp64(x, y_tbl, y_ref, stream=None):
    """The sampler's float64 exponential of x (y_tbl) and CUDA's exp (y_ref), float64 device tensors."""
    st = _lib.s3r_debug_exp64(_ptr(x), _ptr(y_tbl), _ptr(y_ref), int(x.numel()), _stream(stream))
    _check("s3r_debug_exp64", st)


class GammaPolicyHandle:
    """The library's draft-length policy (host code): init, update with a round's
    acceptance counts, choose the next gamma (0: drafting off)."""

    def __init__(self, gamma_max: int, decay: float, prior_accept: float, prior_weight: float, cost_us):
        self.p = GammaPolicy()
        c = (ctypes.c_double * 17)(*[float(x) for x in cost_us])
        _check("s3r_gamma_policy_init", _lib.s3r_gamma_policy_init(ctypes.byref(self.p), int(gamma_max),
                                                                   float(decay), float(prior_accept),
                                                                   float(prior_weight), c))

    def update(self, num_accepted, gamma_used: int):
        n = [int(x) for x in num_accepted]
        arr = (ctypes.c_int32 * len(n))(*n)
        _check("s3r_gamma_policy_update", _lib.s3r_gamma_policy_update(ctypes.byref(self.p), arr, len(n),
                                                                       int(gamma_used)))

    def choose(self):
        """(gamma, alpha, rate)."""
        g, a, r = ctypes.c_int32(0), ctypes.c_double(0), ctypes.c_double(0)
        _check("s3r_gamma_policy_choose", _lib.s3r_gamma_policy_choose(ctypes.byref(self.p), ctypes.byref(g),
                                                                       ctypes.byref(a), ctypes.byref(r)))
        return int(g.value), float(a.value), float(r.value)


def s3r_attend_cost_us(*args) -> float:
    return float(_lib.s3r_attend_cost_us(*args))


def s3r_round_cost_us(*args) -> float:
    return float(_lib.s3r_round_cost_us(*args))


def s3r_version() -> int:
    return int(_lib.s3r_version())
