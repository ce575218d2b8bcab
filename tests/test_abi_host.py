"""The C ABI without a GPU: the library loads, exports every entry point that
include/s3r.h declares, and rejects bad arguments on the host before any CUDA
call (so these run on a machine without a GPU)."""
import ctypes
import os
import re

import pytest

from self_sparse_speculative_b200 import s3r

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "s3r.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(s3r_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_and_library_exports_every_entry_point():
    names = _declared()
    assert "s3r_verify_attn" in names and len(names) >= 10
    lib = ctypes.CDLL(s3r.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(s3r.EXPORTED)


def test_status_strings_and_version():
    assert s3r.status_str(0) == "S3R_OK"
    assert s3r.status_str(3) == "S3R_ERR_WORKSPACE"
    assert s3r.s3r_version() >= 100


FAKE = 0x10000   # a 16-byte-aligned non-null address; never dereferenced on these paths


def _kv(**kw):
    d = dict(num_seqs=2, num_q_heads=8, num_kv_heads=2, head_dim=128, page_size=64, max_pages_per_seq=4,
             num_pages_total=8, dtype=s3r.S3R_BF16, k_cache=FAKE, v_cache=FAKE, block_table=FAKE,
             context_lens=FAKE)
    d.update(kw)
    kv = s3r.PagedKV()
    for k, v in d.items():
        setattr(kv, k, v)
    return kv


@pytest.mark.parametrize("field,value,status", [
    ("num_seqs", 0, s3r.S3R_ERR_INVALID_ARG),
    ("num_q_heads", 7, s3r.S3R_ERR_INVALID_ARG),       # not a multiple of Hkv
    ("head_dim", 96, s3r.S3R_ERR_UNSUPPORTED),
    ("page_size", 32, s3r.S3R_ERR_UNSUPPORTED),
    ("num_q_heads", 32, s3r.S3R_ERR_UNSUPPORTED),      # G = 16 > 8
    ("max_pages_per_seq", 9000, s3r.S3R_ERR_UNSUPPORTED),
    ("k_cache", 0, s3r.S3R_ERR_INVALID_ARG),
    ("k_cache", FAKE + 4, s3r.S3R_ERR_INVALID_ARG),    # misaligned
    ("dtype", 7, s3r.S3R_ERR_INVALID_ARG),
])
def test_verify_rejects_bad_cache_description(field, value, status):
    kv = _kv(**{field: value})
    lib = s3r.lib()
    st = lib.s3r_verify_attn(ctypes.byref(kv), FAKE, 5, 0.1, FAKE, None, FAKE, 1 << 30, None)
    assert st == status
    assert lib.s3r_attn_workspace_bytes(ctypes.byref(kv), 5, 0) == 0


def test_attention_argument_checks():
    lib = s3r.lib()
    kv = _kv()
    need = lib.s3r_attn_workspace_bytes(ctypes.byref(kv), 5, 0)
    assert need > 0
    # rows * G > 128
    assert lib.s3r_verify_attn(ctypes.byref(kv), FAKE, 33, 0.1, FAKE, None, FAKE, 1 << 30, None) == s3r.S3R_ERR_UNSUPPORTED
    assert lib.s3r_verify_attn(ctypes.byref(kv), FAKE, 0, 0.1, FAKE, None, FAKE, 1 << 30, None) == s3r.S3R_ERR_INVALID_ARG
    assert lib.s3r_verify_attn(ctypes.byref(kv), None, 5, 0.1, FAKE, None, FAKE, 1 << 30, None) == s3r.S3R_ERR_INVALID_ARG
    assert lib.s3r_verify_attn(ctypes.byref(kv), FAKE, 5, float("nan"), FAKE, None, FAKE, 1 << 30, None) == s3r.S3R_ERR_INVALID_ARG
    assert lib.s3r_verify_attn(ctypes.byref(kv), FAKE, 5, 0.1, FAKE, None, FAKE, need - 1, None) == s3r.S3R_ERR_WORKSPACE
    assert lib.s3r_verify_attn(ctypes.byref(kv), FAKE, 5, 0.1, FAKE, None, None, need, None) == s3r.S3R_ERR_WORKSPACE
    need_d = lib.s3r_attn_workspace_bytes(ctypes.byref(kv), 1, 2)
    args = [FAKE, FAKE, FAKE]
    assert lib.s3r_sparse_draft_attn(ctypes.byref(kv), *args, 0, 0.1, FAKE, FAKE, None, FAKE, need_d, None) == s3r.S3R_ERR_INVALID_ARG
    assert lib.s3r_sparse_draft_attn(ctypes.byref(kv), *args, 2, 0.1, None, FAKE, None, FAKE, need_d, None) == s3r.S3R_ERR_INVALID_ARG
    assert lib.s3r_sparse_draft_attn(ctypes.byref(kv), *args, 2, 0.1, FAKE, FAKE, None, FAKE, need_d - 1, None) == s3r.S3R_ERR_WORKSPACE
    assert lib.s3r_page_summaries(None, 0, FAKE, FAKE, None) == s3r.S3R_ERR_INVALID_ARG
    assert lib.s3r_page_summaries(ctypes.byref(kv), 2, FAKE, FAKE, None) == s3r.S3R_ERR_INVALID_ARG


def test_sampling_argument_checks():
    lib = s3r.lib()
    need = lib.s3r_sample_workspace_bytes(4, 3, 1000)
    assert need > 0
    assert lib.s3r_sample_workspace_bytes(0, 3, 1000) == 0
    assert lib.s3r_sample_workspace_bytes(4, 17, 1000) == 0
    call = lambda **kw: lib.s3r_spec_sample(
        kw.get("t", FAKE), FAKE, kw.get("dt", s3r.S3R_BF16), FAKE, FAKE, FAKE, kw.get("S", 4), kw.get("g", 3),
        kw.get("V", 1000), kw.get("T", 1.0), FAKE, FAKE, FAKE, kw.get("wb", need), None)
    assert call(t=None) == s3r.S3R_ERR_INVALID_ARG
    assert call(dt=5) == s3r.S3R_ERR_INVALID_ARG
    assert call(g=0) == s3r.S3R_ERR_INVALID_ARG
    assert call(g=17) == s3r.S3R_ERR_UNSUPPORTED
    assert call(T=0.0) == s3r.S3R_ERR_INVALID_ARG
    assert call(T=float("inf")) == s3r.S3R_ERR_INVALID_ARG
    assert call(V=0) == s3r.S3R_ERR_INVALID_ARG
    # a workspace below what either logit type needs (the size query covers both types,
    # so need - 1 could still suffice for one of them and reach a launch)
    assert call(wb=16) == s3r.S3R_ERR_WORKSPACE
    assert call(wb=16, dt=s3r.S3R_F32) == s3r.S3R_ERR_WORKSPACE
    need_t = lib.s3r_sample_workspace_bytes(8, 0, 1000)
    assert need_t > 0
    assert lib.s3r_sample_tokens(FAKE, s3r.S3R_F32, 8, 1000, 1.0, FAKE, FAKE, FAKE, 16, None) == s3r.S3R_ERR_WORKSPACE
    assert lib.s3r_sample_tokens(FAKE, s3r.S3R_F32, 0, 1000, 1.0, FAKE, FAKE, FAKE, need_t, None) == s3r.S3R_ERR_INVALID_ARG
    assert lib.s3r_device_status(None, None, None) == s3r.S3R_ERR_INVALID_ARG


def test_kv_upkeep_rejects_bad_arguments_on_the_host():
    lib = s3r.lib()
    kv = _kv()
    need = s3r.s3r_kv_workspace_bytes(2)
    assert need > 0 and s3r.s3r_kv_workspace_bytes(0) == 0
    app = lambda **k: lib.s3r_kv_append(ctypes.byref(k.get("kv", kv)), k.get("lens", FAKE), k.get("kn", FAKE), FAKE,
                                        k.get("n", 1), k.get("ow", 0), FAKE, FAKE, FAKE, k.get("wb", need), None)
    # the lengths must be the cache's own (they are updated where the cache reads them)
    assert app(lens=FAKE + 256) == s3r.S3R_ERR_INVALID_ARG
    assert app(n=-1) == s3r.S3R_ERR_INVALID_ARG
    assert app(ow=-2) == s3r.S3R_ERR_INVALID_ARG
    assert app(n=2000) == s3r.S3R_ERR_INVALID_ARG
    assert app(kn=FAKE + 8) == s3r.S3R_ERR_INVALID_ARG              # rows not 16-byte aligned
    assert app(wb=need - 1) == s3r.S3R_ERR_WORKSPACE
    assert app(kv=_kv(head_dim=96)) == s3r.S3R_ERR_UNSUPPORTED
    assert app(n=0, ow=0) == s3r.S3R_OK                              # nothing to do, nothing enqueued
    rb = lambda **k: lib.s3r_kv_rollback(ctypes.byref(kv), k.get("lens", FAKE), k.get("nacc", FAKE), k.get("rows", 5),
                                         FAKE, FAKE, FAKE, k.get("wb", need), None)
    assert rb(rows=0) == s3r.S3R_ERR_INVALID_ARG
    assert rb(rows=18) == s3r.S3R_ERR_INVALID_ARG
    assert rb(nacc=0) == s3r.S3R_ERR_INVALID_ARG
    assert rb(lens=FAKE + 4) == s3r.S3R_ERR_INVALID_ARG
    assert rb(wb=8) == s3r.S3R_ERR_WORKSPACE
