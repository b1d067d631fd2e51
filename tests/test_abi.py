"""The C ABI: the library loads, exports every symbol include/flashblock.h
declares, and its host-side argument checks answer without a GPU (CPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flashblock.h")


def _built():
    from cached_split_attention_b200 import build
    return build.build()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fb_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fb_out_attn", "fb_in_attn", "fb_merge", "fb_step", "fb_head_similarity", "fb_cache_invalidate",
              "fb_workspace_size", "fb_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_built())
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def _problem(B, **kw):
    args = dict(num_seqs=1, num_heads_q=32, num_heads_kv=32, head_dim=128, softmax_scale=0.088,
                cu_seqlens_q=16, q_rows=0, cu_seqlens_kv_out=16, cu_seqlens_kv_in=16, total_q=32,
                total_kv_out=4096, total_kv_in=32, max_q=32, max_kv_out=4096, max_kv_in=32, out_splits=0)
    args.update(kw)
    return B.FbProblem(**args)


def test_host_validation_without_gpu():
    _built()
    from cached_split_attention_b200 import binding as B
    n = ctypes.c_size_t()
    ok = _problem(B)
    assert B._lib.fb_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == B.OK and n.value > 0
    cases = [
        (dict(head_dim=96), B.ERR_UNSUPPORTED, "head_dim"),
        (dict(num_heads_q=12, num_heads_kv=8), B.ERR_UNSUPPORTED, "multiple"),
        (dict(num_heads_q=66, num_heads_kv=1), B.ERR_UNSUPPORTED, "query heads"),
        (dict(max_q=64), B.ERR_INVALID_ARG, "exceeds"),
        (dict(total_q=-1), B.ERR_INVALID_ARG, "negative"),
        (dict(softmax_scale=0.0), B.ERR_INVALID_ARG, "softmax_scale"),
        (dict(cu_seqlens_q=0), B.ERR_INVALID_ARG, "cu_seqlens"),
        (dict(out_splits=-2), B.ERR_INVALID_ARG, "out_splits"),
    ]
    for kw, code, word in cases:
        bad = _problem(B, **kw)
        assert B._lib.fb_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == code, kw
        assert word in B.last_error(), (kw, B.last_error())
    # pointer checks of the compute calls fail before any CUDA call
    assert B._lib.fb_in_attn(ctypes.byref(ok), None, 16, 16, 16, 16, None) == B.ERR_INVALID_ARG
    assert "q is NULL" in B.last_error()
    assert B._lib.fb_in_attn(ctypes.byref(ok), 24, 16, 16, 16, 16, None) == B.ERR_INVALID_ARG
    assert "aligned" in B.last_error()
    prm = B.params(4, 0.0, B.FORCE_RECOMPUTE | B.FORCE_REUSE)
    cache = B.FbCache(16, 16, 16, 0)
    rc = B._lib.fb_step(ctypes.byref(ok), ctypes.byref(prm), ctypes.byref(cache), 16, 16, 16, 16, 16, 16, None,
                        16, 16, None, 16, 1 << 30, None)
    assert rc == B.ERR_INVALID_ARG and "exclusive" in B.last_error()
    prm = B.params(4, 0.0, B.GATE_TAU)
    rc = B._lib.fb_step(ctypes.byref(ok), ctypes.byref(prm), ctypes.byref(cache), 16, 16, 16, 16, 16, None, None,
                        16, 16, None, 16, 1 << 30, None)
    assert rc == B.ERR_INVALID_ARG and "n_updated" in B.last_error()
    # the cumulative gate: exclusive with the per-step one, needs the count array
    prm = B.params(4, 0.0, B.GATE_TAU | B.GATE_TAU_CUM)
    rc = B._lib.fb_step(ctypes.byref(ok), ctypes.byref(prm), ctypes.byref(cache), 16, 16, 16, 16, 16, 16, None,
                        16, 16, None, 16, 1 << 30, None)
    assert rc == B.ERR_INVALID_ARG and "exclusive" in B.last_error()
    prm = B.params(4, 0.0, B.GATE_TAU_CUM)
    rc = B._lib.fb_step(ctypes.byref(ok), ctypes.byref(prm), ctypes.byref(cache), 16, 16, 16, 16, 16, 16, None,
                        16, 16, None, 16, 1 << 30, None)
    assert rc == B.ERR_INVALID_ARG and "m_acc" in B.last_error()
    prm = B.params(4, 0.0, 32)
    rc = B._lib.fb_step(ctypes.byref(ok), ctypes.byref(prm), ctypes.byref(cache), 16, 16, 16, 16, 16, 16, None,
                        16, 16, None, 16, 1 << 30, None)
    assert rc == B.ERR_INVALID_ARG and "unknown flag" in B.last_error()
    assert B._lib.fb_merge(-1, 4, 16, 16, 16, 16, 16, None, None, None) == B.ERR_INVALID_ARG
    # branch hooks and the sparse layout: argument checks before any device work
    cache5 = B.FbCache(16, 16, 16, 0, 0)
    assert B._lib.fb_cache_copy_seq(ctypes.byref(ok), ctypes.byref(cache5), 0, 3, None) == B.ERR_INVALID_ARG
    assert "out of range" in B.last_error()
    assert B._lib.fb_cache_copy_seq(ctypes.byref(ok), ctypes.byref(cache5), 0, 0, None) == B.OK  # no-op
    rc = B._lib.fb_sparse_layout(ctypes.byref(ok), 16, 16, 5000, 16, 16, 16, 16, 16, 16, 16, 16, None, None, None)
    assert rc == B.ERR_INVALID_ARG and "total_sel" in B.last_error()
    rc = B._lib.fb_sparse_layout(ctypes.byref(ok), None, 16, 4, 16, 16, 16, 16, 16, 16, 16, 16, None, None, None)
    assert rc == B.ERR_INVALID_ARG and "cu_sel" in B.last_error()


def test_workspace_size_is_counter_plus_scores():
    """The workspace holds a completion counter (256-byte slot) and one fp32
    similarity score per (sequence, q-head); partials stay on chip."""
    _built()
    from cached_split_attention_b200 import binding as B
    for seqs, hq, expect in [(1, 32, 256 + 256), (8, 32, 256 + 1024), (3, 40, 256 + 512)]:
        n = ctypes.c_size_t()
        prob = _problem(B, num_seqs=seqs, num_heads_q=hq, num_heads_kv=hq, out_splits=4)
        assert B._lib.fb_workspace_size(ctypes.byref(prob), ctypes.byref(n)) == B.OK
        assert n.value == expect, (seqs, hq, n.value)
    # a multi-head problem of 256+ rows per head may take the two-tile kernel: its
    # work order (one int32 per (sequence, head, 256-row pair)) follows
    n = ctypes.c_size_t()
    prob = _problem(B, num_heads_q=40, num_heads_kv=40, total_q=1560, max_q=1560, total_kv_in=1560,
                    max_kv_in=1560)
    assert B._lib.fb_workspace_size(ctypes.byref(prob), ctypes.byref(n)) == B.OK
    assert n.value == 256 + 256 + 1280, n.value  # 40 x 7 items x 4 bytes = 1120 -> 1280
