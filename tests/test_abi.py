"""The C ABI: the library loads, exports every symbol include/flashblock.h
declares, and its host-side argument checks answer without a GPU (CPU)."""
import ctypes
import os
import re

import numpy as np
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
                total_kv_out=4096, total_kv_in=32, max_q=32, max_kv_out=4096, max_kv_in=32, out_splits=0,
                kv_out_skip=None)
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
    assert B._lib.fb_merge(2 ** 62, 4, 16, 16, 16, 16, 16, None, None, None) == B.ERR_INVALID_ARG
    assert "overflows" in B.last_error()
    # branch hooks and the sparse layout: argument checks before any device work
    cache5 = B.FbCache(16, 16, 16, 0, 0)
    assert B._lib.fb_cache_copy_seq(ctypes.byref(ok), ctypes.byref(cache5), 0, 3, None) == B.ERR_INVALID_ARG
    assert "out of range" in B.last_error()
    assert B._lib.fb_cache_copy_seq(ctypes.byref(ok), ctypes.byref(cache5), 0, 0, None) == B.OK  # no-op
    rc = B._lib.fb_sparse_layout(ctypes.byref(ok), 16, 16, 5000, 16, 16, 16, 16, 16, 16, 16, None, None)
    assert rc == B.ERR_INVALID_ARG and "total_sel" in B.last_error()
    rc = B._lib.fb_sparse_layout(ctypes.byref(ok), None, 16, 4, 16, 16, 16, 16, 16, 16, 16, None, None)
    assert rc == B.ERR_INVALID_ARG and "cu_sel" in B.last_error()
    many = _problem(B, num_seqs=70000, total_q=0, max_q=0, total_kv_in=0, max_kv_in=0, total_kv_out=0, max_kv_out=0)
    rc = B._lib.fb_sparse_layout(ctypes.byref(many), 16, 16, 0, 16, 16, 16, 16, 16, 16, 16, None, None)
    assert rc == B.ERR_UNSUPPORTED and "65535" in B.last_error()
    rc = B._lib.fb_sparse_layout(ctypes.byref(ok), 16, 16, 4, 16, 16, 16, 16, 16, 16, None, None, None)
    assert rc == B.ERR_INVALID_ARG and "kv_out_skip" in B.last_error()
    rc = B._lib.fb_sparse_layout(ctypes.byref(ok), 16, 16, 4, 16, 16, 16, 16, 16, 16, 18, None, None)
    assert rc == B.ERR_INVALID_ARG and "aligned" in B.last_error()
    skewed = _problem(B, kv_out_skip=18)
    assert B._lib.fb_workspace_size(ctypes.byref(skewed), ctypes.byref(n)) == B.ERR_INVALID_ARG
    assert "kv_out_skip" in B.last_error()
    # block transition: in place only for one sequence, K and V alike
    two = _problem(B, num_seqs=2)
    rc = B._lib.fb_prefix_append(ctypes.byref(two), 16, 32, 48, 64, 16, 32, None, None)
    assert rc == B.ERR_UNSUPPORTED and "in-place" in B.last_error()
    rc = B._lib.fb_prefix_append(ctypes.byref(ok), 16, 32, 48, 64, 16, 80, None, None)
    assert rc == B.ERR_INVALID_ARG and "both" in B.last_error()
    rc = B._lib.fb_prefix_append(ctypes.byref(ok), 16, 32, 48, 64, None, 80, None, None)
    assert rc == B.ERR_INVALID_ARG and "k_dst" in B.last_error()


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


def _shape_problems():
    """The step-0 problems of the bench workloads (shapes only; no K/V drawn)."""
    from cached_split_attention_b200.workloads import make_problem
    rng = np.random.default_rng(0)
    return {
        "dllm_layer": make_problem([np.arange(32)], [4096], [32], 32, 32, 128),
        "tiny": make_problem([np.arange(32)], [256], [32], 4, 4, 64),
        "long_context_gqa": make_problem([np.sort(rng.permutation(64)[:32]) for _ in range(8)], [32768] * 8,
                                         [64] * 8, 32, 8, 128),
        "varlen_branches": make_problem([np.arange(b) for b in (4, 8, 16, 32, 64, 128)], [2048] * 6,
                                        [4, 8, 16, 32, 64, 128], 32, 32, 128),
        "video": make_problem([np.arange(1560)], [9360], [1560], 40, 40, 128),
    }


def test_plan_query_matches_the_bench_kernel_map():
    """fb_plan_query on the CPU: the fused step of each bench workload takes the
    kernel bench.py attributes its roofline and counters to; the grid is items x
    splits; the two-tile kernel and the block-only pass never split the prefix; the
    warp-MMA kernel's split grid fits one wave."""
    _built()
    import bench
    from cached_split_attention_b200 import binding as B
    for name, p in _shape_problems().items():
        dp = B.DeviceProblem(p, "cpu")
        step = B.plan_query(dp, B.CALL_STEP)
        assert step["kernel_name"] == bench.KERNEL_OF[name], (name, step)
        for call in (B.CALL_STEP, B.CALL_OUT, B.CALL_IN):
            pl = B.plan_query(dp, call)
            assert pl["ctas"] == pl["work_items"] * pl["splits"] > 0, (name, call, pl)
            assert 1 <= pl["splits"] <= 16
            if call == B.CALL_IN or pl["kernel"] == 2:
                assert pl["splits"] == 1, (name, call, pl)
            if pl["kernel"] == 0 and call != B.CALL_IN and pl["splits"] > 1:
                per_sm = max(1, min(233472 // (pl["smem_bytes"] + 1024), 2048 // pl["threads"]))
                assert pl["ctas"] <= pl["num_sms"] * per_sm, (name, pl)
        # the unfused prefix pass never takes the two-tile kernel (that is fb_step's)
        assert B.plan_query(dp, B.CALL_OUT)["kernel"] != 2
    video = B.plan_query(B.DeviceProblem(_shape_problems()["video"], "cpu"))
    assert (video["rows_per_tile"], video["tiles"], video["work_items"]) == (128, 13, 40 * 7)
    dllm = B.plan_query(B.DeviceProblem(_shape_problems()["dllm_layer"], "cpu"))
    assert (dllm["rows_per_tile"], dllm["tiles"], dllm["work_items"]) == (32, 1, 32)
    gqa = B.plan_query(B.DeviceProblem(_shape_problems()["long_context_gqa"], "cpu"))
    assert (gqa["rows_per_tile"], gqa["tiles"], gqa["work_items"]) == (128, 1, 64)


def test_plan_query_lean_reuse_path():
    """The lean reuse path: planned for fused steps of blocks of at most 128 keys
    (every bench workload but the 1560-token video block), never for the unfused
    passes, and only when the kernel's shared memory holds what it needs.  Its loads
    start before the reuse decision only when the whole grid is resident at once
    (one CTA per SM here: at most num_sms CTAs), so not for the 192-CTA varlen grid."""
    _built()
    from cached_split_attention_b200 import binding as B
    for name, p in _shape_problems().items():
        dp = B.DeviceProblem(p, "cpu")
        step = B.plan_query(dp, B.CALL_STEP)
        assert step["lean_reuse"] == (0 if name == "video" else 1), (name, step)
        if step["lean_reuse"]:
            assert 0 < step["lean_smem_bytes"] <= step["smem_bytes"], (name, step)
            one_wave = step["ctas"] <= step["num_sms"] * max(1, 233472 // (step["smem_bytes"] + 1024))
            assert step["lean_early"] == int(one_wave), (name, step)
        else:
            assert step["lean_early"] == 0
        for call in (B.CALL_OUT, B.CALL_IN):
            info = B.plan_query(dp, call)
            assert info["lean_reuse"] == 0 and info["lean_early"] == 0
    early = {n: B.plan_query(B.DeviceProblem(p, "cpu"))["lean_early"] for n, p in _shape_problems().items()}
    assert early["long_context_gqa"] == 1 and early["dllm_layer"] == 1 and early["varlen_branches"] == 0


def test_plan_query_tensor_core_threads_per_row():
    """The tensor-core kernel runs one softmax thread per tile row in a grid that one
    wave holds (192 threads) and two per row beyond it (320 threads): the long-context
    GQA batch is one wave of 128 CTAs, the varlen branches 192 CTAs."""
    _built()
    from cached_split_attention_b200 import binding as B
    probs = _shape_problems()
    gqa = B.plan_query(B.DeviceProblem(probs["long_context_gqa"], "cpu"))
    var = B.plan_query(B.DeviceProblem(probs["varlen_branches"], "cpu"))
    assert gqa["kernel_name"] == var["kernel_name"] == "tc_attn_kernel"
    assert gqa["ctas"] <= gqa["num_sms"] and gqa["threads"] == 192
    assert var["ctas"] > var["num_sms"] and var["threads"] == 320


def test_plan_query_reaches_the_variants_the_gpu_tests_name():
    """The reduced shapes of the GPU tests reach the launch variants those tests are
    named for (so that a change of the host plan shows up here, without a GPU): the
    largest portable cluster on both streaming kernels, the largest group (32 q-heads
    per kv-head) on both, the two-tile kernel with one-row and empty sequences, and
    the warp-MMA kernel for a call whose rows are all locked."""
    _built()
    from cached_split_attention_b200 import binding as B
    from cached_split_attention_b200 import workloads as W
    mk = W.make_problem
    none = np.zeros(0, np.int64)
    cases = [
        # (problem, kernel, threads, splits or None)
        (W.dllm_layer(steps=1, prefix=2000, heads=8).problem, "attn_kernel", 256, 8),
        (W.dllm_layer(steps=1, prefix=2000, heads=8, head_dim=64).problem, "attn_kernel", 256, 8),
        (W.long_context_gqa(steps=1, batch=1, prefix=2085).problem, "tc_attn_kernel", 192, 8),
        (mk([np.arange(29), np.arange(40)], [150, 150], [64, 47], 64, 2, 128), "tc_attn_kernel", 192, None),
        (mk([np.array([1, 6]), np.array([0, 3])], [150, 150], [8, 5], 64, 2, 128), "attn_kernel", 256, None),
        (mk([np.arange(300), np.array([7]), none], [200] * 3, [300, 40, 24], 2, 2, 128), "tc2_attn_kernel", 320, 1),
        (mk([none, none], [150, 150], [32, 64], 8, 2, 128), "attn_kernel", 128, None),
        (W.varlen_branches(steps=1, prefix=337).problem, "tc_attn_kernel", 320, None),
    ]
    for p, kernel, threads, splits in cases:
        info = B.plan_query(B.DeviceProblem(p, "cpu"))
        assert (info["kernel_name"], info["threads"]) == (kernel, threads), info
        if splits is not None:
            assert info["splits"] == splits, info


def test_plan_query_rejects_bad_arguments():
    _built()
    from cached_split_attention_b200 import binding as B
    ok = _problem(B)
    info = B.FbPlanInfo()
    assert B._lib.fb_plan_query(ctypes.byref(ok), 3, ctypes.byref(info)) == B.ERR_INVALID_ARG
    assert "unknown call" in B.last_error()
    assert B._lib.fb_plan_query(ctypes.byref(ok), 0, None) == B.ERR_INVALID_ARG
    bad = _problem(B, head_dim=96)
    assert B._lib.fb_plan_query(ctypes.byref(bad), 0, ctypes.byref(info)) == B.ERR_UNSUPPORTED


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "flashblock.h"

int main(void) {
  /* 1 sequence, MHA 32 heads, d 128, prefix 4096, block 32 (host-only calls: the
     index arrays are not read, so host arrays serve) */
  static const int32_t cu_q[2] = {0, 32}, cu_out[2] = {0, 4096}, cu_in[2] = {0, 32};
  fb_problem p;
  memset(&p, 0, sizeof(p));
  p.num_seqs = 1; p.num_heads_q = 32; p.num_heads_kv = 32; p.head_dim = 128;
  p.softmax_scale = 0.08838834764831845f;
  p.cu_seqlens_q = cu_q; p.cu_seqlens_kv_out = cu_out; p.cu_seqlens_kv_in = cu_in;
  p.total_q = 32; p.total_kv_out = 4096; p.total_kv_in = 32;
  p.max_q = 32; p.max_kv_out = 4096; p.max_kv_in = 32;
  size_t ws = 0;
  if (fb_workspace_size(&p, &ws) != FB_OK) return 2;
  fb_plan_info info;
  if (fb_plan_query(&p, FB_CALL_STEP, &info) != FB_OK) return 3;
  p.head_dim = 96;
  if (fb_workspace_size(&p, &ws) != FB_ERR_UNSUPPORTED || strlen(fb_last_error()) == 0) return 4;
  printf("%d %zu %d %d %d\n", fb_version(), ws, info.kernel, info.work_items, info.ctas);
  return 0;
}
"""


def test_header_serves_a_plain_c_caller(tmp_path):
    """The boundary is C: a C99 program includes flashblock.h, links the library and
    makes host-only calls (no GPU needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = _built()
    src = tmp_path / "caller.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(lib)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-L", libdir, "-lflashblock", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    version, ws, kernel, items, ctas = map(int, r.stdout.split())
    assert version >= 100 and ws == 512 and kernel == 0 and items == 32 and ctas == 128


def test_host_checks_hold_for_any_problem_fields():
    """Random (also absurd) fb_problem fields: the host-only calls answer OK or an
    argument/unsupported error, never crash; an accepted problem's workspace holds
    the counter slot and one fp32 score per (sequence, q-head), and its plan's grid
    is work items x splits."""
    from hypothesis import given, settings
    from hypothesis import strategies as st
    _built()
    from cached_split_attention_b200 import binding as B
    i32 = st.one_of(st.integers(-3, 70), st.integers(0, 1 << 20),
                    st.sampled_from([2 ** 31 - 1, -2 ** 31, 2 ** 30, 600_000_000, 1 << 16]))

    @settings(max_examples=400, deadline=None)
    @given(ns=i32, hq=i32, hkv=st.sampled_from([1, 2, 4, 8, 0, -1]), d=st.sampled_from([64, 128, 96]), tq=i32,
           to=i32, ti=i32, mq=i32, mo=i32, mi=i32, sp=st.integers(-1, 20), call=st.integers(-1, 3))
    def check(ns, hq, hkv, d, tq, to, ti, mq, mo, mi, sp, call):
        p = B.FbProblem(ns, hq, hkv, d, 0.1, 16, 0, 16, 16, tq, to, ti, mq, mo, mi, sp)
        n = ctypes.c_size_t()
        rc = B._lib.fb_workspace_size(ctypes.byref(p), ctypes.byref(n))
        assert rc in (B.OK, B.ERR_INVALID_ARG, B.ERR_UNSUPPORTED)
        if rc == B.OK:
            assert n.value >= 256 + 4 * ns * hq, (ns, hq, n.value)
        info = B.FbPlanInfo()
        rc = B._lib.fb_plan_query(ctypes.byref(p), call, ctypes.byref(info))
        assert rc in (B.OK, B.ERR_INVALID_ARG, B.ERR_UNSUPPORTED)
        if rc == B.OK:
            assert info.ctas == info.work_items * info.splits >= 0 and 1 <= info.splits <= 16

    check()
    # the overflow this guards against: 600M sequences x 4 heads
    big = _problem(B, num_seqs=600_000_000, num_heads_q=4, num_heads_kv=4, total_q=0, max_q=0, total_kv_in=0,
                   max_kv_in=0, total_kv_out=0, max_kv_out=0)
    n = ctypes.c_size_t()
    assert B._lib.fb_workspace_size(ctypes.byref(big), ctypes.byref(n)) == B.ERR_UNSUPPORTED
