"""fb_step_noalloc: fb_step for callers that cannot allocate device memory.

Some integrations cannot give the library a workspace (their framework's
allocator owns all device memory, or allocating inside the step loop is not
acceptable).  fb_step_noalloc serves them from a fixed scratch array built into
the library.  These tests call it through the C ABI and check it against the
ordinary fb_step (which takes a caller workspace, bit for bit) and against the
fp64 oracle on two calls in a row -- a recompute step and a reuse step -- and
check that problems needing more scratch than the built-in array are refused with
a clear message.

This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from cached_split_attention_b200 import workloads as W
from gpu_util import assert_close, bf16_to_f64_torch, torch_and_binding


def _run(B, torch, w, use_noalloc):
    p0 = w.problem
    cache = B.Cache(p0, "cuda", with_q_ref=True)
    k_out, v_out = B.bf16_tensor(w.k_out), B.bf16_tensor(w.v_out)
    prm = B.params(w.tau, w.gamma, w.flags)
    ws = None if use_noalloc else B.alloc_workspace(B.DeviceProblem(p0))
    outs = []
    for st in w.steps:  # two calls in a row
        p = st.problem
        dp = B.DeviceProblem(p)
        args = (dp, prm, cache, B.bf16_tensor(st.q), B.bf16_tensor(st.k_in), B.bf16_tensor(st.v_in), k_out, v_out,
                torch.as_tensor(st.n_updated).cuda())
        a = torch.full((p.total_q, p.num_heads_q, p.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
        l = torch.full((p.total_q, p.num_heads_q), float("nan"), device="cuda")
        dec = torch.full((p.num_seqs, p.num_heads_q), 7, dtype=torch.uint8, device="cuda")
        if use_noalloc:
            B.step_noalloc(*args, a, l_full=l, decision_out=dec)
        else:
            B.step(*args, a, ws, l_full=l, decision_out=dec)
        torch.cuda.synchronize()
        outs.append((bf16_to_f64_torch(a), l.double().cpu().numpy(), dec.cpu().numpy()))
    assert B.device_status() == 0
    return outs


@pytest.mark.gpu
@pytest.mark.parametrize("make", [lambda: W.dllm_layer(steps=2),
                                  lambda: W.locking_tiny(steps=2),
                                  lambda: W.video(steps=2, block=300, prefix_blocks=1, heads=4)],
                         ids=["dllm_layer", "locking_gqa", "video_block_two_tile"])
def test_noalloc_matches_fb_step_and_the_oracle(make):
    """Two calls in a row (a recompute step, then a reuse step): fb_step_noalloc
    gives exactly the bits of fb_step -- the same plan and kernels run on the same
    inputs, and the fused path is deterministic (fixed reduction orders, no atomics
    on the data) -- and, compared with the fp64 oracle applying the same policy,
    stays within the tolerances of every other test (A max-abs 2e-2, mean-abs
    1e-3; L 1e-3; decisions bit-exact)."""
    from oracle import policy
    torch, B = torch_and_binding()
    w = make()
    ref = _run(B, torch, w, use_noalloc=False)
    got = _run(B, torch, w, use_noalloc=True)
    orc = policy.run_policy(w)
    for s, ((a0, l0, d0), (a1, l1, d1), r) in enumerate(zip(ref, got, orc)):
        assert np.array_equal(d0, d1), f"step {s}: decisions differ from fb_step"
        assert np.array_equal(a1, a0), f"step {s}: A_full differs from fb_step"
        assert np.array_equal(l1, l0), f"step {s}: L_full differs from fb_step"
        assert np.array_equal(d1.astype(bool), r.recompute), f"step {s}: decisions differ from the oracle"
        assert_close(a1, r.a_full, l1, r.l_full, f"{w.name} no-alloc step {s}")
    # step 0 recomputes (empty cache); step 1 reuses for at least one head
    assert ref[0][2].all() and not orc[1].recompute.all()


def test_noalloc_refuses_oversize_problems():
    """A problem whose scratch would exceed the built-in 64 KiB is refused before
    any device work (no GPU needed)."""
    from cached_split_attention_b200 import binding as B
    prob = B.FbProblem(600, 32, 32, 128, 0.088, 16, 0, 16, 16, 600 * 32, 4096, 600 * 32, 32, 64, 32, 0)
    prm = B.params(4, 0.0, B.GATE_TAU)
    cache = B.FbCache(16, 16, 16, 0)
    rc = B._lib.fb_step_noalloc(ctypes.byref(prob), ctypes.byref(prm), ctypes.byref(cache), 16, 16, 16, 16, 16, 16,
                                None, 16, 16, None, None)
    assert rc == B.ERR_UNSUPPORTED
    msg = B._lib.fb_noalloc_last_error().decode()
    assert "scratch" in msg and "65536" in msg, msg
